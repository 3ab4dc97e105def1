// attn_tc.cu — tensor-core (tcgen05) attention for 16-bit storage, head dim 64,
// forward and backward.  The S x S score matrix never reaches HBM.
//
// Computes, per (sequence b, head h), with d = 64 and c = 1/sqrt(d):
//   S = Q K^T * c + mask_b (additive over keys); P = softmax over keys;
//   Pd = P * keep / (1 - p) (dropout on the probabilities, site 0);
//   ctx = Pd V, heads merged into (B*S, H); LSE per row kept for backward.
// ("Transformer deployment", section 1 pseudo-code: softmax(Q K^T / sqrt(d_k))
// then the product with V; "DeepSpeed Transformer Kernel usage guide", Step 3:
// the attention-dropout input is not stored, backward regenerates it.)
// Backward regenerates P from LSE and the dropout bits from Philox:
//   dV = Pd^T dO; dPd = dO V^T; dP = dPd * keep / (1 - p);
//   dS = P * (dP - D) with D = rowsum(dO * O); dQ = dS K c; dK = dS^T Q c.
//
// Tiles are 128 queries x 128 keys.  One elected thread issues every MMA
// (M = 128) into TMEM; softmax warps own one TMEM lane (one query row) each,
// so each thread's dropout bits are its own row's Philox draws.  P and dS go
// back to shared memory in the 128-byte-swizzled layout TMA uses for a
// [rows][64] tile, which serves as a K-major operand (rows x keys) and as an
// MN-major operand (keys x rows) alike; Q, K, V and dO tiles likewise serve
// both roles without any transpose.  TMA loads are per CTA (no multicast).
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>

#include <algorithm>
#include <type_traits>

#include "kernels.h"
#include "profile.h"
#include "sm100.cuh"

namespace tlp {

using namespace sm100;

// D = rowsum(dO * O) per (b, h, query), attn_simt.cu.
void dvec_launch(int dt, const AttnArgs& a, cudaStream_t s);

namespace {

constexpr int HD = 64;                  // head dim served here
constexpr int TILE = 128;               // queries or keys per tile
constexpr int TB = TILE * HD * 2;       // bytes of one [128][64] 16-bit tile (16 KB)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct AttnTc {
  int B, S, nh, H;
  const float* mask;
  float scale;          // 1/sqrt(d)
  DropoutParams drop;
  void* ctx;
  float* lse;
  const void* ctx_in;   // backward: forward output O (for D)
  const void* dctx;
  const float* dvec;    // precomputed D, or null to compute it in-kernel
  void* dqkv;
  float* colsum;        // fused QKV bias-gradient partials (persistent backward), or null
  int fuse_dq;
  int ctx_tma;          // persistent kernels: ctx (forward) or dQKV (backward) rows leave by TMA store (S % 32 == 0)
  uint8_t* keep;        // attention keep bits (forward writes, backward reads) or null: persistent path
                        // [B*nh][128][16]; longer sequences flat, byte e/8 for element e of site 0
  int bf16;
  int* err;
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Descriptors of a [128 rows][64] swizzled tile at `base` (K-major operand:
// rows x 64, K step kk of 16 columns) and of a [128 rows][128] pair of such
// tiles (regions of 16 KB holding columns 0-63 and 64-127).
__device__ __forceinline__ uint64_t dk_tile(uint32_t base, int kk) { return smem_desc_sw128(base + kk * 32, 16, 1024); }
__device__ __forceinline__ uint64_t dk_pair(uint32_t base, int kk) {
  return smem_desc_sw128(base + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
}
// MN-major views (K runs along the rows, 16 rows per step): a single tile
// (64 MN elements) or a pair (128 MN elements, second 64 at +16 KB).
__device__ __forceinline__ uint64_t dmn_tile(uint32_t base, int kk) { return smem_desc_sw128(base + kk * 2048, 8192, 1024); }
__device__ __forceinline__ uint64_t dmn_pair(uint32_t base, int kk) { return smem_desc_sw128(base + kk * 2048, 16384, 1024); }

// Stores 8 values as the 8-element chunk k8 (0..15) of row r of a
// [128][128] swizzled pair.
template <typename T>
__device__ __forceinline__ void pair_store8(uint8_t* pair, int r, int k8, const float (&v)[8]) {
  const int region = k8 >> 3, c = k8 & 7;
  store8<T>(reinterpret_cast<T*>(pair + region * 16384 + r * 128 + ((c ^ (r & 7)) << 4)), v);
}

__device__ __forceinline__ float mask_log2(const AttnTc& a, int b, int key) {
  if (key >= a.S) return -INFINITY;
  return a.mask ? a.mask[(size_t)b * a.S + key] * kLog2e : 0.0f;
}
// The additive mask of keys key0 .. key0+7 (key0 % 8 == 0, S % 8 == 0), in
// log2 units: two 16-byte loads that every lane of a warp shares.
__device__ __forceinline__ void mask8_log2(const AttnTc& a, int b, int key0, float (&m)[8]) {
  if (key0 >= a.S) {
#pragma unroll
    for (int t = 0; t < 8; ++t) m[t] = -INFINITY;
  } else if (!a.mask) {
#pragma unroll
    for (int t = 0; t < 8; ++t) m[t] = 0.0f;
  } else {
    const float4* p = reinterpret_cast<const float4*>(a.mask + (size_t)b * a.S + key0);
    const float4 u = __ldg(p), v = __ldg(p + 1);
    m[0] = u.x * kLog2e; m[1] = u.y * kLog2e; m[2] = u.z * kLog2e; m[3] = u.w * kLog2e;
    m[4] = v.x * kLog2e; m[5] = v.y * kLog2e; m[6] = v.z * kLog2e; m[7] = v.w * kLog2e;
  }
}

// One past the last key of sequence b whose additive mask is not -inf (S
// without a mask), found by the whole block.  Key tiles at or beyond it hold
// only masked keys: their probabilities are exactly 0 (2^-inf), so they add
// nothing to any row sum, output or gradient, and the long-sequence kernels
// skip them ("AI-infra engineers and the Transformer", section 2.1 Step 4:
// dynamic padding keeps padded positions out of the work).  Call after
// pdl_wait, from every thread of the block.
__device__ __forceinline__ int key_extent(const AttnTc& a, int b) {
  if (!a.mask) return a.S;
  __shared__ int ext;
  if (threadIdx.x == 0) ext = 0;
  __syncthreads();
  int e = 0;
  for (int j = threadIdx.x; j < a.S; j += blockDim.x)
    if (a.mask[(size_t)b * a.S + j] != -INFINITY) e = j + 1;
  if (e) atomicMax(&ext, e);
  __syncthreads();
  return ext;
}

// ============================================================================ forward
// Warps: 0 TMA, 1 MMA (+TMEM owner), 2-5 softmax (thread = query row).
constexpr int kFwdThreads = 192;
constexpr int kFwdSmem = 5 * TB + 1024 + 256;   // Q, K, V, P pair

template <typename T>
__global__ void __launch_bounds__(kFwdThreads)
    attn_fwd_tc(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                const __grid_constant__ CUtensorMap tv, AttnTc a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  uint8_t* sQ = sm;
  uint8_t* sK = sm + TB;
  uint8_t* sV = sm + 2 * TB;
  uint8_t* sP = sm + 3 * TB;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + 5 * TB);
  uint64_t *q_full = bar, *kv_full = bar + 1, *kv_empty = bar + 2, *s_full = bar + 3, *s_free = bar + 4,
           *p_full = bar + 5, *o_full = bar + 6, *o_free = bar + 7;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar + 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y, b = blockIdx.z;
  const int S = a.S;
  const int row0 = (b * a.nh + h) * S;
  const int q0 = blockIdx.x * TILE;
  const int ntiles_all = (S + TILE - 1) / TILE;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1);
    mbar_init(s_full, 1);
    mbar_init(s_free, 128);
    mbar_init(p_full, 128);
    mbar_init(o_full, 1);
    mbar_init(o_free, 128);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tslot, 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  pdl_wait();
  pdl_launch_dependents();
  const uint32_t tS = tmem, tO = tmem + 128;
  // key tiles past the last unmasked key are skipped (at least one is run,
  // so a fully masked row still ends with its zero output)
  const int ntiles = max(1, min(ntiles_all, (key_extent(a, b) + TILE - 1) / TILE));

  if (warp == 0) {
    if (lane == 0) {
      bool ok = true;
      mbar_arrive_expect_tx(q_full, TB);
      tma_load_2d(sQ, &tq, q_full, 0, row0 + q0);
      int j = 0;
      for (; j < ntiles; ++j) {
        if (!mbar_wait(kv_empty, (j & 1) ^ 1, a.err, 11)) { ok = false; break; }
        mbar_arrive_expect_tx(kv_full, 2 * TB);
        tma_load_2d(sK, &tk, kv_full, 0, row0 + j * TILE);
        tma_load_2d(sV, &tv, kv_full, 0, row0 + j * TILE);
      }
      if (!ok) {
        mbar_wait(q_full, 0, nullptr, 0);
        if (j > 0) mbar_wait(kv_full, (j - 1) & 1, nullptr, 0);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id_s = idesc_f16(128, 128, a.bf16 != 0, false, false);
      const uint32_t id_o = idesc_f16(128, 64, a.bf16 != 0, false, true);
      const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV), aP = smem_u32(sP);
      if (mbar_wait(q_full, 0, a.err, 12)) {
        for (int j = 0; j < ntiles; ++j) {
          if (!mbar_wait(kv_full, j & 1, a.err, 13)) break;
          if (!mbar_wait(s_free, (j & 1) ^ 1, a.err, 14)) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) mma_f16(tS, dk_tile(aQ, kk), dk_tile(aK, kk), id_s, kk > 0);
          mma_commit(s_full);
          if (!mbar_wait(p_full, j & 1, a.err, 15)) break;
          if (!mbar_wait(o_free, (j & 1) ^ 1, a.err, 16)) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < TILE / 16; ++kk) mma_f16(tO, dk_pair(aP, kk), dmn_tile(aV, kk), id_o, kk > 0);
          mma_commit(o_full);
          mma_commit(kv_empty);
        }
      }
    }
  } else {
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int i = q0 + r;
    const uint32_t lo = (uint32_t)(quarter * 32) << 16;
    const float c2 = a.scale * kLog2e;
    const float dsc = a.drop.thr ? a.drop.scale : 1.0f;
    const uint64_t erow = ((uint64_t)row0 + (uint64_t)i) * (uint64_t)S;
    const bool row_ok = i < S;
    float o[HD];
#pragma unroll
    for (int c = 0; c < HD; ++c) o[c] = 0.0f;
    float m = -INFINITY, l = 0.0f, alpha_prev = 0.0f;
    bool ok = true;
    for (int j = 0; j < ntiles && ok; ++j) {
      const int k0 = j * TILE;
      if (!mbar_wait_warp(s_full, j & 1, a.err, 17)) { ok = false; break; }
      tc_fence_after();
      // pass 1: row maximum of the scaled, masked scores (log2 domain)
      float mx = -INFINITY;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float sv[32];
        tmem_ld32(tS + lo + c * 32, sv);
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          float ml[8];
          mask8_log2(a, b, k0 + c * 32 + g * 8, ml);
#pragma unroll
          for (int t = 0; t < 8; ++t) mx = fmaxf(mx, fmaf(sv[g * 8 + t], c2, ml[t]));
        }
      }
      const float m_new = fmaxf(m, mx);
      const float alpha = (m == -INFINITY) ? 0.0f : exp2f(m - m_new);
      // the P buffer and O_part of the previous tile must be consumed first
      if (j > 0) {
        if (!mbar_wait_warp(o_full, (j - 1) & 1, a.err, 18)) { ok = false; break; }
        tc_fence_after();
        float pv[32];
        tmem_ld32(tO + lo, pv);
#pragma unroll
        for (int c = 0; c < 32; ++c) o[c] = fmaf(o[c], alpha_prev, pv[c]);
        tmem_ld32(tO + lo + 32, pv);
#pragma unroll
        for (int c = 0; c < 32; ++c) o[32 + c] = fmaf(o[32 + c], alpha_prev, pv[c]);
        tc_fence_before();
        mbar_arrive(o_free);
      }
      // pass 2: probabilities, dropout, P to shared memory; the keep bits are
      // also written out for the backward (byte e/8 of site 0, e the flat index)
      float lsum = 0.0f;
      const float msub = m_new == -INFINITY ? 0.0f : m_new;   // 2^(-inf - msub) = 0
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float sv[32];
        tmem_ld32(tS + lo + c * 32, sv);
        uint32_t kw = 0xFFFFFFFFu;
        if (a.drop.thr) {
          const uint64_t e8 = (erow + (uint64_t)(k0 + c * 32)) >> 3;
          kw = 0;
#pragma unroll
          for (int g = 0; g < 4; ++g) kw |= dropout_bits8(a.drop, 0, e8 + g) << (8 * g);
          if (a.keep && row_ok) {
            // a 32-bit word when it is 4-byte aligned (S % 32 == 0), else bytes
            if ((e8 & 3) == 0) {
              *reinterpret_cast<uint32_t*>(a.keep + e8) = kw;
            } else {
#pragma unroll
              for (int g = 0; g < 4; ++g) a.keep[e8 + g] = (uint8_t)(kw >> (8 * g));
            }
          }
        }
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int kb = k0 + c * 32 + g * 8;
          const uint32_t bits = (kw >> (8 * g)) & 0xFFu;
          float ml[8];
          mask8_log2(a, b, kb, ml);
          float pv[8];
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            const float p = ex2_approx(fmaf(sv[g * 8 + t], c2, ml[t]) - msub);
            lsum += p;
            pv[t] = ((bits >> t) & 1u) ? p * dsc : 0.0f;
          }
          pair_store8<T>(sP, r, c * 4 + g, pv);
        }
      }
      tc_fence_before();
      mbar_arrive(s_free);
      fence_proxy_async_smem();
      mbar_arrive(p_full);
      l = l * alpha + lsum;
      m = m_new;
      alpha_prev = alpha;
    }
    if (ok && mbar_wait_warp(o_full, (ntiles - 1) & 1, a.err, 19)) {
      tc_fence_after();
      float pv[32];
      tmem_ld32(tO + lo, pv);
#pragma unroll
      for (int c = 0; c < 32; ++c) o[c] = fmaf(o[c], alpha_prev, pv[c]);
      tmem_ld32(tO + lo + 32, pv);
#pragma unroll
      for (int c = 0; c < 32; ++c) o[32 + c] = fmaf(o[32 + c], alpha_prev, pv[c]);
      if (i < S) {
        const float inv = l > 0.0f ? 1.0f / l : 0.0f;
        T* dst = static_cast<T*>(a.ctx) + ((size_t)b * S + i) * a.H + h * HD;
#pragma unroll
        for (int c = 0; c < HD; c += 8) {
          float v[8];
#pragma unroll
          for (int t = 0; t < 8; ++t) v[t] = o[c + t] * inv;
          store8<T>(dst + c, v);
        }
        a.lse[row0 + i] = l > 0.0f ? (m + log2f(l)) * kLn2 : INFINITY;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 256);
}

// ============================================================================ backward
// Warps: 0 TMA, 1 MMA (+TMEM owner), 2-9 softmax: warp w serves TMEM lanes
// 32*(w%4).. and key columns 64*((w-2)/4) .. +63 of each 128-key tile.
constexpr int kBwdThreads = 320;
constexpr int kSoftThreads = 256;

// Per-thread D_i = sum_c dO[i, c] O[i, c] (from global memory).
template <typename T>
__device__ __forceinline__ float dvec_row(const AttnTc& a, int b, int h, int i) {
  const size_t off = ((size_t)b * a.S + i) * a.H + h * HD;
  const T* dO = static_cast<const T*>(a.dctx) + off;
  const T* O = static_cast<const T*>(a.ctx_in) + off;
  float s = 0.0f;
#pragma unroll
  for (int c = 0; c < HD; c += 8) {
    float x[8], y[8];
    load8<T>(dO + c, x);
    load8<T>(O + c, y);
#pragma unroll
    for (int t = 0; t < 8; ++t) s = fmaf(x[t], y[t], s);
  }
  return s;
}

// Softmax-side work of one (query tile, key tile) pair for one thread: row r
// of the tile (query i), key columns [kc0, kc0 + 64) of the tile starting at
// key k0.  Writes Pd (if sPd) and dS rows to shared memory.
template <typename T>
__device__ __forceinline__ void bwd_pair_rows(const AttnTc& a, int b, int row0, int i, int r, int k0, int kc0,
                                              uint32_t tS, uint32_t tdP, uint32_t lo, float lse2, float Di,
                                              uint8_t* sPd, uint8_t* sdS) {
  const float c2 = a.scale * kLog2e;
  const float dsc = a.drop.thr ? a.drop.scale : 1.0f;
  const uint64_t erow = ((uint64_t)row0 + (uint64_t)i) * (uint64_t)a.S;
  const bool row_ok = i < a.S;
#pragma unroll 1
  for (int c = 0; c < 2; ++c) {
    float sv[32], dv[32];
    tmem_ld32(tS + lo + kc0 + c * 32, sv);
    tmem_ld32(tdP + lo + kc0 + c * 32, dv);
    // the forward's keep bits of these 32 keys (one 32-bit word), or drawn again
    uint32_t kw = 0xFFFFFFFFu;
    if (a.drop.thr) {
      const uint64_t e8 = (erow + (uint64_t)(k0 + kc0 + c * 32)) >> 3;
      if (a.keep) {
        if (!row_ok) {
          kw = 0u;
        } else if ((e8 & 3) == 0) {
          kw = __ldg(reinterpret_cast<const uint32_t*>(a.keep + e8));
        } else {
          kw = 0u;
#pragma unroll
          for (int g = 0; g < 4; ++g) kw |= (uint32_t)__ldg(a.keep + e8 + g) << (8 * g);
        }
      } else {
        kw = 0;
#pragma unroll
        for (int g = 0; g < 4; ++g) kw |= dropout_bits8(a.drop, 0, e8 + g) << (8 * g);
      }
    }
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const int kt = kc0 + c * 32 + g * 8;   // column within the key tile
      const int kb = k0 + kt;
      const uint32_t bits = (kw >> (8 * g)) & 0xFFu;
      float ml[8];
      mask8_log2(a, b, kb, ml);
      float pd[8], ds[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        // lse2 = +inf for rows past the sequence end: 2^-inf = 0
        const float p = ex2_approx(fmaf(sv[g * 8 + t], c2, ml[t]) - lse2);
        const bool keep = (bits >> t) & 1u;
        pd[t] = keep ? p * dsc : 0.0f;
        const float dp = keep ? dv[g * 8 + t] * dsc : 0.0f;
        ds[t] = p * (dp - Di);
      }
      if (sPd) pair_store8<T>(sPd, r, kt >> 3, pd);
      pair_store8<T>(sdS, r, kt >> 3, ds);
    }
  }
}

// Key-tile CTA: dK, dV of 128 keys accumulated over every query tile; with
// fuse_dq (one key tile covers the sequence) also dQ of each query tile.
constexpr int kBwdKvSmem = 8 * TB + 1024 + 256;   // K, V, Q[2], dO... see layout below

template <typename T>
__global__ void __launch_bounds__(kBwdThreads)
    attn_bwd_kv_tc(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                   const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo, AttnTc a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  uint8_t* sK = sm;
  uint8_t* sV = sm + TB;
  uint8_t* sQ = sm + 2 * TB;    // one stage: Q then dO
  uint8_t* sdO = sm + 3 * TB;
  uint8_t* sPd = sm + 4 * TB;   // pair
  uint8_t* sdS = sm + 6 * TB;   // pair
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + 8 * TB);
  uint64_t *kv_full = bar, *qd_full = bar + 1, *qd_empty = bar + 2, *s_full = bar + 3, *s_free = bar + 4,
           *ds_full = bar + 5, *ds_free = bar + 6, *dq_full = bar + 7, *dq_free = bar + 8, *acc_full = bar + 9;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar + 10);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y, b = blockIdx.z;
  const int S = a.S;
  const int row0 = (b * a.nh + h) * S;
  const int k0 = blockIdx.x * TILE;
  const int nq_all = (S + TILE - 1) / TILE;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(qd_full, 1);
    mbar_init(qd_empty, 1);
    mbar_init(s_full, 1);
    mbar_init(s_free, kSoftThreads);
    mbar_init(ds_full, kSoftThreads);
    mbar_init(ds_free, 1);
    mbar_init(dq_full, 1);
    mbar_init(dq_free, kSoftThreads);
    mbar_init(acc_full, 1);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tslot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  pdl_wait();
  pdl_launch_dependents();
  const uint32_t tS = tmem, tdP = tmem + 128, tdV = tmem + 256, tdK = tmem + 320, tdQ = tmem + 384;
  // every key of this tile masked: no query attends to them, dK = dV = 0
  // exactly (this CTA runs no product; dQ never comes from here then, since
  // fuse_dq needs one key tile that covers the sequence)
  const bool keys_masked = !a.fuse_dq && k0 >= key_extent(a, b);
  const int nq = keys_masked ? 0 : nq_all;
  if (keys_masked && warp >= 2) {
    const int sw = warp - 2, quarter = warp & 3, half = sw >> 2;
    const int key = k0 + quarter * 32 + lane;
    if (key < S) {
      T* dst = static_cast<T*>(a.dqkv) + ((size_t)b * S + key) * 3 * a.H + h * HD + half * 32;
      const float z[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
      for (int c = 0; c < 32; c += 8) {
        store8<T>(dst + a.H + c, z);
        store8<T>(dst + 2 * a.H + c, z);
      }
    }
  }

  if (keys_masked) {
    // nothing is loaded or multiplied
  } else if (warp == 0) {
    if (lane == 0) {
      bool ok = true;
      mbar_arrive_expect_tx(kv_full, 2 * TB);
      tma_load_2d(sK, &tk, kv_full, 0, row0 + k0);
      tma_load_2d(sV, &tv, kv_full, 0, row0 + k0);
      int i = 0;
      for (; i < nq; ++i) {
        if (!mbar_wait(qd_empty, (i & 1) ^ 1, a.err, 21)) { ok = false; break; }
        mbar_arrive_expect_tx(qd_full, 2 * TB);
        tma_load_2d(sQ, &tq, qd_full, 0, row0 + i * TILE);
        tma_load_2d(sdO, &tdo, qd_full, h * HD, b * S + i * TILE);
      }
      if (!ok) {
        mbar_wait(kv_full, 0, nullptr, 0);
        if (i > 0) mbar_wait(qd_full, (i - 1) & 1, nullptr, 0);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const bool bf = a.bf16 != 0;
      const uint32_t id_kk = idesc_f16(128, 128, bf, false, false);
      const uint32_t id_mm = idesc_f16(128, 64, bf, true, true);
      const uint32_t id_km = idesc_f16(128, 64, bf, false, true);
      const uint32_t aK = smem_u32(sK), aV = smem_u32(sV), aQ = smem_u32(sQ), adO = smem_u32(sdO);
      const uint32_t aPd = smem_u32(sPd), adS = smem_u32(sdS);
      bool ok = mbar_wait(kv_full, 0, a.err, 22);
      for (int i = 0; i < nq && ok; ++i) {
        if (!(ok = mbar_wait(qd_full, i & 1, a.err, 23))) break;
        if (!(ok = mbar_wait(s_free, (i & 1) ^ 1, a.err, 24))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) mma_f16(tS, dk_tile(aQ, kk), dk_tile(aK, kk), id_kk, kk > 0);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) mma_f16(tdP, dk_tile(adO, kk), dk_tile(aV, kk), id_kk, kk > 0);
        mma_commit(s_full);
        if (!(ok = mbar_wait(ds_full, i & 1, a.err, 25))) break;
        tc_fence_after();
        // dV += Pd^T dO ; dK += dS^T Q   (K runs over the 128 queries)
#pragma unroll
        for (int kk = 0; kk < TILE / 16; ++kk)
          mma_f16(tdV, dmn_pair(aPd, kk), dmn_tile(adO, kk), id_mm, (i > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < TILE / 16; ++kk)
          mma_f16(tdK, dmn_pair(adS, kk), dmn_tile(aQ, kk), id_mm, (i > 0 || kk > 0) ? 1u : 0u);
        if (a.fuse_dq) {
          if (!(ok = mbar_wait(dq_free, (i & 1) ^ 1, a.err, 26))) break;
          tc_fence_after();
          // dQ = dS K   (K runs over the 128 keys)
#pragma unroll
          for (int kk = 0; kk < TILE / 16; ++kk) mma_f16(tdQ, dk_pair(adS, kk), dmn_tile(aK, kk), id_km, kk > 0);
          mma_commit(dq_full);
        }
        mma_commit(ds_free);
        mma_commit(qd_empty);
      }
      if (ok) mma_commit(acc_full);
    }
  } else {
    const int sw = warp - 2;
    const int quarter = warp & 3;
    const int half = sw >> 2;
    const int r = quarter * 32 + lane;
    const uint32_t lo = (uint32_t)(quarter * 32) << 16;
    bool ok = true;
    for (int i = 0; i < nq && ok; ++i) {
      const int q = i * TILE + r;
      const bool qv = q < S;
      const float lse2 = qv ? a.lse[row0 + q] * kLog2e : INFINITY;
      const float Di = qv ? (a.dvec ? a.dvec[row0 + q] : dvec_row<T>(a, b, h, q)) : 0.0f;
      if (!(ok = mbar_wait_warp(s_full, i & 1, a.err, 27))) break;
      tc_fence_after();
      if (!(ok = mbar_wait_warp(ds_free, (i & 1) ^ 1, a.err, 28))) break;
      bwd_pair_rows<T>(a, b, row0, q, r, k0, half * 64, tS, tdP, lo, lse2, Di, sPd, sdS);
      tc_fence_before();
      mbar_arrive(s_free);
      fence_proxy_async_smem();
      mbar_arrive(ds_full);
      if (a.fuse_dq) {
        if (!(ok = mbar_wait_warp(dq_full, i & 1, a.err, 29))) break;
        tc_fence_after();
        float v[32];
        tmem_ld32(tdQ + lo + half * 32, v);
        tc_fence_before();
        mbar_arrive(dq_free);
        if (qv) {
          T* dst = static_cast<T*>(a.dqkv) + ((size_t)b * S + q) * 3 * a.H + h * HD + half * 32;
#pragma unroll
          for (int c = 0; c < 32; c += 8) {
            float w8[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) w8[t] = v[c + t] * a.scale;
            store8<T>(dst + c, w8);
          }
        }
      }
    }
    if (ok && mbar_wait_warp(acc_full, 0, a.err, 30)) {
      tc_fence_after();
      const int key = k0 + r;
      float dv[32], dk[32];
      tmem_ld32(tdV + lo + half * 32, dv);
      tmem_ld32(tdK + lo + half * 32, dk);
      if (key < S) {
        T* dst = static_cast<T*>(a.dqkv) + ((size_t)b * S + key) * 3 * a.H + h * HD + half * 32;
#pragma unroll
        for (int c = 0; c < 32; c += 8) {
          float w8[8], u8[8];
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            w8[t] = dk[c + t] * a.scale;
            u8[t] = dv[c + t];
          }
          store8<T>(dst + a.H + c, w8);
          store8<T>(dst + 2 * a.H + c, u8);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// Query-tile CTA: dQ of 128 queries accumulated over every key tile (used
// when the sequence spans several key tiles).
constexpr int kBwdQSmem = 6 * TB + 1024 + 256;

template <typename T>
__global__ void __launch_bounds__(kBwdThreads)
    attn_bwd_q_tc(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                  const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo, AttnTc a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  uint8_t* sQ = sm;
  uint8_t* sdO = sm + TB;
  uint8_t* sK = sm + 2 * TB;
  uint8_t* sV = sm + 3 * TB;
  uint8_t* sdS = sm + 4 * TB;   // pair
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + 6 * TB);
  uint64_t *qd_full = bar, *kv_full = bar + 1, *kv_empty = bar + 2, *s_full = bar + 3, *s_free = bar + 4,
           *ds_full = bar + 5, *ds_free = bar + 6, *acc_full = bar + 7;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar + 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y, b = blockIdx.z;
  const int S = a.S;
  const int row0 = (b * a.nh + h) * S;
  const int q0 = blockIdx.x * TILE;
  const int nk_all = (S + TILE - 1) / TILE;

  if (threadIdx.x == 0) {
    mbar_init(qd_full, 1);
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1);
    mbar_init(s_full, 1);
    mbar_init(s_free, kSoftThreads);
    mbar_init(ds_full, kSoftThreads);
    mbar_init(ds_free, 1);
    mbar_init(acc_full, 1);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tslot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  pdl_wait();
  pdl_launch_dependents();
  const uint32_t tS = tmem, tdP = tmem + 128, tdQ = tmem + 256;
  // key tiles past the last unmasked key add nothing to dQ (at least one runs)
  const int nk = max(1, min(nk_all, (key_extent(a, b) + TILE - 1) / TILE));

  if (warp == 0) {
    if (lane == 0) {
      bool ok = true;
      mbar_arrive_expect_tx(qd_full, 2 * TB);
      tma_load_2d(sQ, &tq, qd_full, 0, row0 + q0);
      tma_load_2d(sdO, &tdo, qd_full, h * HD, b * S + q0);
      int j = 0;
      for (; j < nk; ++j) {
        if (!mbar_wait(kv_empty, (j & 1) ^ 1, a.err, 31)) { ok = false; break; }
        mbar_arrive_expect_tx(kv_full, 2 * TB);
        tma_load_2d(sK, &tk, kv_full, 0, row0 + j * TILE);
        tma_load_2d(sV, &tv, kv_full, 0, row0 + j * TILE);
      }
      if (!ok) {
        mbar_wait(qd_full, 0, nullptr, 0);
        if (j > 0) mbar_wait(kv_full, (j - 1) & 1, nullptr, 0);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const bool bf = a.bf16 != 0;
      const uint32_t id_kk = idesc_f16(128, 128, bf, false, false);
      const uint32_t id_km = idesc_f16(128, 64, bf, false, true);
      const uint32_t aK = smem_u32(sK), aV = smem_u32(sV), aQ = smem_u32(sQ), adO = smem_u32(sdO);
      const uint32_t adS = smem_u32(sdS);
      bool ok = mbar_wait(qd_full, 0, a.err, 32);
      for (int j = 0; j < nk && ok; ++j) {
        if (!(ok = mbar_wait(kv_full, j & 1, a.err, 33))) break;
        if (!(ok = mbar_wait(s_free, (j & 1) ^ 1, a.err, 34))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) mma_f16(tS, dk_tile(aQ, kk), dk_tile(aK, kk), id_kk, kk > 0);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) mma_f16(tdP, dk_tile(adO, kk), dk_tile(aV, kk), id_kk, kk > 0);
        mma_commit(s_full);
        if (!(ok = mbar_wait(ds_full, j & 1, a.err, 35))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < TILE / 16; ++kk)
          mma_f16(tdQ, dk_pair(adS, kk), dmn_tile(aK, kk), id_km, (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(ds_free);
        mma_commit(kv_empty);
      }
      if (ok) mma_commit(acc_full);
    }
  } else {
    const int sw = warp - 2;
    const int quarter = warp & 3;
    const int half = sw >> 2;
    const int r = quarter * 32 + lane;
    const uint32_t lo = (uint32_t)(quarter * 32) << 16;
    const int q = q0 + r;
    const bool qv = q < S;
    const float lse2 = qv ? a.lse[row0 + q] * kLog2e : INFINITY;
    const float Di = qv ? (a.dvec ? a.dvec[row0 + q] : dvec_row<T>(a, b, h, q)) : 0.0f;
    bool ok = true;
    for (int j = 0; j < nk && ok; ++j) {
      if (!(ok = mbar_wait_warp(s_full, j & 1, a.err, 36))) break;
      tc_fence_after();
      if (!(ok = mbar_wait_warp(ds_free, (j & 1) ^ 1, a.err, 37))) break;
      bwd_pair_rows<T>(a, b, row0, q, r, j * TILE, half * 64, tS, tdP, lo, lse2, Di, nullptr, sdS);
      tc_fence_before();
      mbar_arrive(s_free);
      fence_proxy_async_smem();
      mbar_arrive(ds_full);
    }
    if (ok && mbar_wait_warp(acc_full, 0, a.err, 38)) {
      tc_fence_after();
      float v[32];
      tmem_ld32(tdQ + lo + half * 32, v);
      if (qv) {
        T* dst = static_cast<T*>(a.dqkv) + ((size_t)b * S + q) * 3 * a.H + h * HD + half * 32;
#pragma unroll
        for (int c = 0; c < 32; c += 8) {
          float w8[8];
#pragma unroll
          for (int t = 0; t < 8; ++t) w8[t] = v[c + t] * a.scale;
          store8<T>(dst + c, w8);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ============================================================================ forward, S <= 128 (persistent)
// One CTA per SM walks (sequence, head) items; every item is one 128-query x
// 128-key tile.  Q/K/V, the score accumulator S and the output accumulator O
// are double-buffered by item parity, so item i+1's loads and Q K^T overlap
// item i's softmax.  Warps: 0 TMA, 1 MMA, 2-9 softmax in two groups of four
// (warps 2-5 take the even items of this CTA, warps 6-9 the odd ones, so two
// items are in their softmax at once); warp w owns TMEM lanes 32*(w%4), one
// thread per query row and all 128 keys of it (a first pass over the
// accumulator for the row maximum, a second for P), so no thread waits for
// another; the same group then writes the item's output rows.
// Warps 10-13 run ahead of the softmax by up to two items: per item they
// draw the dropout keep bits of all 128 x 128 elements (thread = query row,
// 16 Philox calls) and stage the item's additive key mask (log2 units, -inf
// past the sequence end), so the softmax threads only read them.
constexpr int kPFwdThreads = 448;
constexpr int kPFwdBits = 128 * 16;                      // keep bits of one item: [row][16 bytes]
constexpr int kPFwdMask = 128 * 4;                       // mask row of one item: [128] float
constexpr int kPFwdIn = 3;                               // Q/K/V input slots (loads run up to 3 items ahead)
constexpr int kPFwdSmem = (3 * kPFwdIn + 4) * TB + 2 * kPFwdBits + 2 * kPFwdMask + 1024 + 256;

__device__ __forceinline__ float ex2_fast(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
// Packed pairs of float32 (one instruction for both lanes on sm_100).
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;"
      : "=l"(d)
      : "l"(*reinterpret_cast<unsigned long long*>(&a)), "l"(*reinterpret_cast<unsigned long long*>(&b)),
        "l"(*reinterpret_cast<unsigned long long*>(&c)));
  return *reinterpret_cast<float2*>(&d);
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  unsigned long long d;
  asm("add.rn.f32x2 %0, %1, %2;"
      : "=l"(d)
      : "l"(*reinterpret_cast<unsigned long long*>(&a)), "l"(*reinterpret_cast<unsigned long long*>(&b)));
  return *reinterpret_cast<float2*>(&d);
}

template <typename T>
__global__ void __launch_bounds__(kPFwdThreads, 1)
    attn_fwd_tc_persist(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                        const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tctx,
                        AttnTc a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  // input slot i: Q at i*3TB, K at +TB, V at +2TB; then the two P pairs (by item parity)
  uint8_t* sP0 = sm + 3 * kPFwdIn * TB;
  uint8_t* sbits = sP0 + 4 * TB;                                          // [2][128][16]
  float* smask = reinterpret_cast<float*>(sbits + 2 * kPFwdBits);         // [2][128]
  uint64_t* bar = reinterpret_cast<uint64_t*>(sbits + 2 * kPFwdBits + 2 * kPFwdMask);
  uint64_t *in_full = bar, *in_empty = bar + kPFwdIn, *s_full = bar + 2 * kPFwdIn, *p_full = s_full + 2,
           *o_full = s_full + 4, *o_free = s_full + 6, *aux_full = s_full + 8, *aux_free = s_full + 10;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(s_full + 12);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = a.S;
  const int nitems = a.B * a.nh;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kPFwdIn; ++i) {
      mbar_init(&in_full[i], 1);
      mbar_init(&in_empty[i], 1);
    }
    for (int j = 0; j < 2; ++j) {
      mbar_init(&s_full[j], 1);
      mbar_init(&p_full[j], 128);
      mbar_init(&o_full[j], 1);
      mbar_init(&o_free[j], 128);
      mbar_init(&aux_full[j], 128);
      mbar_init(&aux_free[j], 128);
    }
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tslot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  pdl_wait();
  pdl_launch_dependents();   // S[j] at 128*j, O[j] at 256 + 64*j

  if (warp == 0) {
    if (lane == 0) {
      int n = 0;
      for (int it = blockIdx.x; it < nitems; it += gridDim.x, ++n) {
        const int i = n % kPFwdIn;
        if (!mbar_wait(&in_empty[i], ((n / kPFwdIn) & 1) ^ 1, a.err, 51)) break;
        uint8_t* base = sm + i * 3 * TB;
        mbar_arrive_expect_tx(&in_full[i], 3 * TB);
        const int row0 = it * S;
        tma_load_2d(base, &tq, &in_full[i], 0, row0);
        tma_load_2d(base + TB, &tk, &in_full[i], 0, row0);
        tma_load_2d(base + 2 * TB, &tv, &in_full[i], 0, row0);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id_s = idesc_f16(128, 128, a.bf16 != 0, false, false);
      const uint32_t id_o = idesc_f16(128, 64, a.bf16 != 0, false, true);
      // S = Q K^T of item n into S[n&1]
      auto mma_s = [&](int n) -> bool {
        const int j = n & 1, i = n % kPFwdIn;
        if (!mbar_wait(&in_full[i], (n / kPFwdIn) & 1, a.err, 52)) return false;
        // S[j] is free once the softmax of item n-2 wrote its P (it read S first)
        if (!mbar_wait(&p_full[j], ((n >> 1) & 1) ^ 1, a.err, 53)) return false;
        tc_fence_after();
        const uint32_t aQ = smem_u32(sm + i * 3 * TB), aK = aQ + TB;
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) mma_f16(tmem + 128 * j, dk_tile(aQ, kk), dk_tile(aK, kk), id_s, kk > 0);
        mma_commit(&s_full[j]);
        return true;
      };
      int n = 0;
      bool ok = true;
      int my_items = 0;
      for (int it = blockIdx.x; it < nitems; it += gridDim.x) ++my_items;
      if (my_items > 0) ok = mma_s(0);
      for (n = 0; n < my_items && ok; ++n) {
        const int j = n & 1;
        if (n + 1 < my_items && !(ok = mma_s(n + 1))) break;
        if (!(ok = mbar_wait(&p_full[j], (n >> 1) & 1, a.err, 54))) break;
        if (!(ok = mbar_wait(&o_free[j], ((n >> 1) & 1) ^ 1, a.err, 55))) break;
        tc_fence_after();
        const uint32_t aV = smem_u32(sm + (n % kPFwdIn) * 3 * TB) + 2 * TB;
        const uint32_t aP = smem_u32(sP0 + j * 2 * TB);
#pragma unroll
        for (int kk = 0; kk < TILE / 16; ++kk)
          mma_f16(tmem + 256 + 64 * j, dk_pair(aP, kk), dmn_tile(aV, kk), id_o, kk > 0);
        mma_commit(&o_full[j]);
        mma_commit(&in_empty[n % kPFwdIn]);
      }
    }
  } else if (warp >= 10) {
    // keep bits and mask row of each item, two items ahead at most
    const int r = threadIdx.x - 320;
    int n = 0;
    for (int it = blockIdx.x; it < nitems; it += gridDim.x, ++n) {
      const int j = n & 1;
      if (!mbar_wait(&aux_free[j], ((n >> 1) & 1) ^ 1, a.err, 58)) break;
      if (a.drop.thr) {
        const uint64_t e8 = (((uint64_t)it * S + (uint64_t)r) * (uint64_t)S) >> 3;
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t v = 0;
#pragma unroll
          for (int g = 0; g < 4; ++g) v |= dropout_bits8(a.drop, 0, e8 + (uint64_t)(q * 4 + g)) << (8 * g);
          w[q] = v;
        }
        const uint4 kv = make_uint4(w[0], w[1], w[2], w[3]);
        *reinterpret_cast<uint4*>(sbits + j * kPFwdBits + r * 16) = kv;
        if (a.keep) *reinterpret_cast<uint4*>(a.keep + ((size_t)it * 128 + r) * 16) = kv;
      }
      const int b = it / a.nh;
      smask[j * 128 + r] = r < S ? (a.mask ? a.mask[(size_t)b * S + r] * kLog2e : 0.0f) : -INFINITY;
      mbar_arrive(&aux_full[j]);
    }
  } else {
    // softmax group grp (0: warps 2-5, 1: warps 6-9) owns the items n with n % 2 == grp, slot j = grp
    const int quarter = warp & 3;
    const int grp = (warp - 2) >> 2;
    const int j = grp;
    const int r = quarter * 32 + lane;
    const uint32_t lo = (uint32_t)(quarter * 32) << 16;
    const float c2 = a.scale * kLog2e;
    const float dsc = a.drop.thr ? a.drop.scale : 1.0f;
    const float* mrow = smask + j * 128;
    // no mask and a full tile of keys: every mask value is 0
    const bool plain = a.mask == nullptr && S == TILE;
    // this warp's 32 output rows staged as one 32 x 128-byte swizzled box
    // inside the group's P pair (free between P V and the next item's P)
    uint8_t* ostage = sP0 + j * 2 * TB + quarter * 4096;
    int k = 0;   // this group's item count: item n = 2k + grp
    for (int it = blockIdx.x + grp * gridDim.x; it < nitems; it += 2 * gridDim.x, ++k) {
      const uint32_t par = k & 1;
      if (!mbar_wait_warp(&aux_full[j], par, a.err, 59)) break;
      const uint4 kb16 = a.drop.thr ? *reinterpret_cast<const uint4*>(sbits + j * kPFwdBits + r * 16)
                                    : make_uint4(~0u, ~0u, ~0u, ~0u);
      if (!mbar_wait_warp(&s_full[j], par, a.err, 57)) break;
      tc_fence_after();
      if (a.ctx_tma) {
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
      }
      const uint32_t ts = tmem + 128 * j + lo;
      // pass 1: row maximum over the 128 keys (scaled scores + mask, log2
      // units); without a mask (and S = 128) the maximum of the raw scores,
      // scaled once (c2 > 0)
      float mx = -INFINITY;
#pragma unroll 1
      for (int hh = 0; hh < 2; ++hh) {
        float sv[64];
        tmem_ld64(ts + hh * 64, sv);
        if (plain) {
#pragma unroll
          for (int t = 0; t < 64; t += 2) mx = max3f(mx, sv[t], sv[t + 1]);
        } else {
#pragma unroll
          for (int t = 0; t < 64; t += 4) {
            const float4 m4 = *reinterpret_cast<const float4*>(mrow + hh * 64 + t);
            const float2 x0 = fma2(make_float2(sv[t], sv[t + 1]), make_float2(c2, c2), make_float2(m4.x, m4.y));
            const float2 x1 = fma2(make_float2(sv[t + 2], sv[t + 3]), make_float2(c2, c2), make_float2(m4.z, m4.w));
            mx = max3f(mx, max3f(x0.x, x0.y, x1.x), x1.y);
          }
        }
      }
      if (plain) mx *= c2;
      // a row whose keys are all masked has mx = -inf: every p is 0
      const float msub = mx == -INFINITY ? 0.0f : mx;
      // pass 2: P = 2^(x - max), dropped, into the P tile; row sum of the undropped P
      float2 ls2 = make_float2(0.0f, 0.0f);
#pragma unroll 1
      for (int hh = 0; hh < 2; ++hh) {
        float sv[64];
        tmem_ld64(ts + hh * 64, sv);
        const uint32_t bw0 = hh == 0 ? kb16.x : kb16.z, bw1 = hh == 0 ? kb16.y : kb16.w;
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          const uint32_t bits = ((g < 4 ? bw0 : bw1) >> (8 * (g & 3))) & 0xFFu;
          float pv[8];
#pragma unroll
          for (int t = 0; t < 8; t += 2) {
            const int k = hh * 64 + g * 8 + t;
            float2 x;
            if (plain) {
              x = fma2(make_float2(sv[g * 8 + t], sv[g * 8 + t + 1]), make_float2(c2, c2), make_float2(-msub, -msub));
            } else {
              const float2 m2 = *reinterpret_cast<const float2*>(mrow + k);
              x = add2(fma2(make_float2(sv[g * 8 + t], sv[g * 8 + t + 1]), make_float2(c2, c2), m2),
                       make_float2(-msub, -msub));
            }
            const float2 p = make_float2(ex2_fast(x.x), ex2_fast(x.y));
            ls2 = add2(ls2, p);
            pv[t] = ((bits >> t) & 1u) ? p.x : 0.0f;
            pv[t + 1] = ((bits >> (t + 1)) & 1u) ? p.y : 0.0f;
          }
          pair_store8<T>(sP0 + j * 2 * TB, r, hh * 8 + g, pv);
        }
      }
      float lsum = ls2.x + ls2.y;
      mbar_arrive(&aux_free[j]);
      // P is written and S has been read: both hand-overs ride on p_full
      tc_fence_before();
      fence_proxy_async_smem();
      mbar_arrive(&p_full[j]);
      if (r < S) a.lse[(size_t)it * S + r] = lsum > 0.0f ? (mx + log2f(lsum)) * kLn2 : INFINITY;
      // this item's output rows once P V is in TMEM (P carried the keep
      // mask only; the dropout scale joins the normalisation here)
      const float inv = lsum > 0.0f ? dsc / lsum : 0.0f;
      if (!mbar_wait_warp(&o_full[j], par, a.err, 56)) break;
      tc_fence_after();
      float o[64];
      tmem_ld32(tmem + 256 + 64 * j + lo, *reinterpret_cast<float(*)[32]>(o));
      tmem_ld32(tmem + 256 + 64 * j + lo + 32, *reinterpret_cast<float(*)[32]>(o + 32));
      tc_fence_before();
      mbar_arrive(&o_free[j]);
      const int b = it / a.nh, h = it - (it / a.nh) * a.nh;
      if (a.ctx_tma) {
        // whole 32-row boxes (S % 32 == 0): swizzled smem rows, one TMA store per warp
        if (quarter * 32 < S) {
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            float w8[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) w8[t] = o[c * 8 + t] * inv;
            store8<T>(reinterpret_cast<T*>(ostage + lane * 128 + ((c ^ (lane & 7)) << 4)), w8);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tctx, ostage, h * HD, b * S + quarter * 32);
            bulk_commit();
          }
        }
      } else if (r < S) {
        T* dst = static_cast<T*>(a.ctx) + ((size_t)b * S + r) * a.H + h * HD;
#pragma unroll
        for (int c = 0; c < 64; c += 8) {
          float w8[8];
#pragma unroll
          for (int t = 0; t < 8; ++t) w8[t] = o[c + t] * inv;
          store8<T>(dst + c, w8);
        }
      }
    }
    if (a.ctx_tma && lane == 0) bulk_wait_all();
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ============================================================================ backward, S <= 128 (persistent)
// One CTA per SM walks (sequence, head) items, each one 128 x 128 tile:
// S = Q K^T and dPd = dO V^T, then Pd and dS to shared memory, then dV, dK and
// dQ in TMEM and out to dQKV.  Q/K/V/dO are double-buffered by item parity so
// the next item's loads overlap this item's work.  Warps 10-13 prepare each
// item ahead of the softmax warps: D = rowsum(dO * O) (dO from the item's
// shared tile, O from global memory), the row's log-sum-exp, the additive
// key mask and the dropout keep bits, all into shared memory.
constexpr int kPBwdThreads = 448;
constexpr int kPBwdAux = 128 * 16 + 3 * 128 * 4;          // bits [128][16], mask, lse2, D [128] floats
constexpr int kPBwdSmem = 12 * TB + 2 * kPBwdAux + 1024 + 256;   // (Q,K,V,dO) x2, Pd pair, dS pair, aux x2

template <typename T>
__global__ void __launch_bounds__(kPBwdThreads, 1)
    attn_bwd_tc_persist(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                        const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo,
                        const __grid_constant__ CUtensorMap tdqkv, AttnTc a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  uint8_t* sPd = sm + 8 * TB;
  uint8_t* sdS = sm + 10 * TB;
  uint8_t* saux = sm + 12 * TB;    // per slot: bits [128][16] | mask [128] | lse2 [128] | D [128]
  uint64_t* bar = reinterpret_cast<uint64_t*>(saux + 2 * kPBwdAux);
  uint64_t *in_full = bar, *in_empty = bar + 2, *s_full = bar + 4, *s_free = bar + 5, *ds_full = bar + 6,
           *g_full = bar + 7, *g_free = bar + 8, *aux_full = bar + 9, *aux_free = bar + 11;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar + 13);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = a.S;
  const int nitems = a.B * a.nh;
  if (threadIdx.x == 0) {
    for (int j = 0; j < 2; ++j) {
      mbar_init(&in_full[j], 1);
      mbar_init(&in_empty[j], 1);
      mbar_init(&aux_full[j], 128);
      mbar_init(&aux_free[j], kSoftThreads);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, kSoftThreads);
    mbar_init(ds_full, kSoftThreads);
    mbar_init(g_full, 1);
    mbar_init(g_free, kSoftThreads);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tslot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  pdl_wait();
  pdl_launch_dependents();
  const uint32_t tS = tmem, tdP = tmem + 128, tdV = tmem + 256, tdK = tmem + 320, tdQ = tmem + 384;

  if (warp == 0) {
    if (lane == 0) {
      int n = 0;
      for (int it = blockIdx.x; it < nitems; it += gridDim.x, ++n) {
        const int j = n & 1;
        if (!mbar_wait(&in_empty[j], ((n >> 1) & 1) ^ 1, a.err, 61)) break;
        uint8_t* base = sm + j * 4 * TB;
        const int b = it / a.nh, h = it - (it / a.nh) * a.nh;
        mbar_arrive_expect_tx(&in_full[j], 4 * TB);
        tma_load_2d(base, &tq, &in_full[j], 0, it * S);
        tma_load_2d(base + TB, &tk, &in_full[j], 0, it * S);
        tma_load_2d(base + 2 * TB, &tv, &in_full[j], 0, it * S);
        tma_load_2d(base + 3 * TB, &tdo, &in_full[j], h * HD, b * S);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const bool bf = a.bf16 != 0;
      const uint32_t id_kk = idesc_f16(128, 128, bf, false, false);
      const uint32_t id_mm = idesc_f16(128, 64, bf, true, true);
      const uint32_t id_km = idesc_f16(128, 64, bf, false, true);
      const uint32_t aPd = smem_u32(sPd), adS = smem_u32(sdS);
      int n = 0;
      for (int it = blockIdx.x; it < nitems; it += gridDim.x, ++n) {
        const int j = n & 1;
        const uint32_t aQ = smem_u32(sm + j * 4 * TB), aK = aQ + TB, aV = aQ + 2 * TB, adO = aQ + 3 * TB;
        if (!mbar_wait(&in_full[j], (n >> 1) & 1, a.err, 62)) break;
        if (!mbar_wait(s_free, (n & 1) ^ 1, a.err, 63)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) mma_f16(tS, dk_tile(aQ, kk), dk_tile(aK, kk), id_kk, kk > 0);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) mma_f16(tdP, dk_tile(adO, kk), dk_tile(aV, kk), id_kk, kk > 0);
        mma_commit(s_full);
        if (!mbar_wait(ds_full, n & 1, a.err, 64)) break;
        if (!mbar_wait(g_free, (n & 1) ^ 1, a.err, 65)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < TILE / 16; ++kk) mma_f16(tdV, dmn_pair(aPd, kk), dmn_tile(adO, kk), id_mm, kk > 0);
#pragma unroll
        for (int kk = 0; kk < TILE / 16; ++kk) mma_f16(tdK, dmn_pair(adS, kk), dmn_tile(aQ, kk), id_mm, kk > 0);
#pragma unroll
        for (int kk = 0; kk < TILE / 16; ++kk) mma_f16(tdQ, dk_pair(adS, kk), dmn_tile(aK, kk), id_km, kk > 0);
        mma_commit(g_full);
        mma_commit(&in_empty[j]);
      }
    }
  } else if (warp >= 10) {
    // per item: keep bits, mask row, lse2 and D of every query row
    const int r = threadIdx.x - 320;
    int n = 0;
    for (int it = blockIdx.x; it < nitems; it += gridDim.x, ++n) {
      const int j = n & 1;
      uint8_t* ax = saux + j * kPBwdAux;
      float* smask = reinterpret_cast<float*>(ax + 2048);
      if (!mbar_wait(&aux_free[j], ((n >> 1) & 1) ^ 1, a.err, 69)) break;
      if (a.drop.thr && a.keep) {
        // the forward's keep bits of this item
        *reinterpret_cast<uint4*>(ax + r * 16) =
            __ldg(reinterpret_cast<const uint4*>(a.keep + ((size_t)it * 128 + r) * 16));
      } else if (a.drop.thr) {
        const uint64_t e8 = (((uint64_t)it * S + (uint64_t)r) * (uint64_t)S) >> 3;
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t v = 0;
#pragma unroll
          for (int g = 0; g < 4; ++g) v |= dropout_bits8(a.drop, 0, e8 + (uint64_t)(q * 4 + g)) << (8 * g);
          w[q] = v;
        }
        *reinterpret_cast<uint4*>(ax + r * 16) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      const int b = it / a.nh, h = it - (it / a.nh) * a.nh;
      const bool qv = r < S;
      smask[r] = qv ? (a.mask ? a.mask[(size_t)b * S + r] * kLog2e : 0.0f) : -INFINITY;
      smask[128 + r] = qv ? a.lse[(size_t)it * S + r] * kLog2e : INFINITY;
      float Di = 0.0f;
      if (qv) {
        // O row from global memory first, then dO from the item's shared tile
        const T* orow = static_cast<const T*>(a.ctx_in) + ((size_t)b * S + r) * a.H + h * HD;
        Raw8<T> o8[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) o8[c] = raw8_load<T>(orow + c * 8);
        if (!mbar_wait(&in_full[j], (n >> 1) & 1, a.err, 70)) break;
        const uint8_t* drow = sm + j * 4 * TB + 3 * TB + r * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          float x[8], y[8];
          load8<T>(reinterpret_cast<const T*>(drow + ((c ^ (r & 7)) << 4)), x);
          raw8_unpack<T>(o8[c], y);
#pragma unroll
          for (int t = 0; t < 8; ++t) Di = fmaf(x[t], y[t], Di);
        }
      }
      smask[256 + r] = Di;
      mbar_arrive(&aux_full[j]);
    }
  } else {
    const int quarter = warp & 3;
    const int hf = (warp - 2) >> 2;
    const int r = quarter * 32 + lane;
    const uint32_t lo = (uint32_t)(quarter * 32) << 16;
    const float c2 = a.scale * kLog2e;
    const float dsc = a.drop.thr ? a.drop.scale : 1.0f;
    const int kc0 = hf * 64;
    // dQ, dK, dV rows of this warp staged as 32 x 64-byte swizzled boxes in
    // the warp's own rows of Pd and dS (free between the dV/dK/dQ products
    // and the next item's Pd, dS)
    uint8_t* stq = sPd + hf * 16384 + quarter * 4096;
    uint8_t* stv = sdS + hf * 16384 + quarter * 4096;
    const int swz = (lane >> 1) & 3;
    int n = 0;
    for (int it = blockIdx.x; it < nitems; it += gridDim.x, ++n) {
      const int j = n & 1;
      const int b = it / a.nh, h = it - (it / a.nh) * a.nh;
      const bool qv = r < S;
      const size_t trow = (size_t)b * S + r;
      const uint8_t* ax = saux + j * kPBwdAux;
      const float* smask = reinterpret_cast<const float*>(ax + 2048);
      if (!mbar_wait_warp(&aux_full[j], (n >> 1) & 1, a.err, 66)) break;
      const uint2 kb8 = a.drop.thr ? *reinterpret_cast<const uint2*>(ax + r * 16 + hf * 8)
                                   : make_uint2(0xFFFFFFFFu, 0xFFFFFFFFu);
      const float lse2 = smask[128 + r];
      const float Di = smask[256 + r];
      if (!mbar_wait_warp(s_full, n & 1, a.err, 67)) break;
      tc_fence_after();
      if (a.ctx_tma) {
        // the previous item's dQKV stores have read the staging rows
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
      }
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        float sv[32], dv[32];
        tmem_ld32(tS + lo + kc0 + c * 32, sv);
        tmem_ld32(tdP + lo + kc0 + c * 32, dv);
        const uint32_t bw = c == 0 ? kb8.x : kb8.y;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int kt = kc0 + c * 32 + g * 8;   // key column
          const uint32_t bits = (bw >> (8 * g)) & 0xFFu;
          const float4 m0 = *reinterpret_cast<const float4*>(smask + kt);
          const float4 m1 = *reinterpret_cast<const float4*>(smask + kt + 4);
          const float ml[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
          float pd[8], ds[8];
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            // lse2 = +inf for rows past the sequence end: p = 0
            const float p = ex2_fast(fmaf(sv[g * 8 + t], c2, ml[t]) - lse2);
            const bool keep = (bits >> t) & 1u;
            pd[t] = keep ? p * dsc : 0.0f;
            const float dp = keep ? dv[g * 8 + t] * dsc : 0.0f;
            ds[t] = p * (dp - Di);
          }
          pair_store8<T>(sPd, r, kt >> 3, pd);
          pair_store8<T>(sdS, r, kt >> 3, ds);
        }
      }
      mbar_arrive(&aux_free[j]);
      tc_fence_before();
      mbar_arrive(s_free);
      fence_proxy_async_smem();
      mbar_arrive(ds_full);
      if (!mbar_wait_warp(g_full, n & 1, a.err, 68)) break;
      tc_fence_after();
      // dQ, dK, dV one after another (w3 = 0, 1, 2): TMEM -> scale -> store
      // (staged for TMA, or direct) -> fused column sums
      const bool staged = a.ctx_tma && quarter * 32 < S;
#pragma unroll 1
      for (int w3 = 0; w3 < 3; ++w3) {
        float x[32];
        tmem_ld32(tdQ - 64 * w3 + lo + hf * 32, x);
        if (w3 == 2) {
          tc_fence_before();
          mbar_arrive(g_free);
        }
        if (w3 < 2) {
#pragma unroll
          for (int c = 0; c < 32; ++c) x[c] *= a.scale;
        }
        if (staged) {
          uint8_t* st = w3 == 0 ? stq : (w3 == 1 ? stq + 2048 : stv);
#pragma unroll
          for (int c = 0; c < 4; ++c)
            store8<T>(reinterpret_cast<T*>(st + lane * 64 + ((c ^ swz) << 4)), *reinterpret_cast<float(*)[8]>(x + c * 8));
        } else if (!a.ctx_tma && qv) {
          // row r is query r for dQ and key r for dK, dV (both < S)
          T* dst = static_cast<T*>(a.dqkv) + trow * 3 * a.H + w3 * a.H + h * HD + hf * 32;
#pragma unroll
          for (int c = 0; c < 32; c += 8) store8<T>(dst + c, *reinterpret_cast<float(*)[8]>(x + c));
        }
        if (a.colsum) {
          // QKV bias gradient fused in: column sums of the stored values over
          // this warp's 32 rows (rows past the sequence end count as zero)
#pragma unroll
          for (int c = 0; c < 32; ++c) x[c] = qv ? round_f<T>(x[c]) : 0.0f;
          a.colsum[(size_t)(b * 4 + quarter) * 3 * a.H + w3 * a.H + h * HD + hf * 32 + lane] = warp_colsum32(x);
        }
      }
      if (staged) {
        // three TMA stores per warp of whole 32-row boxes (S % 32 == 0)
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          const int x = h * HD + hf * 32, y = b * S + quarter * 32;
          tma_store_2d(&tdqkv, stq, x, y);
          tma_store_2d(&tdqkv, stq + 2048, x + a.H, y);
          tma_store_2d(&tdqkv, stv, x + 2 * a.H, y);
          bulk_commit();
        }
      }
    }
    if (a.ctx_tma && lane == 0) bulk_wait_all();
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// [rows][cols] row-major 16-bit matrix with row stride ld; box 64 x box_rows
// (128-byte swizzle), or 32 x box_rows (64-byte swizzle) with narrow.
bool map_tile(CUtensorMap* m, const void* p, bool bf16, uint64_t cols, uint64_t rows, uint64_t ld,
              uint32_t box_rows = 128, bool narrow = false) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {narrow ? 32u : 64u, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(p),
            dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            narrow ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Error word of the attention kernels' bounded waits (layout in sm100.cuh).
int* attn_error_word() {
  static int* p = nullptr;
  if (!p) cudaMalloc(&p, 4 * sizeof(int)), cudaMemset(p, 0, 4 * sizeof(int));
  return p;
}

AttnTc make_args(int dt, const AttnArgs& a) {
  AttnTc t;
  t.B = a.B; t.S = a.S; t.nh = a.nh; t.H = a.nh * a.d;
  t.mask = a.mask;
  t.scale = a.scale;
  t.drop = a.drop;
  t.ctx = a.ctx;
  t.lse = a.lse;
  t.ctx_in = a.ctx;
  t.dctx = a.dctx;
  t.dvec = nullptr;
  t.dqkv = a.dqkv;
  t.colsum = a.colsum;
  t.fuse_dq = 0;
  t.ctx_tma = 0;
  t.keep = a.keep;
  t.bf16 = dt == DT_BF16;
  t.err = attn_error_word();
  return t;
}

template <typename T>
void fwd_t(const AttnArgs& a, cudaStream_t s) {
  AttnTc t = make_args(std::is_same<T, bf16_t>::value ? DT_BF16 : DT_F16, a);
  const uint64_t rows = (uint64_t)a.B * a.nh * a.S;
  CUtensorMap mq, mk, mv;
  if (!map_tile(&mq, a.q, t.bf16, HD, rows, HD) || !map_tile(&mk, a.k, t.bf16, HD, rows, HD) ||
      !map_tile(&mv, a.v, t.bf16, HD, rows, HD))
    return;
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(attn_fwd_tc<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, kFwdSmem);
    cudaFuncSetAttribute(attn_fwd_tc_persist<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, kPFwdSmem);
    attr = true;
  }
  if (a.S <= TILE) {
    int nsm = 148;
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, 0);
    const int grid = std::min(a.B * a.nh, nsm);
    // ctx (B*S, H) in 32-row boxes of one head; rows of a box stay inside one sequence when S % 32 == 0
    CUtensorMap mc;
    t.ctx_tma = a.S % 32 == 0 && map_tile(&mc, a.ctx, t.bf16, t.H, (uint64_t)a.B * a.S, t.H, 32) ? 1 : 0;
    if (!t.ctx_tma) mc = mq;   // unused
    launch_pdl(attn_fwd_tc_persist<T>, grid, kPFwdThreads, kPFwdSmem, s, mq, mk, mv, mc, t);
  } else {
    dim3 grid((a.S + TILE - 1) / TILE, a.nh, a.B);
    launch_pdl(attn_fwd_tc<T>, grid, kFwdThreads, kFwdSmem, s, mq, mk, mv, t);
  }
  count_launch();
}

template <typename T>
void bwd_t(const AttnArgs& a, cudaStream_t s) {
  AttnTc t = make_args(std::is_same<T, bf16_t>::value ? DT_BF16 : DT_F16, a);
  const uint64_t rows = (uint64_t)a.B * a.nh * a.S;
  const uint64_t tokens = (uint64_t)a.B * a.S;
  CUtensorMap mq, mk, mv, mdo;
  if (!map_tile(&mq, a.q, t.bf16, HD, rows, HD) || !map_tile(&mk, a.k, t.bf16, HD, rows, HD) ||
      !map_tile(&mv, a.v, t.bf16, HD, rows, HD) || !map_tile(&mdo, a.dctx, t.bf16, t.H, tokens, t.H))
    return;
  const int ntile = (a.S + TILE - 1) / TILE;
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(attn_bwd_kv_tc<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, kBwdKvSmem);
    cudaFuncSetAttribute(attn_bwd_q_tc<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, kBwdQSmem);
    cudaFuncSetAttribute(attn_bwd_tc_persist<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, kPBwdSmem);
    attr = true;
  }
  if (ntile == 1) {
    int nsm = 148;
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, 0);
    // dQKV (B*S, 3H) in 32 x 32 boxes; a box's rows stay inside one sequence when S % 32 == 0
    CUtensorMap mdq;
    t.ctx_tma = a.S % 32 == 0 && map_tile(&mdq, a.dqkv, t.bf16, 3 * (uint64_t)t.H, tokens, 3 * (uint64_t)t.H, 32, true)
                    ? 1 : 0;
    if (!t.ctx_tma) mdq = mq;   // unused
    launch_pdl(attn_bwd_tc_persist<T>, std::min(a.B * a.nh, nsm), kPBwdThreads, kPBwdSmem, s, mq, mk, mv, mdo, mdq,
               t);
    count_launch();
    return;
  }
  dvec_launch(t.bf16 ? DT_BF16 : DT_F16, a, s);
  t.dvec = a.dvec;
  t.fuse_dq = 0;
  dim3 grid(ntile, a.nh, a.B);
  launch_pdl(attn_bwd_kv_tc<T>, grid, kBwdThreads, kBwdKvSmem, s, mq, mk, mv, mdo, t);
  count_launch();
  if (!t.fuse_dq) {
    launch_pdl(attn_bwd_q_tc<T>, grid, kBwdThreads, kBwdQSmem, s, mq, mk, mv, mdo, t);
    count_launch();
  }
}

}  // namespace

// Whether attn_tc_bwd_run writes the QKV bias-gradient partials (AttnArgs.colsum).
bool attn_tc_fuses_colsum(int dt, const AttnArgs& a) { return dt != DT_F32 && a.d == HD && a.S <= TILE; }

bool attn_tc_supports(int dt, const AttnArgs& a) {
  if (dt == DT_F32 || a.d != HD || a.S < 8) return false;
  // TMA row coordinates are 32-bit
  return (uint64_t)a.B * a.nh * a.S < (1ull << 31);
}

void attn_tc_fwd_run(int dt, const AttnArgs& a, cudaStream_t s) {
  if (dt == DT_F16) fwd_t<half_t>(a, s);
  else fwd_t<bf16_t>(a, s);
}

void attn_tc_bwd_run(int dt, const AttnArgs& a, cudaStream_t s) {
  if (dt == DT_F16) bwd_t<half_t>(a, s);
  else bwd_t<bf16_t>(a, s);
}

void attn_tc_set_wait_limit(uint64_t ns) {
  cudaMemcpy(attn_error_word() + 2, &ns, sizeof(ns), cudaMemcpyHostToDevice);
}

int attn_tc_take_error() {
  int v = 0;
  int* p = attn_error_word();
  cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost);
  if (v) cudaMemset(p, 0, sizeof(int));
  return v;
}

}  // namespace tlp
