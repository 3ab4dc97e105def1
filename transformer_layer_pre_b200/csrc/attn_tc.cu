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
// Backward regenerates P from LSE and reads the forward's dropout keep bits
// (one bit per element, written by the forward next to its output):
//   dV = Pd^T dO; dPd = dO V^T; dP = dPd * keep / (1 - p);
//   dS = P * (dP - D) with D = rowsum(dO * O); dQ = dS K c; dK = dS^T Q c.
//
// Tiles are 128 queries x 128 keys.  One elected thread issues every MMA
// (M = 128) into TMEM; softmax warps own one TMEM lane (one query row) each;
// helper warps draw the dropout bits of a row (forward) ahead of the softmax
// warps, or stage the stored ones (backward).  Every kernel is persistent
// (one CTA per SM walking work items).  P and dS go
// back to shared memory in the 128-byte-swizzled layout TMA uses for a
// [rows][64] tile, which serves as a K-major operand (rows x keys) and as an
// MN-major operand (keys x rows) alike; Q, K, V and dO tiles likewise serve
// both roles without any transpose.  TMA loads are per CTA (no multicast).
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <tuple>
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
  int colsum_acc;       // 1: added into row 0 of colsum with atomics (arrival order)
  int ctx_tma;          // persistent kernels: ctx (forward) or dQKV (backward) rows leave by TMA store (S % 32 == 0)
  const int* kv_ext;    // per sequence, one past its last unmasked key (long forward), or null
  int keep_ready;       // persistent forward: the keep bits are already in `keep` (read, not drawn)
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

// ============================================================================ backward
// Softmax-side threads of the backward kernels: warps 2-9, two threads per
// query row (TMEM lane), each 64 of the 128 key columns.
constexpr int kSoftThreads = 256;

// ============================================================================ forward, S > 128 (persistent)
// One CTA per SM walks items (sequence b, head h, 128-query tile), each over
// the key tiles up to the sequence's last unmasked key.  Warps: 0 TMA (Q of
// the item, K/V tiles into a three-slot ring, running ahead across items),
// 1 MMA, 2-5 softmax (thread = query row), 6-9 helpers (per key tile: the
// dropout keep bits of the 128 x 128 elements, also written out for the
// backward, and the key mask row, up to two tiles ahead).  The score
// accumulator S and the probability tile P are double-buffered by the
// running tile count g, so Q K^T of tile g+1 and the helpers' work overlap
// the softmax of tile g; O accumulates in TMEM over the item's key tiles.
// Online softmax with a lazy reference: P = 2^(x - m_ref) where m_ref is the
// running row maximum at the last rescale; O and the row sum are rescaled
// (in TMEM) only when the maximum has grown by more than 2^8 since then, so
// P stays below 256 (exact in fp16/bf16 range) and most tiles skip the
// rescale.  The result is the same softmax: every term carries the same
// reference until the final normalisation.
constexpr int kLThreads = 448;
constexpr int kLKv = 3;                                     // K/V ring slots
constexpr int kLAux = 128 * 16 + 128 * 4;                   // per slot: keep bits [128][16], mask [128]
constexpr int kLSmem = 2 * TB + kLKv * 2 * TB + 4 * TB + 2 * kLAux + 1024 + 256 + 4096;   // + row exchange
constexpr float kLRescale = 8.0f;                           // log2 units: P < 2^8

// One past the last unmasked key of each sequence (kv_ext[b]), or S when the
// mask leaves the last key valid; one block per sequence.
__global__ void key_extent_kernel(const float* __restrict__ mask, int S, int* __restrict__ kv_ext) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ int ext;
  if (threadIdx.x == 0) ext = 0;
  __syncthreads();
  const int b = blockIdx.x;
  int e = 0;
  for (int j = threadIdx.x; j < S; j += blockDim.x)
    if (mask[(size_t)b * S + j] != -INFINITY) e = j + 1;
  if (e) atomicMax(&ext, e);
  __syncthreads();
  if (threadIdx.x == 0) kv_ext[b] = ext;
}

// Writes 32 x 32-bit registers to 32 consecutive TMEM columns of this warp's lanes.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15])),
      "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])), "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])),
      "r"(__float_as_uint(v[20])), "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])), "r"(__float_as_uint(v[27])),
      "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])), "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Key tiles item `it` runs over (at least one).
__device__ __forceinline__ int long_item_tiles(const AttnTc& a, int b, int ntiles_all) {
  if (!a.kv_ext) return ntiles_all;
  return max(1, min(ntiles_all, (a.kv_ext[b] + TILE - 1) / TILE));
}

template <typename T>
__global__ void __launch_bounds__(kLThreads, 1)
    attn_fwd_tc_long(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                     const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tctx, AttnTc a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  uint8_t* sQ = sm;                                   // [2] Q tiles
  uint8_t* sKV = sm + 2 * TB;                         // [kLKv] x (K, V)
  uint8_t* sP = sKV + kLKv * 2 * TB;                  // [2] P pairs (also output staging)
  uint8_t* saux = sP + 4 * TB;                        // [2] x (bits [128][16], mask [128])
  uint64_t* bar = reinterpret_cast<uint64_t*>(saux + 2 * kLAux);
  uint64_t *q_full = bar, *q_empty = bar + 2, *kv_full = bar + 4, *kv_empty = kv_full + kLKv;
  uint64_t *s_full = kv_empty + kLKv, *s_free = s_full + 2, *p_full = s_free + 2, *pv_done = p_full + 2;
  uint64_t *aux_full = pv_done + 2, *aux_free = aux_full + 2;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(aux_free + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = a.S;
  const int nq = (S + TILE - 1) / TILE;
  const int nitems = a.B * a.nh * nq;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], kSoftThreads);
      mbar_init(&p_full[i], kSoftThreads);
      mbar_init(&pv_done[i], 1);
      mbar_init(&aux_full[i], 128);
      mbar_init(&aux_free[i], kSoftThreads);
    }
    for (int i = 0; i < kLKv; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tslot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;   // S[0] at 0, S[1] at 128, O at 256
  pdl_wait();
  pdl_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      uint32_t g = 0;
      int n = 0;
      bool ok = true;
      for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x, ++n) {
        const int bh = it / nq, q0 = (it - bh * nq) * TILE;
        const int nt = long_item_tiles(a, bh / a.nh, nq);
        const int row0 = bh * S;
        const int qs = n & 1;
        if (!(ok = mbar_wait(&q_empty[qs], ((n >> 1) & 1) ^ 1, a.err, 81))) break;
        mbar_arrive_expect_tx(&q_full[qs], TB);
        tma_load_2d(sQ + qs * TB, &tq, &q_full[qs], 0, row0 + q0);
        for (int j = 0; j < nt; ++j, ++g) {
          const int ks = g % kLKv;
          if (!(ok = mbar_wait(&kv_empty[ks], ((g / kLKv) & 1) ^ 1, a.err, 82))) break;
          mbar_arrive_expect_tx(&kv_full[ks], 2 * TB);
          tma_load_2d(sKV + ks * 2 * TB, &tk, &kv_full[ks], 0, row0 + j * TILE);
          tma_load_2d(sKV + ks * 2 * TB + TB, &tv, &kv_full[ks], 0, row0 + j * TILE);
        }
      }
      // a wait that gave up: the loads already issued land before the CTA exits
      if (!ok) {
        for (int i = 0; i < 2; ++i) mbar_wait(&q_full[i], 0, nullptr, 0);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id_s = idesc_f16(128, 128, a.bf16 != 0, false, false);
      const uint32_t id_o = idesc_f16(128, 64, a.bf16 != 0, false, true);
      uint32_t g = 0;
      int n = 0;
      bool ok = true;
      // O += P(gp) V(gp); the first product of an item overwrites O
      auto pv = [&](uint32_t gp, bool acc) -> bool {
        const int ps = gp & 1, ks = gp % kLKv;
        if (!mbar_wait(&p_full[ps], (gp >> 1) & 1, a.err, 83)) return false;
        tc_fence_after();
        const uint32_t aP = smem_u32(sP + ps * 2 * TB), aV = smem_u32(sKV + ks * 2 * TB + TB);
#pragma unroll
        for (int kk = 0; kk < TILE / 16; ++kk)
          mma_f16(tmem + 256, dk_pair(aP, kk), dmn_tile(aV, kk), id_o, (acc || kk > 0) ? 1u : 0u);
        mma_commit(&pv_done[ps]);
        mma_commit(&kv_empty[ks]);
        return true;
      };
      for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x, ++n) {
        const int bh = it / nq;
        const int nt = long_item_tiles(a, bh / a.nh, nq);
        const int qs = n & 1;
        if (!(ok = mbar_wait(&q_full[qs], (n >> 1) & 1, a.err, 84))) break;
        const uint32_t aQ = smem_u32(sQ + qs * TB);
        for (int j = 0; j < nt; ++j, ++g) {
          const int ks = g % kLKv, ss = g & 1;
          if (!(ok = mbar_wait(&kv_full[ks], (g / kLKv) & 1, a.err, 85))) break;
          if (!(ok = mbar_wait(&s_free[ss], ((g >> 1) & 1) ^ 1, a.err, 86))) break;
          tc_fence_after();
          const uint32_t aK = smem_u32(sKV + ks * 2 * TB);
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk)
            mma_f16(tmem + 128 * ss, dk_tile(aQ, kk), dk_tile(aK, kk), id_s, kk > 0);
          mma_commit(&s_full[ss]);
          if (j == nt - 1) mma_commit(&q_empty[qs]);
          if (j > 0 && !(ok = pv(g - 1, j > 1))) break;
        }
        if (ok) ok = pv(g - 1, nt > 1);
      }
    }
  } else if (warp >= 10) {
    // helpers: keep bits and mask row of each key tile, two tiles ahead at most
    const int r = threadIdx.x - 320;
    uint32_t g = 0;
    for (int it = blockIdx.x; it < nitems; it += gridDim.x) {
      const int bh = it / nq, q0 = (it - bh * nq) * TILE;
      const int b = bh / a.nh;
      const int nt = long_item_tiles(a, b, nq);
      const bool row_ok = q0 + r < S;
      bool ok = true;
      for (int j = 0; j < nt; ++j, ++g) {
        const int as = g & 1;
        const int k0 = j * TILE;
        // the tile's bits and mask value before the wait for the slot
        const uint64_t e8 = (((uint64_t)bh * S + (uint64_t)(q0 + r)) * (uint64_t)S + (uint64_t)k0) >> 3;
        uint32_t w[4] = {0u, 0u, 0u, 0u};
        if (a.drop.thr) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t v = 0;
#pragma unroll
            for (int gg = 0; gg < 4; ++gg) v |= dropout_bits8(a.drop, 0, e8 + (uint64_t)(q * 4 + gg)) << (8 * gg);
            w[q] = v;
          }
        }
        const int key = k0 + r;
        const float mv = key < S ? (a.mask ? __ldg(a.mask + (size_t)b * S + key) * kLog2e : 0.0f) : -INFINITY;
        if (!(ok = mbar_wait(&aux_free[as], ((g >> 1) & 1) ^ 1, a.err, 87))) break;
        uint8_t* ax = saux + as * kLAux;
        if (a.drop.thr) {
          *reinterpret_cast<uint4*>(ax + r * 16) = make_uint4(w[0], w[1], w[2], w[3]);
          if (a.keep && row_ok) {
            // 16 bytes when they are 16-byte aligned (S % 128 == 0), else words or bytes
            if ((e8 & 15) == 0) {
              *reinterpret_cast<uint4*>(a.keep + e8) = make_uint4(w[0], w[1], w[2], w[3]);
            } else if ((e8 & 3) == 0) {
#pragma unroll
              for (int q = 0; q < 4; ++q) reinterpret_cast<uint32_t*>(a.keep + e8)[q] = w[q];
            } else {
#pragma unroll
              for (int q = 0; q < 16; ++q) a.keep[e8 + q] = (uint8_t)(w[q >> 2] >> (8 * (q & 3)));
            }
          }
        }
        reinterpret_cast<float*>(ax + 2048)[r] = mv;
        mbar_arrive(&aux_full[as]);
      }
      if (!ok) break;
    }
  } else {
    // softmax: warp w owns TMEM lanes 32*(w%4) (query rows) and key columns
    // 64*hf .. +63 of each tile, hf = (w-2)/4: two threads per query row,
    // warps w and w+4 meet at a named barrier to combine their row maxima
    const int quarter = warp & 3;
    const int hf = (warp - 2) >> 2;
    const int r = quarter * 32 + lane;
    const int bar_id = 1 + quarter;
    const uint32_t lo = (uint32_t)(quarter * 32) << 16;
    const float c2 = a.scale * kLog2e;
    const float dsc = a.drop.thr ? a.drop.scale : 1.0f;
    float* xch = reinterpret_cast<float*>(tslot + 4);   // [2 tiles][2 halves][128] row maxima, then row sums
    uint32_t g = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
      const int bh = it / nq, q0 = (it - bh * nq) * TILE;
      const int b = bh / a.nh, h = bh - b * a.nh;
      const int nt = long_item_tiles(a, b, nq);
      const int i = q0 + r;
      float mref = -INFINITY, l = 0.0f;
      for (int j = 0; j < nt; ++j, ++g) {
        const int ss = g & 1;
        const uint8_t* ax = saux + ss * kLAux;
        const float* mrow = reinterpret_cast<const float*>(ax + 2048) + hf * 64;
        if (!(ok = mbar_wait_warp(&aux_full[ss], (g >> 1) & 1, a.err, 88))) break;
        const uint2 kb8 = a.drop.thr ? *reinterpret_cast<const uint2*>(ax + r * 16 + hf * 8) : make_uint2(~0u, ~0u);
        if (!(ok = mbar_wait_warp(&s_full[ss], (g >> 1) & 1, a.err, 89))) break;
        tc_fence_after();
        const uint32_t ts = tmem + 128 * ss + lo + hf * 64;
        float sv[64];
        // pass 1: this half's row maximum (scaled scores + mask, log2 units),
        // combined with the other half's
        tmem_ld64(ts, sv);
        float mx = -INFINITY;
#pragma unroll
        for (int t = 0; t < 64; t += 4) {
          const float4 m4 = *reinterpret_cast<const float4*>(mrow + t);
          const float2 x0 = fma2(make_float2(sv[t], sv[t + 1]), make_float2(c2, c2), make_float2(m4.x, m4.y));
          const float2 x1 = fma2(make_float2(sv[t + 2], sv[t + 3]), make_float2(c2, c2), make_float2(m4.z, m4.w));
          mx = max3f(mx, max3f(x0.x, x0.y, x1.x), x1.y);
        }
        xch[(ss * 2 + hf) * 128 + r] = mx;
        named_barrier(bar_id, 64);
        mx = fmaxf(xch[(ss * 2) * 128 + r], xch[(ss * 2 + 1) * 128 + r]);
        const float mnew = fmaxf(mref, mx);
        if (j == 0) {
          mref = mnew;   // the item's first product overwrites O
        } else {
          const bool need = mnew > mref + kLRescale;
          if (__any_sync(0xffffffffu, need)) {
            // O (and the row sum) to the new reference, once the previous product is in
            if (!(ok = mbar_wait_warp(&pv_done[(g - 1) & 1], ((g - 1) >> 1) & 1, a.err, 90))) break;
            tc_fence_after();
            const float alpha = need ? ex2_approx(mref - mnew) : 1.0f;
            float o[32];
            tmem_ld32(tmem + 256 + lo + hf * 32, o);
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] *= alpha;
            tmem_st32(tmem + 256 + lo + hf * 32, o);
            tmem_st_wait();
            if (need) {
              l *= alpha;
              mref = mnew;
            }
          }
        }
        const float msub = mref == -INFINITY ? 0.0f : mref;   // 2^(-inf - msub) = 0
        // the P slot is free once the product of tile g-2 is done
        if (g >= 2 && !(ok = mbar_wait_warp(&pv_done[ss], ((g - 2) >> 1) & 1, a.err, 91))) break;
        // pass 2: P = 2^(x - m_ref), dropped, into this half of the P tile;
        // row sum of the undropped P (the S values are still in registers)
        float2 ls2 = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int gg = 0; gg < 8; ++gg) {
          const uint32_t bits = ((gg < 4 ? kb8.x : kb8.y) >> (8 * (gg & 3))) & 0xFFu;
          float pv[8];
#pragma unroll
          for (int t = 0; t < 8; t += 2) {
            const float2 m2 = *reinterpret_cast<const float2*>(mrow + gg * 8 + t);
            const float2 x = add2(fma2(make_float2(sv[gg * 8 + t], sv[gg * 8 + t + 1]), make_float2(c2, c2), m2),
                                  make_float2(-msub, -msub));
            const float2 p = make_float2(ex2_approx(x.x), ex2_approx(x.y));
            ls2 = add2(ls2, p);
            pv[t] = ((bits >> t) & 1u) ? p.x : 0.0f;
            pv[t + 1] = ((bits >> (t + 1)) & 1u) ? p.y : 0.0f;
          }
          pair_store8<T>(sP + ss * 2 * TB, r, hf * 8 + gg, pv);
        }
        l += ls2.x + ls2.y;
        mbar_arrive(&aux_free[ss]);
        tc_fence_before();
        mbar_arrive(&s_free[ss]);
        fence_proxy_async_smem();
        mbar_arrive(&p_full[ss]);
      }
      if (!ok) break;
      // the item's output once its last product is in: this thread's 32
      // columns of the row; the row sum is the two halves' sums
      const uint32_t gl = g - 1;
      if (!(ok = mbar_wait_warp(&pv_done[gl & 1], (gl >> 1) & 1, a.err, 92))) break;
      tc_fence_after();
      float o[32];
      tmem_ld32(tmem + 256 + lo + hf * 32, o);
      xch[(512 + hf * 128) + r] = l;
      named_barrier(bar_id, 64);
      const float lt = xch[512 + r] + xch[640 + r];
      named_barrier(bar_id, 64);   // both have read the sums before the next item's tile maxima land
      const float inv = lt > 0.0f ? dsc / lt : 0.0f;
      if (i < S) {
        if (hf == 0) a.lse[(size_t)bh * S + i] = lt > 0.0f ? (mref + log2f(lt)) * kLn2 : INFINITY;
        T* dst = static_cast<T*>(a.ctx) + ((size_t)b * S + i) * a.H + h * HD + hf * 32;
#pragma unroll
        for (int c = 0; c < 32; c += 8) {
          float w8[8];
#pragma unroll
          for (int t = 0; t < 8; ++t) w8[t] = o[c + t] * inv;
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

// ============================================================================ backward, S > 128 (persistent)
// Two persistent kernels.  attn_bwd_kv_long walks items (key tile, b, h): K
// and V stay in shared memory while every query tile of the sequence passes
// (Q, dO through a two-slot ring); per query tile S = Q K^T and dPd = dO V^T
// go to TMEM, the softmax warps turn them into Pd and dS in shared memory,
// and dV += Pd^T dO, dK += dS^T Q accumulate in TMEM.  attn_bwd_q_long walks
// items (query tile, b, h) over the key tiles up to the sequence's last
// unmasked key and accumulates dQ += dS K.  In both, the products of the next
// tile are issued as soon as the softmax has read the current S and dPd, so
// they run while the softmax finishes; keep bits come from the forward (no
// Philox), the log-sum-exp, D = rowsum(dO O) and the key mask are staged by
// helper warps one tile ahead.  Key tiles holding only masked keys get dK =
// dV = 0 without any product (their probabilities are all exactly 0).
constexpr int kBLThreads = 448;                              // 0 TMA, 1 MMA, 2-9 softmax, 10-13 helpers
constexpr int kBLAux = 128 * 16 + 3 * 128 * 4;               // bits [128][16], mask, lse2, D [128]
constexpr int kBLKvSmem = 4 * TB + 4 * TB + 4 * TB + 2 * kBLAux + 1024 + 256;   // K/V x2, Q/dO x2, Pd+dS pairs
constexpr int kBLQSmem = 4 * TB + 4 * TB + 2 * TB + 2 * kBLAux + 1024 + 256;    // Q/dO x2, K/V x2, dS pair

// Helper-warp staging of one (query tile q0, key tile k0) pair of item bh:
// lse2, D and the 16 keep-bit bytes of query row q0 + r, and the mask of key
// k0 + r.  bl_load_aux issues every global load (before the wait for the
// shared-memory slot, so the latencies overlap one another and the wait),
// bl_store_aux writes the slot.
struct BlAux {
  uint4 kb;
  float mv, lv, dv;
};
__device__ __forceinline__ BlAux bl_load_aux(const AttnTc& a, int bh, int b, int q0, int k0, int r) {
  const int S = a.S;
  const int q = q0 + r;
  const bool qv = q < S;
  BlAux x;
  x.kb = make_uint4(~0u, ~0u, ~0u, ~0u);
  if (a.drop.thr) {
    if (!qv) {
      x.kb = make_uint4(0u, 0u, 0u, 0u);
    } else {
      const uint64_t e8 = (((uint64_t)bh * S + (uint64_t)q) * (uint64_t)S + (uint64_t)k0) >> 3;
      if (a.keep) {
        if ((e8 & 15) == 0) {
          x.kb = __ldg(reinterpret_cast<const uint4*>(a.keep + e8));
        } else {
          uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
          for (int t = 0; t < 16; ++t) w[t >> 2] |= (uint32_t)__ldg(a.keep + e8 + t) << (8 * (t & 3));
          x.kb = make_uint4(w[0], w[1], w[2], w[3]);
        }
      } else {
        uint32_t w[4];
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          uint32_t v = 0;
#pragma unroll
          for (int gg = 0; gg < 4; ++gg) v |= dropout_bits8(a.drop, 0, e8 + (uint64_t)(qq * 4 + gg)) << (8 * gg);
          w[qq] = v;
        }
        x.kb = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  }
  const int key = k0 + r;
  x.mv = key < S ? (a.mask ? __ldg(a.mask + (size_t)b * S + key) * kLog2e : 0.0f) : -INFINITY;
  x.lv = qv ? __ldg(a.lse + (size_t)bh * S + q) * kLog2e : INFINITY;
  x.dv = qv ? __ldg(a.dvec + (size_t)bh * S + q) : 0.0f;
  return x;
}
__device__ __forceinline__ void bl_store_aux(uint8_t* ax, int r, const BlAux& x) {
  float* smask = reinterpret_cast<float*>(ax + 2048);
  *reinterpret_cast<uint4*>(ax + r * 16) = x.kb;
  smask[r] = x.mv;
  smask[128 + r] = x.lv;
  smask[256 + r] = x.dv;
}

// Softmax-side work of one (query tile, key tile) pair for one thread: query
// row r, key columns [kc0, kc0 + 64).  Reads S and dPd from TMEM (then
// releases them on s_free), waits until the previous pair's products have
// read the shared tiles (ds_free), writes Pd (when sPd) and dS.
template <typename T>
__device__ __forceinline__ bool bl_softmax_pair(const AttnTc& a, const uint8_t* ax, int r, int kc0, uint32_t tS,
                                                uint32_t tdP, uint32_t lo, uint64_t* s_free, uint64_t* ds_free,
                                                uint32_t ds_parity, uint8_t* sPd, uint8_t* sdS) {
  const float c2 = a.scale * kLog2e;
  const float dsc = a.drop.thr ? a.drop.scale : 1.0f;
  const float* smask = reinterpret_cast<const float*>(ax + 2048);
  const float lse2 = smask[128 + r], Di = smask[256 + r];
  const uint2 kb8 = *reinterpret_cast<const uint2*>(ax + r * 16 + (kc0 >> 3));
  // first 32 columns: computed while the previous pair's products may still
  // read the shared tiles, held packed; the shared tiles are written once
  // those products are done (ds_free); the second 32 columns go straight there
  uint4 pdp[4], dsp[4];
  auto compute = [&](int c, const float (&sv)[32], const float (&dv)[32], int g, float (&pd)[8], float (&ds)[8]) {
    const uint32_t bits = ((c == 0 ? kb8.x : kb8.y) >> (8 * g)) & 0xFFu;
    const int kt = kc0 + c * 32 + g * 8;
    const float4 m0 = *reinterpret_cast<const float4*>(smask + kt);
    const float4 m1 = *reinterpret_cast<const float4*>(smask + kt + 4);
    const float ml[8] = {m0.x - lse2, m0.y - lse2, m0.z - lse2, m0.w - lse2,
                         m1.x - lse2, m1.y - lse2, m1.z - lse2, m1.w - lse2};
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      // lse2 = +inf for query rows past the sequence end: p = 0
      const float p = ex2_approx(fmaf(sv[g * 8 + t], c2, ml[t]));
      const bool keep = (bits >> t) & 1u;
      pd[t] = keep ? p * dsc : 0.0f;
      const float dp = keep ? dv[g * 8 + t] * dsc : 0.0f;
      ds[t] = p * (dp - Di);
    }
  };
  auto put = [&](int k8, const uint4& pdv, const uint4& dsv) {
    const int region = k8 >> 3, cc = k8 & 7;
    if (sPd) *reinterpret_cast<uint4*>(sPd + region * 16384 + r * 128 + ((cc ^ (r & 7)) << 4)) = pdv;
    *reinterpret_cast<uint4*>(sdS + region * 16384 + r * 128 + ((cc ^ (r & 7)) << 4)) = dsv;
  };
  {
    float sv[32], dv[32];
    tmem_ld32x2(tS + lo + kc0, sv, tdP + lo + kc0, dv);
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      float pd[8], ds[8];
      compute(0, sv, dv, g, pd, ds);
      pdp[g] = pack8<T>(pd);
      dsp[g] = pack8<T>(ds);
    }
  }
  if (!mbar_wait_warp(ds_free, ds_parity, a.err, 95)) return false;
#pragma unroll
  for (int g = 0; g < 4; ++g) put((kc0 >> 3) + g, pdp[g], dsp[g]);
  {
    float sv[32], dv[32];
    tmem_ld32x2(tS + lo + kc0 + 32, sv, tdP + lo + kc0 + 32, dv);
    // every TMEM read of this pair is done: S and dPd may be overwritten
    tc_fence_before();
    mbar_arrive(s_free);
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      float pd[8], ds[8];
      compute(1, sv, dv, g, pd, ds);
      put((kc0 >> 3) + 4 + g, pack8<T>(pd), pack8<T>(ds));
    }
  }
  return true;
}

__device__ __forceinline__ int bl_key_tiles(const AttnTc& a, int b, int nk) {
  if (!a.kv_ext) return nk;
  return max(1, min(nk, (a.kv_ext[b] + TILE - 1) / TILE));
}

template <typename T>
__global__ void __launch_bounds__(kBLThreads, 1)
    attn_bwd_kv_long(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                     const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo, AttnTc a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  uint8_t* sKV = sm;                      // [2] x (K, V)
  uint8_t* sQD = sm + 4 * TB;             // [2] x (Q, dO)
  uint8_t* sPd = sm + 8 * TB;             // pair
  uint8_t* sdS = sm + 10 * TB;            // pair
  uint8_t* saux = sm + 12 * TB;           // [2]
  uint64_t* bar = reinterpret_cast<uint64_t*>(saux + 2 * kBLAux);
  uint64_t *kv_full = bar, *kv_empty = bar + 2, *qd_full = bar + 4, *qd_empty = bar + 6, *aux_full = bar + 8,
           *aux_free = bar + 10, *s_full = bar + 12, *s_free = bar + 13, *ds_full = bar + 14, *ds_free = bar + 15,
           *acc_full = bar + 16, *acc_free = bar + 17;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar + 18);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = a.S;
  const int nk = (S + TILE - 1) / TILE, nq = nk;
  const int nitems = a.B * a.nh * nk;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
      mbar_init(&qd_full[i], 1);
      mbar_init(&qd_empty[i], 1);
      mbar_init(&aux_full[i], 128);
      mbar_init(&aux_free[i], kSoftThreads);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, kSoftThreads);
    mbar_init(ds_full, kSoftThreads);
    mbar_init(ds_free, 1);
    mbar_init(acc_full, 1);
    mbar_init(acc_free, kSoftThreads);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tslot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  pdl_wait();
  pdl_launch_dependents();
  const uint32_t tS = tmem, tdP = tmem + 128, tdV = tmem + 256, tdK = tmem + 320;
  // an item (key tile j of sequence b, head h) whose keys are all masked
  auto masked = [&](int b, int j) { return j >= bl_key_tiles(a, b, nk) || (a.kv_ext && j * TILE >= a.kv_ext[b]); };

  if (warp == 0) {
    if (lane == 0) {
      int n = 0;
      uint32_t g = 0;
      bool ok = true;
      for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
        const int bh = it / nk, j = it - bh * nk, b = bh / a.nh, h = bh - b * a.nh;
        if (masked(b, j)) continue;
        const int ks = n & 1;
        if (!(ok = mbar_wait(&kv_empty[ks], ((n >> 1) & 1) ^ 1, a.err, 101))) break;
        mbar_arrive_expect_tx(&kv_full[ks], 2 * TB);
        tma_load_2d(sKV + ks * 2 * TB, &tk, &kv_full[ks], 0, bh * S + j * TILE);
        tma_load_2d(sKV + ks * 2 * TB + TB, &tv, &kv_full[ks], 0, bh * S + j * TILE);
        for (int i = 0; i < nq; ++i, ++g) {
          const int qs = g & 1;
          if (!(ok = mbar_wait(&qd_empty[qs], ((g >> 1) & 1) ^ 1, a.err, 102))) break;
          mbar_arrive_expect_tx(&qd_full[qs], 2 * TB);
          tma_load_2d(sQD + qs * 2 * TB, &tq, &qd_full[qs], 0, bh * S + i * TILE);
          tma_load_2d(sQD + qs * 2 * TB + TB, &tdo, &qd_full[qs], h * HD, b * S + i * TILE);
        }
        ++n;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const bool bf = a.bf16 != 0;
      const uint32_t id_kk = idesc_f16(128, 128, bf, false, false);
      const uint32_t id_mm = idesc_f16(128, 64, bf, true, true);
      const uint32_t aPd = smem_u32(sPd), adS = smem_u32(sdS);
      int n = 0;
      uint32_t g = 0;
      bool ok = true;
      // dV += Pd^T dO, dK += dS^T Q of pair gp; the first pair of an item overwrites
      auto dvdk = [&](uint32_t gp, bool acc, int nn) -> bool {
        if (!acc && !mbar_wait(acc_free, (nn & 1) ^ 1, a.err, 103)) return false;
        if (!mbar_wait(ds_full, gp & 1, a.err, 104)) return false;
        tc_fence_after();
        const uint32_t aQ = smem_u32(sQD + (gp & 1) * 2 * TB), adO = aQ + TB;
#pragma unroll
        for (int kk = 0; kk < TILE / 16; ++kk)
          mma_f16(tdV, dmn_pair(aPd, kk), dmn_tile(adO, kk), id_mm, (acc || kk > 0) ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < TILE / 16; ++kk)
          mma_f16(tdK, dmn_pair(adS, kk), dmn_tile(aQ, kk), id_mm, (acc || kk > 0) ? 1u : 0u);
        mma_commit(ds_free);
        mma_commit(&qd_empty[gp & 1]);
        return true;
      };
      for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
        const int bh = it / nk, j = it - bh * nk, b = bh / a.nh;
        if (masked(b, j)) continue;
        const int ks = n & 1;
        if (!(ok = mbar_wait(&kv_full[ks], (n >> 1) & 1, a.err, 105))) break;
        const uint32_t aK = smem_u32(sKV + ks * 2 * TB), aV = aK + TB;
        for (int i = 0; i < nq; ++i, ++g) {
          const int qs = g & 1;
          if (!(ok = mbar_wait(&qd_full[qs], (g >> 1) & 1, a.err, 106))) break;
          if (!(ok = mbar_wait(s_free, (g & 1) ^ 1, a.err, 107))) break;
          tc_fence_after();
          const uint32_t aQ = smem_u32(sQD + qs * 2 * TB), adO = aQ + TB;
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) mma_f16(tS, dk_tile(aQ, kk), dk_tile(aK, kk), id_kk, kk > 0);
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) mma_f16(tdP, dk_tile(adO, kk), dk_tile(aV, kk), id_kk, kk > 0);
          mma_commit(s_full);
          if (i > 0 && !(ok = dvdk(g - 1, i > 1, n))) break;
        }
        if (ok) ok = dvdk(g - 1, nq > 1, n);
        if (!ok) break;
        mma_commit(acc_full);
        mma_commit(&kv_empty[ks]);
        ++n;
      }
    }
  } else if (warp >= 10) {
    const int r = threadIdx.x - 320;
    uint32_t g = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
      const int bh = it / nk, j = it - bh * nk, b = bh / a.nh;
      if (masked(b, j)) continue;
      for (int i = 0; i < nq; ++i, ++g) {
        const int as = g & 1;
        const BlAux x = bl_load_aux(a, bh, b, i * TILE, j * TILE, r);
        if (!(ok = mbar_wait(&aux_free[as], ((g >> 1) & 1) ^ 1, a.err, 108))) break;
        bl_store_aux(saux + as * kBLAux, r, x);
        mbar_arrive(&aux_full[as]);
      }
    }
  } else {
    const int quarter = warp & 3;
    const int hf = (warp - 2) >> 2;
    const int r = quarter * 32 + lane;
    const uint32_t lo = (uint32_t)(quarter * 32) << 16;
    int n = 0;
    uint32_t g = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
      const int bh = it / nk, j = it - bh * nk, b = bh / a.nh, h = bh - b * a.nh;
      const int key = j * TILE + r;   // TMEM lane r of dV, dK = key row
      if (masked(b, j)) {
        // no query attends to these keys: dK = dV = 0
        if (key < S) {
          T* dst = static_cast<T*>(a.dqkv) + ((size_t)b * S + key) * 3 * a.H + h * HD + hf * 32;
          const float z[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
          for (int c = 0; c < 32; c += 8) {
            store8<T>(dst + a.H + c, z);
            store8<T>(dst + 2 * a.H + c, z);
          }
        }
        continue;
      }
      for (int i = 0; i < nq; ++i, ++g) {
        const int as = g & 1;
        if (!(ok = mbar_wait_warp(&aux_full[as], (g >> 1) & 1, a.err, 109))) break;
        if (!(ok = mbar_wait_warp(s_full, g & 1, a.err, 110))) break;
        tc_fence_after();
        if (!(ok = bl_softmax_pair<T>(a, saux + as * kBLAux, r, hf * 64, tS, tdP, lo, s_free, ds_free, (g & 1) ^ 1,
                                      sPd, sdS)))
          break;
        mbar_arrive(&aux_free[as]);
        fence_proxy_async_smem();
        mbar_arrive(ds_full);
      }
      if (!ok) break;
      if (!(ok = mbar_wait_warp(acc_full, n & 1, a.err, 111))) break;
      tc_fence_after();
      float dv[32], dk[32];
      tmem_ld32x2(tdV + lo + hf * 32, dv, tdK + lo + hf * 32, dk);
      tc_fence_before();
      mbar_arrive(acc_free);
      if (key < S) {
        T* dst = static_cast<T*>(a.dqkv) + ((size_t)b * S + key) * 3 * a.H + h * HD + hf * 32;
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
      ++n;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

template <typename T>
__global__ void __launch_bounds__(kBLThreads, 1)
    attn_bwd_q_long(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                    const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo, AttnTc a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  uint8_t* sQD = sm;                      // [2] x (Q, dO)
  uint8_t* sKV = sm + 4 * TB;             // [2] x (K, V)
  uint8_t* sdS = sm + 8 * TB;             // pair
  uint8_t* saux = sm + 10 * TB;           // [2]
  uint64_t* bar = reinterpret_cast<uint64_t*>(saux + 2 * kBLAux);
  uint64_t *qd_full = bar, *qd_empty = bar + 2, *kv_full = bar + 4, *kv_empty = bar + 6, *aux_full = bar + 8,
           *aux_free = bar + 10, *s_full = bar + 12, *s_free = bar + 13, *ds_full = bar + 14, *ds_free = bar + 15,
           *acc_full = bar + 16, *acc_free = bar + 17;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar + 18);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = a.S;
  const int nq = (S + TILE - 1) / TILE, nk_all = nq;
  const int nitems = a.B * a.nh * nq;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&qd_full[i], 1);
      mbar_init(&qd_empty[i], 1);
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
      mbar_init(&aux_full[i], 128);
      mbar_init(&aux_free[i], kSoftThreads);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, kSoftThreads);
    mbar_init(ds_full, kSoftThreads);
    mbar_init(ds_free, 1);
    mbar_init(acc_full, 1);
    mbar_init(acc_free, kSoftThreads);
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

  if (warp == 0) {
    if (lane == 0) {
      int n = 0;
      uint32_t g = 0;
      bool ok = true;
      for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x, ++n) {
        const int bh = it / nq, i = it - bh * nq, b = bh / a.nh, h = bh - b * a.nh;
        const int nk = bl_key_tiles(a, b, nk_all);
        const int qs = n & 1;
        if (!(ok = mbar_wait(&qd_empty[qs], ((n >> 1) & 1) ^ 1, a.err, 121))) break;
        mbar_arrive_expect_tx(&qd_full[qs], 2 * TB);
        tma_load_2d(sQD + qs * 2 * TB, &tq, &qd_full[qs], 0, bh * S + i * TILE);
        tma_load_2d(sQD + qs * 2 * TB + TB, &tdo, &qd_full[qs], h * HD, b * S + i * TILE);
        for (int j = 0; j < nk; ++j, ++g) {
          const int ks = g & 1;
          if (!(ok = mbar_wait(&kv_empty[ks], ((g >> 1) & 1) ^ 1, a.err, 122))) break;
          mbar_arrive_expect_tx(&kv_full[ks], 2 * TB);
          tma_load_2d(sKV + ks * 2 * TB, &tk, &kv_full[ks], 0, bh * S + j * TILE);
          tma_load_2d(sKV + ks * 2 * TB + TB, &tv, &kv_full[ks], 0, bh * S + j * TILE);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const bool bf = a.bf16 != 0;
      const uint32_t id_kk = idesc_f16(128, 128, bf, false, false);
      const uint32_t id_km = idesc_f16(128, 64, bf, false, true);
      const uint32_t adS = smem_u32(sdS);
      int n = 0;
      uint32_t g = 0;
      bool ok = true;
      // dQ += dS K of pair gp; the first pair of an item overwrites
      auto dq = [&](uint32_t gp, bool acc, int nn) -> bool {
        if (!acc && !mbar_wait(acc_free, (nn & 1) ^ 1, a.err, 123)) return false;
        if (!mbar_wait(ds_full, gp & 1, a.err, 124)) return false;
        tc_fence_after();
        const uint32_t aK = smem_u32(sKV + (gp & 1) * 2 * TB);
#pragma unroll
        for (int kk = 0; kk < TILE / 16; ++kk)
          mma_f16(tdQ, dk_pair(adS, kk), dmn_tile(aK, kk), id_km, (acc || kk > 0) ? 1u : 0u);
        mma_commit(ds_free);
        mma_commit(&kv_empty[gp & 1]);
        return true;
      };
      for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x, ++n) {
        const int bh = it / nq, b = bh / a.nh;
        const int nk = bl_key_tiles(a, b, nk_all);
        const int qs = n & 1;
        if (!(ok = mbar_wait(&qd_full[qs], (n >> 1) & 1, a.err, 125))) break;
        const uint32_t aQ = smem_u32(sQD + qs * 2 * TB), adO = aQ + TB;
        for (int j = 0; j < nk; ++j, ++g) {
          const int ks = g & 1;
          if (!(ok = mbar_wait(&kv_full[ks], (g >> 1) & 1, a.err, 126))) break;
          if (!(ok = mbar_wait(s_free, (g & 1) ^ 1, a.err, 127))) break;
          tc_fence_after();
          const uint32_t aK = smem_u32(sKV + ks * 2 * TB), aV = aK + TB;
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) mma_f16(tS, dk_tile(aQ, kk), dk_tile(aK, kk), id_kk, kk > 0);
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) mma_f16(tdP, dk_tile(adO, kk), dk_tile(aV, kk), id_kk, kk > 0);
          mma_commit(s_full);
          if (j > 0 && !(ok = dq(g - 1, j > 1, n))) break;
        }
        if (ok) ok = dq(g - 1, nk > 1, n);
        if (!ok) break;
        mma_commit(acc_full);
        mma_commit(&qd_empty[qs]);
      }
    }
  } else if (warp >= 10) {
    const int r = threadIdx.x - 320;
    uint32_t g = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
      const int bh = it / nq, i = it - bh * nq, b = bh / a.nh;
      const int nk = bl_key_tiles(a, b, nk_all);
      for (int j = 0; j < nk; ++j, ++g) {
        const int as = g & 1;
        const BlAux x = bl_load_aux(a, bh, b, i * TILE, j * TILE, r);
        if (!(ok = mbar_wait(&aux_free[as], ((g >> 1) & 1) ^ 1, a.err, 128))) break;
        bl_store_aux(saux + as * kBLAux, r, x);
        mbar_arrive(&aux_full[as]);
      }
    }
  } else {
    const int quarter = warp & 3;
    const int hf = (warp - 2) >> 2;
    const int r = quarter * 32 + lane;
    const uint32_t lo = (uint32_t)(quarter * 32) << 16;
    int n = 0;
    uint32_t g = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x, ++n) {
      const int bh = it / nq, i = it - bh * nq, b = bh / a.nh, h = bh - b * a.nh;
      const int nk = bl_key_tiles(a, b, nk_all);
      for (int j = 0; j < nk; ++j, ++g) {
        const int as = g & 1;
        if (!(ok = mbar_wait_warp(&aux_full[as], (g >> 1) & 1, a.err, 129))) break;
        if (!(ok = mbar_wait_warp(s_full, g & 1, a.err, 130))) break;
        tc_fence_after();
        if (!(ok = bl_softmax_pair<T>(a, saux + as * kBLAux, r, hf * 64, tS, tdP, lo, s_free, ds_free, (g & 1) ^ 1,
                                      nullptr, sdS)))
          break;
        mbar_arrive(&aux_free[as]);
        fence_proxy_async_smem();
        mbar_arrive(ds_full);
      }
      if (!ok) break;
      if (!(ok = mbar_wait_warp(acc_full, n & 1, a.err, 131))) break;
      tc_fence_after();
      float v[32];
      tmem_ld32(tdQ + lo + hf * 32, v);
      tc_fence_before();
      mbar_arrive(acc_free);
      const int q = i * TILE + r;
      if (q < S) {
        T* dst = static_cast<T*>(a.dqkv) + ((size_t)b * S + q) * 3 * a.H + h * HD + hf * 32;
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
  if (threadIdx.x == 32) {
    // kernel parameters, not the previous kernel's output
    prefetch_tensormap(&tq);
    prefetch_tensormap(&tk);
    prefetch_tensormap(&tv);
    if (a.ctx_tma) prefetch_tensormap(&tctx);
  }
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
      // the item's global loads go out before the wait for its slot
      const bool ready = a.drop.thr && a.keep_ready;
      uint4 kb = make_uint4(0u, 0u, 0u, 0u);
      if (ready) kb = __ldg(reinterpret_cast<const uint4*>(a.keep + ((size_t)it * 128 + r) * 16));
      const int b = it / a.nh;
      const float mv = r < S && a.mask ? a.mask[(size_t)b * S + r] : 0.0f;
      if (!mbar_wait(&aux_free[j], ((n >> 1) & 1) ^ 1, a.err, 58)) break;
      if (ready) {
        // drawn ahead of this kernel (by the LayerNorm forward before it)
        *reinterpret_cast<uint4*>(sbits + j * kPFwdBits + r * 16) = kb;
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
        const uint4 kv = make_uint4(w[0], w[1], w[2], w[3]);
        *reinterpret_cast<uint4*>(sbits + j * kPFwdBits + r * 16) = kv;
        if (a.keep) *reinterpret_cast<uint4*>(a.keep + ((size_t)it * 128 + r) * 16) = kv;
      }
      smask[j * 128 + r] = r < S ? mv * kLog2e : -INFINITY;
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
// Warps 2-9 (softmax) turn item n's S and dPd into Pd and dS while warps
// 14-21 (epilogue) drain item n-1's dV, dK, dQ, and the MMA issuer puts item
// n+1's S and dPd ahead of item n's gradient products: the tensor core, the
// softmax and the epilogue each work on a different item.  dV, dK and dQ each
// have their own full/free barrier pair, so each product starts as soon as
// the epilogue has read its accumulator.  Each epilogue warp
// stages its rows through a box of its own (dQ, dK, dV in turn, each leaving
// by TMA store).
constexpr int kPBwdThreads = 704;                        // 0 TMA, 1 MMA, 2-9 softmax, 10-13 helpers, 14-21 epilogue
constexpr int kPBwdAux = 128 * 16 + 3 * 128 * 4;          // bits [128][16], mask, lse2, D [128] floats
constexpr int kPBwdStage = 8 * 2048;                      // per epilogue warp: one 32 x 64-byte box
constexpr int kPBwdSmem = 12 * TB + 2 * kPBwdAux + kPBwdStage + 1024 + 256;   // (Q,K,V,dO) x2, Pd, dS, aux x2, stage
static_assert(kPBwdSmem <= 227 * 1024, "the persistent backward's shared memory exceeds a CTA's maximum");

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
  uint8_t* sstage = saux + 2 * kPBwdAux;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sstage + kPBwdStage);
  uint64_t *in_full = bar, *in_empty = bar + 2, *s_full = bar + 4, *s_free = bar + 5, *ds_full = bar + 6,
           *aux_full = bar + 7, *aux_free = bar + 9, *g_full = bar + 11, *g_free = bar + 14;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar + 17);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = a.S;
  const int nitems = a.B * a.nh;
  if (threadIdx.x == 32) {
    // kernel parameters, not the previous kernel's output
    prefetch_tensormap(&tq);
    prefetch_tensormap(&tk);
    prefetch_tensormap(&tv);
    prefetch_tensormap(&tdo);
    if (a.ctx_tma) prefetch_tensormap(&tdqkv);
  }
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
    for (int q = 0; q < 3; ++q) {
      mbar_init(&g_full[q], 1);
      mbar_init(&g_free[q], kSoftThreads);
    }
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
      int my_items = 0;
      for (int it = blockIdx.x; it < nitems; it += gridDim.x) ++my_items;
      // S and dPd of item n (TMEM free once the softmax of item n-1 read it)
      auto mma_s = [&](int n) -> bool {
        const int j = n & 1;
        const uint32_t aQ = smem_u32(sm + j * 4 * TB), aK = aQ + TB, aV = aQ + 2 * TB, adO = aQ + 3 * TB;
        if (!mbar_wait(&in_full[j], (n >> 1) & 1, a.err, 62)) return false;
        if (!mbar_wait(s_free, (n & 1) ^ 1, a.err, 63)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) mma_f16(tS, dk_tile(aQ, kk), dk_tile(aK, kk), id_kk, kk > 0);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) mma_f16(tdP, dk_tile(adO, kk), dk_tile(aV, kk), id_kk, kk > 0);
        mma_commit(s_full);
        return true;
      };
      bool ok = my_items > 0 ? mma_s(0) : true;
      for (int n = 0; n < my_items && ok; ++n) {
        const int j = n & 1;
        const uint32_t aQ = smem_u32(sm + j * 4 * TB), aK = aQ + TB, adO = aQ + 3 * TB;
        if (!(ok = mbar_wait(ds_full, n & 1, a.err, 64))) break;
        if (n + 1 < my_items && !(ok = mma_s(n + 1))) break;
        // dV, dK, dQ one by one, each as soon as the epilogue of item n-1
        // has read that accumulator (g_free[0..2]), each with its own commit
        if (!(ok = mbar_wait(&g_free[0], (n & 1) ^ 1, a.err, 65))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < TILE / 16; ++kk) mma_f16(tdV, dmn_pair(aPd, kk), dmn_tile(adO, kk), id_mm, kk > 0);
        mma_commit(&g_full[0]);
        if (!(ok = mbar_wait(&g_free[1], (n & 1) ^ 1, a.err, 72))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < TILE / 16; ++kk) mma_f16(tdK, dmn_pair(adS, kk), dmn_tile(aQ, kk), id_mm, kk > 0);
        mma_commit(&g_full[1]);
        if (!(ok = mbar_wait(&g_free[2], (n & 1) ^ 1, a.err, 73))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < TILE / 16; ++kk) mma_f16(tdQ, dk_pair(adS, kk), dmn_tile(aK, kk), id_km, kk > 0);
        mma_commit(&g_full[2]);
        mma_commit(&in_empty[j]);
      }
    }
  } else if (warp >= 10 && warp < 14) {
    // per item: keep bits, mask row, lse2 and D of every query row.  Every
    // global load of an item (keep bits, mask, LSE, O) is issued before the
    // wait for its shared-memory slot, so their latencies overlap one another
    // and the wait.
    const int r = threadIdx.x - 320;
    const int ch = lane & 7, sub = lane >> 3, r0 = (warp - 10) * 32;
    const bool qv = r < S;
    int n = 0;
    for (int it = blockIdx.x; it < nitems; it += gridDim.x, ++n) {
      const int j = n & 1;
      const int b = it / a.nh, h = it - (it / a.nh) * a.nh;
      uint4 kb = make_uint4(0u, 0u, 0u, 0u);
      if (a.drop.thr && a.keep) kb = __ldg(reinterpret_cast<const uint4*>(a.keep + ((size_t)it * 128 + r) * 16));
      const float mv = qv && a.mask ? a.mask[(size_t)b * S + r] : 0.0f;
      const float lv = qv ? a.lse[(size_t)it * S + r] : 0.0f;
      // O for D = rowsum(dO * O) with whole-line loads: 8 lanes per 128-byte
      // row, 4 rows per load, 32 rows per warp
      const T* obase = static_cast<const T*>(a.ctx_in) + (size_t)b * S * a.H + h * HD + ch * 8;
      Raw8<T> o8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int rr = r0 + k * 4 + sub;
        o8[k] = rr < S ? raw8_load<T>(obase + (size_t)rr * a.H) : raw8_zero<T>();
      }
      uint8_t* ax = saux + j * kPBwdAux;
      float* smask = reinterpret_cast<float*>(ax + 2048);
      if (!mbar_wait(&aux_free[j], ((n >> 1) & 1) ^ 1, a.err, 69)) break;
      if (a.drop.thr && !a.keep) {
        // no stored forward bits: draw them again
        const uint64_t e8 = (((uint64_t)it * S + (uint64_t)r) * (uint64_t)S) >> 3;
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t v = 0;
#pragma unroll
          for (int g = 0; g < 4; ++g) v |= dropout_bits8(a.drop, 0, e8 + (uint64_t)(q * 4 + g)) << (8 * g);
          w[q] = v;
        }
        kb = make_uint4(w[0], w[1], w[2], w[3]);
      }
      if (a.drop.thr) *reinterpret_cast<uint4*>(ax + r * 16) = kb;
      smask[r] = qv ? mv * kLog2e : -INFINITY;
      smask[128 + r] = qv ? lv * kLog2e : INFINITY;
      // D: dO from the item's shared tile, the 8 lanes of a row reduced by shuffles
      if (!mbar_wait(&in_full[j], (n >> 1) & 1, a.err, 70)) break;
      const uint8_t* dtile = sm + j * 4 * TB + 3 * TB;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int rr = r0 + k * 4 + sub;
        float x[8], y[8];
        load8<T>(reinterpret_cast<const T*>(dtile + rr * 128 + ((ch ^ (rr & 7)) << 4)), x);
        raw8_unpack<T>(o8[k], y);
        float d = 0.0f;
#pragma unroll
        for (int t = 0; t < 8; ++t) d = fmaf(x[t], y[t], d);
        d += __shfl_xor_sync(0xffffffffu, d, 1);
        d += __shfl_xor_sync(0xffffffffu, d, 2);
        d += __shfl_xor_sync(0xffffffffu, d, 4);
        if (ch == 0) smask[256 + rr] = rr < S ? d : 0.0f;
      }
      mbar_arrive(&aux_full[j]);
    }
  } else if (warp < 10) {
    const int quarter = warp & 3;
    const int hf = (warp - 2) >> 2;
    const int r = quarter * 32 + lane;
    const uint32_t lo = (uint32_t)(quarter * 32) << 16;
    const float c2 = a.scale * kLog2e;
    const float dsc = a.drop.thr ? a.drop.scale : 1.0f;
    const int kc0 = hf * 64;
    // no mask and a full tile of keys: every mask value is 0
    const bool plain = a.mask == nullptr && S == TILE;
    int my_items = 0;
    for (int it = blockIdx.x; it < nitems; it += gridDim.x) ++my_items;
    for (int n = 0; n < my_items; ++n) {
      // ---- softmax of item n: Pd and dS into shared memory
      const int j = n & 1;
      const uint8_t* ax = saux + j * kPBwdAux;
      const float* smask = reinterpret_cast<const float*>(ax + 2048);
      if (!mbar_wait_warp(&aux_full[j], (n >> 1) & 1, a.err, 66)) break;
      const uint2 kb8 = a.drop.thr ? *reinterpret_cast<const uint2*>(ax + r * 16 + hf * 8)
                                   : make_uint2(0xFFFFFFFFu, 0xFFFFFFFFu);
      const float lse2 = smask[128 + r];
      const float Di = smask[256 + r];
      if (!mbar_wait_warp(s_full, n & 1, a.err, 67)) break;
      // the previous item's products have read its Pd and dS
      // (dQ, the last of them, is done: MMAs complete in issue order)
      if (n > 0 && !mbar_wait_warp(&g_full[2], (n - 1) & 1, a.err, 71)) break;
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float sv[16], dv[16];
        tmem_ld16x2(tS + lo + kc0 + c * 16, sv, tdP + lo + kc0 + c * 16, dv);
        const uint32_t bw = (c < 2 ? kb8.x : kb8.y) >> (16 * (c & 1));
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          const int kt = kc0 + c * 16 + g * 8;   // key column
          const uint32_t bits = (bw >> (8 * g)) & 0xFFu;
          float ml[8];
          if (plain) {
#pragma unroll
            for (int t = 0; t < 8; ++t) ml[t] = -lse2;
          } else {
            const float4 m0 = *reinterpret_cast<const float4*>(smask + kt);
            const float4 m1 = *reinterpret_cast<const float4*>(smask + kt + 4);
            ml[0] = m0.x - lse2; ml[1] = m0.y - lse2; ml[2] = m0.z - lse2; ml[3] = m0.w - lse2;
            ml[4] = m1.x - lse2; ml[5] = m1.y - lse2; ml[6] = m1.z - lse2; ml[7] = m1.w - lse2;
          }
          float pd[8], ds[8];
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            // lse2 = +inf for rows past the sequence end: p = 0
            const float p = ex2_fast(fmaf(sv[g * 8 + t], c2, ml[t]));
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
    }
  } else {
    // ---- epilogue warps: item n's dV, dK, dQ out of TMEM -> scale -> staging
    // box -> fused column sums and TMA store (whole-row-segment stores at a
    // sequence's ragged end), dQ, dK, dV in turn
    const int quarter = warp & 3;
    const int hf = (warp - 14) >> 2;
    const uint32_t lo = (uint32_t)(quarter * 32) << 16;
    // this warp's staging box: dQ, dK, dV rows (32 x 64 bytes, 64-byte swizzle) in turn
    uint8_t* stg = sstage + (warp - 14) * 2048;
    const int swz = (lane >> 1) & 3;
    // whole 32-row boxes inside the sequence leave by TMA store
    const bool tma = a.ctx_tma && quarter * 32 + 32 <= S;
    int n = 0;
    for (int it = blockIdx.x; it < nitems; it += gridDim.x, ++n) {
      const int b = it / a.nh, h = it - b * a.nh;
      // dV, dK, dQ in the order the MMA issuer produces them (w3 = 2, 1, 0),
      // each accumulator handed back right after its read
      bool ok = true;
#pragma unroll 1
      for (int w3 = 2; w3 >= 0; --w3) {
        if (!(ok = mbar_wait_warp(&g_full[2 - w3], n & 1, a.err, 68))) break;
        tc_fence_after();
        float x[32];
        tmem_ld32(tdQ - 64 * w3 + lo + hf * 32, x);
        tc_fence_before();
        mbar_arrive(&g_free[2 - w3]);
        if (w3 < 2) {
#pragma unroll
          for (int c = 0; c < 32; ++c) x[c] *= a.scale;
        }
        // the box's previous store has read it
        if (a.ctx_tma) {
          if (lane == 0) bulk_wait_read<0>();
          __syncwarp();
        }
#pragma unroll
        for (int c = 0; c < 4; ++c)
          store8<T>(reinterpret_cast<T*>(stg + lane * 64 + ((c ^ swz) << 4)), *reinterpret_cast<float(*)[8]>(x + c * 8));
        if (tma) fence_proxy_async_smem();
        __syncwarp();
        if (tma && lane == 0) {
          tma_store_2d(&tdqkv, stg, w3 * a.H + h * HD + hf * 32, b * S + quarter * 32);
          bulk_commit();
        }
        if (a.colsum) {
          // QKV bias gradient fused in: column sums of the stored (rounded)
          // values over this warp's rows inside the sequence, by a shuffle
          // reduction in registers (shared memory is the contended path here)
          const bool rv = quarter * 32 + lane < S;
#pragma unroll
          for (int c = 0; c < 32; ++c) x[c] = rv ? round_f<T>(x[c]) : 0.0f;
          const float cs = warp_colsum32(x);
          const int col = w3 * a.H + h * HD + hf * 32 + lane;
          if (a.colsum_acc) atomicAdd(a.colsum + col, cs);
          else a.colsum[(size_t)(b * 4 + quarter) * 3 * a.H + col] = cs;
        }
        if (!tma) {
          // rows r of the box: query r for dQ, key r for dK and dV; 4 lanes
          // per row's 64 bytes, 8 rows per store
          const int ch = lane & 3;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int rr = i * 8 + (lane >> 2);
            const uint4 v = *reinterpret_cast<const uint4*>(stg + rr * 64 + ((ch ^ ((rr >> 1) & 3)) << 4));
            if (quarter * 32 + rr < S)
              *reinterpret_cast<uint4*>(static_cast<T*>(a.dqkv) + ((size_t)b * S + quarter * 32 + rr) * 3 * a.H +
                                        w3 * a.H + h * HD + hf * 32 + ch * 8) = v;
          }
        }
        __syncwarp();
      }
      if (!ok) break;
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
bool encode_tile(CUtensorMap* m, const void* p, bool bf16, uint64_t cols, uint64_t rows, uint64_t ld,
                 uint32_t box_rows, bool narrow) {
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

// The same, from a cache keyed on every argument: a tensor map is a pure
// function of them (address, shape, box), so a call with the buffers of an
// earlier call encodes nothing.  Bounded: cleared when it reaches 1024 maps.
std::mutex g_map_mu;
std::map<std::tuple<uintptr_t, uint64_t, uint64_t, uint64_t, uint32_t, int, int>, CUtensorMap> g_maps;

bool map_tile(CUtensorMap* m, const void* p, bool bf16, uint64_t cols, uint64_t rows, uint64_t ld,
              uint32_t box_rows = 128, bool narrow = false) {
  const auto key = std::make_tuple(reinterpret_cast<uintptr_t>(p), cols, rows, ld, box_rows, (int)narrow, (int)bf16);
  std::lock_guard<std::mutex> lk(g_map_mu);
  const auto it = g_maps.find(key);
  if (it != g_maps.end()) {
    *m = it->second;
    return true;
  }
  if (!encode_tile(m, p, bf16, cols, rows, ld, box_rows, narrow)) return false;
  if (g_maps.size() >= 1024) g_maps.clear();
  g_maps.emplace(key, *m);
  return true;
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
  t.colsum_acc = a.colsum_acc;
  t.ctx_tma = 0;
  t.keep = a.keep;
  t.kv_ext = a.mask ? a.kv_ext : nullptr;
  t.keep_ready = a.keep && a.S <= TILE ? a.keep_ready : 0;
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
    static bool lattr = false;
    if (!lattr) {
      cudaFuncSetAttribute(attn_fwd_tc_long<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, kLSmem);
      lattr = true;
    }
    if (t.kv_ext) {
      // each sequence's key extent, so items skip key tiles past it
      launch_pdl(key_extent_kernel, a.B, 256, 0, s, a.mask, a.S, a.kv_ext);
      count_launch();
    }
    int nsm = 148;
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, 0);
    const int nitems = a.B * a.nh * ((a.S + TILE - 1) / TILE);
    CUtensorMap mc;
    t.ctx_tma = a.S % 32 == 0 && map_tile(&mc, a.ctx, t.bf16, t.H, (uint64_t)a.B * a.S, t.H, 32) ? 1 : 0;
    if (!t.ctx_tma) mc = mq;   // unused
    launch_pdl(attn_fwd_tc_long<T>, std::min(nitems, nsm), kLThreads, kLSmem, s, mq, mk, mv, mc, t);
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
  static bool lattr = false;
  if (!lattr) {
    cudaFuncSetAttribute(attn_bwd_kv_long<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, kBLKvSmem);
    cudaFuncSetAttribute(attn_bwd_q_long<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, kBLQSmem);
    lattr = true;
  }
  int nsm = 148;
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, 0);
  const int nitems = a.B * a.nh * ntile;
  launch_pdl(attn_bwd_kv_long<T>, std::min(nitems, nsm), kBLThreads, kBLKvSmem, s, mq, mk, mv, mdo, t);
  launch_pdl(attn_bwd_q_long<T>, std::min(nitems, nsm), kBLThreads, kBLQSmem, s, mq, mk, mv, mdo, t);
  count_launch(2);
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
