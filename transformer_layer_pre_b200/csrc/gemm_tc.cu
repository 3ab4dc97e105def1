// gemm_tc.cu — tcgen05 tensor-core GEMM for 16-bit storage (fp16 / bf16),
// float32 accumulation in TMEM, with the layer's fused epilogues.
//
// C[m, n] = sum_k A(m, k) B(n, k).  Each operand is K-major (row-major with
// K contiguous: activations and weights in forward, the output gradient in
// dgrad) or MN-major (K rows with M or N contiguous: the weight in dgrad,
// both operands of a weight gradient), so no operand is ever transposed in
// memory ("AI-infra engineers and the Transformer", section 2.3: the second
// FFN weight stored transposed for the backward pass is made unnecessary here
// by reading either major directly).
//
// Structure (one CTA per SM, persistent over output tiles of 128 x BN):
//   warp 0   TMA producer: per K block of 64, one 128-byte-swizzled box per
//            64-wide slice of each operand into a STAGES-deep ring
//            (no cluster multicast: every CTA loads its own tiles);
//   warp 1   allocates TMEM (two BN-column fp32 accumulators) and issues
//            tcgen05.mma (M=128, N=BN, K=16) from one thread, committing each
//            stage back to the producer and each finished tile to the epilogue;
//   warps 2-9  epilogue: two warps per TMEM lane quarter split the tile's
//            columns; tcgen05.ld 32 columns at a time, fused epilogue
//            (epilogue.cuh), global stores.  Residual / U inputs of the
//            epilogue are loaded before the accumulator is ready.
// Accumulators are double-buffered so a tile's epilogue overlaps the next
// tile's main loop.  Weight gradients (K = tokens) may split K across CTAs
// into float32 partial tiles that a second kernel sums in a fixed order.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <mutex>
#include <string>
#include <type_traits>
#include <unordered_map>
#include <vector>

#include "epilogue.cuh"
#include "kernels.h"
#include "profile.h"
#include "sm100.cuh"

namespace tlp {

using namespace sm100;

namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;   // TMA warp, MMA warp, epilogue warps

template <int BN> struct TileCfg {
  static constexpr int kStages = BN == 256 ? 4 : 6;
  static constexpr int kABytes = BM * BK * 2;
  static constexpr int kBBytes = BN * BK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kSmem = kStages * kStageBytes + 1024 + 256;
  static constexpr int kTmemCols = 2 * BN;
};

struct TcArgs {
  int M, N, K;
  int a_mn, b_mn;      // operand is MN-major
  int bf16;
  int b_early;         // B may be loaded before the wait for the previous kernel
  int tiles_m, tiles_n, splits, kb_per_split, kblocks;
  size_t split_stride;  // floats between the partial outputs of consecutive splits
  int* err;
};

__device__ __forceinline__ void decode_tile(const TcArgs& g, int t, int& mb, int& nb, int& sp) {
  const int per = g.tiles_m * g.tiles_n;
  sp = t / per;
  const int r = t - sp * per;
  mb = r / g.tiles_n;
  nb = r - mb * g.tiles_n;
}

template <typename T, int BN, int KIND>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, TcArgs g,
                   EpiParams e) {
  using C = TileCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes);
  uint64_t* empty = full + C::kStages;
  uint64_t* tfull = empty + C::kStages;
  uint64_t* tempty = tfull + 2;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(tempty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 32 * kEpiWarps);
    }
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tslot, C::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const int total = g.tiles_m * g.tiles_n * g.splits;
  pdl_wait();
  pdl_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tensormap(&tmA);
      prefetch_tensormap(&tmB);
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      uint32_t issued_phase[8];
      bool issued[8];
      for (int i = 0; i < C::kStages; ++i) issued[i] = false;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        int mb, nb, sp;
        decode_tile(g, t, mb, nb, sp);
        const int kb0 = sp * g.kb_per_split;
        const int kb1 = min(g.kblocks, kb0 + g.kb_per_split);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1u, g.err, 1)) { ok = false; break; }
          uint8_t* a_dst = smem + s * C::kStageBytes;
          uint8_t* b_dst = a_dst + C::kABytes;
          mbar_arrive_expect_tx(&full[s], C::kStageBytes);
          const int k0 = kb * BK;
          if (!g.a_mn) {
            tma_load_2d(a_dst, &tmA, &full[s], k0, mb * BM);
          } else {
#pragma unroll
            for (int j = 0; j < BM / 64; ++j) tma_load_2d(a_dst + j * 8192, &tmA, &full[s], mb * BM + 64 * j, k0);
          }
          if (!g.b_mn) {
            tma_load_2d(b_dst, &tmB, &full[s], k0, nb * BN);
          } else {
#pragma unroll
            for (int j = 0; j < BN / 64; ++j) tma_load_2d(b_dst + j * 8192, &tmB, &full[s], nb * BN + 64 * j, k0);
          }
          issued[s] = true;
          issued_phase[s] = ph;
          if (++s == C::kStages) { s = 0; ph ^= 1u; }
        }
      }
      if (!ok) {
        // wind down: let every load already issued land before the CTA exits
        for (int i = 0; i < C::kStages; ++i)
          if (issued[i]) mbar_wait(&full[i], issued_phase[i], nullptr, 0);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_f16(BM, BN, g.bf16 != 0, g.a_mn != 0, g.b_mn != 0);
      int s = 0;
      uint32_t ph = 0;
      int acc = 0;
      uint32_t aph = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        int mb, nb, sp;
        decode_tile(g, t, mb, nb, sp);
        const int kb0 = sp * g.kb_per_split;
        const int kb1 = min(g.kblocks, kb0 + g.kb_per_split);
        if (!mbar_wait(&tempty[acc], aph ^ 1u, g.err, 2)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem + acc * BN;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[s], ph, g.err, 3)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + s * C::kStageBytes);
          const uint32_t b_base = a_base + C::kABytes;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t ad = g.a_mn ? smem_desc_sw128(a_base + k * 2048, 8192, 1024)
                                       : smem_desc_sw128(a_base + k * 32, 16, 1024);
            const uint64_t bd = g.b_mn ? smem_desc_sw128(b_base + k * 2048, 8192, 1024)
                                       : smem_desc_sw128(b_base + k * 32, 16, 1024);
            mma_f16(d, ad, bd, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
          }
          mma_commit(&empty[s]);
          if (++s == C::kStages) { s = 0; ph ^= 1u; }
        }
        if (!ok) break;
        mma_commit(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) aph ^= 1u;
      }
    }
  } else {
    // Epilogue warps 2..9: warp w may access TMEM lanes 32*(w%4) .. +31 (one
    // output row per thread) and takes half of the tile's columns.
    constexpr int CW = BN / (kEpiWarps / 4);
    const int quarter = warp & 3;
    const int part = (warp - 2) >> 2;
    const int row = quarter * 32 + lane;
    int acc = 0;
    uint32_t aph = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      int mb, nb, sp;
      decode_tile(g, t, mb, nb, sp);
      const int m = mb * BM + row;
      const int nbase = nb * BN + part * CW;
      const bool mrow = m < g.M;
      // the residual / U values of this thread's columns are fetched before
      // the accumulator is ready, so their latency hides under the main loop
      uint4 pre[EpiAux<KIND>::kNeeds ? CW / 8 : 1];
      if constexpr (EpiAux<KIND>::kNeeds) {
        const T* ap = static_cast<const T*>(epi_aux_ptr(e, epi_base(KIND)));
#pragma unroll
        for (int j = 0; j < CW / 8; ++j) {
          const int n = nbase + j * 8;
          pre[j] = (ap && mrow && n < g.N) ? *reinterpret_cast<const uint4*>(ap + (size_t)m * e.ldo + n)
                                            : make_uint4(0u, 0u, 0u, 0u);
        }
      }
      size_t rb = 0;
      if constexpr (epi_base(KIND) == EPI_QKV) rb = mrow ? qkv_row_base(e, m) : 0;
      if (!mbar_wait_warp(&tfull[acc], aph, g.err, 4)) break;
      tc_fence_after();
      EpiParams ep = e;
      if constexpr (epi_base(KIND) == EPI_F32) ep.out = static_cast<float*>(e.out) + (size_t)sp * g.split_stride;
      const uint32_t tbase = tmem + ((uint32_t)(quarter * 32) << 16) + acc * BN + part * CW;
#pragma unroll
      for (int c0 = 0; c0 < CW; c0 += 32) {
        float v[32];
        tmem_ld32(tbase + c0, v);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int n = nbase + c0 + q * 8;
          if (mrow && n < g.N) {
            float aux[8];
            if constexpr (EpiAux<KIND>::kNeeds) unpack8<T>(pre[(c0 >> 3) + q], aux);
            else {
#pragma unroll
              for (int i = 0; i < 8; ++i) aux[i] = 0.0f;
            }
            epi_apply8<T, KIND>(ep, m, n, *reinterpret_cast<float(*)[8]>(v + q * 8), aux, rb);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      acc ^= 1;
      if (acc == 0) aph ^= 1u;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, C::kTmemCols);
}

// ============================================================================
// CTA-pair variant (cta_group::2): a cluster of two CTAs computes a 256 x 256
// output tile.  Each CTA loads its own 128 rows of A and its own 128 rows
// (N columns) of B into its own shared memory, signalling the leader CTA's
// "full" barrier; the leader issues tcgen05.mma.cta_group::2 (M = 256,
// N = 256), which reads both CTAs' operands and writes each CTA's 128 rows of
// the accumulator into that CTA's TMEM.  Per SM this halves the B traffic
// into shared memory (32 KB per 64-wide K block instead of 48 KB).  Commits multicast to both CTAs'
// barriers; both CTAs' epilogues arrive on the leader's "accumulator empty"
// barrier.  No TMA multicast is used.
// Six stages and one staging box per epilogue warp (225 KB of shared
// memory): against five stages with two boxes per warp, measured on the
// layer's GEMMs in isolation, 1-2 us faster per launch (the dW2|dU launch
// 7.7 us); five stages had been 1-6 us faster than four.
constexpr int kPairStages = 6;
constexpr int kPairStageBytes = 2 * 128 * BK * 2;                  // A half + B half, 32 KB
constexpr int kPairEpiWarps = 16;
constexpr int kPairThreads = 64 + 32 * kPairEpiWarps;
constexpr int kStageOut = 2048;                                    // one 32-row x 64-byte store box
constexpr int kPairOutBytes = kPairEpiWarps * kStageOut;           // one staging box per epilogue warp
constexpr int kPairSmem = kPairStages * kPairStageBytes + kPairOutBytes + 1024 + 256;
static_assert(kPairSmem <= 227 * 1024, "the pair kernel's shared memory exceeds a CTA's maximum");

// Store destinations of the pair kernel's epilogue (TMA tensor maps).
struct OutMaps {
  CUtensorMap out;    // (rows, N) row-major, box 32 rows x 128 bytes, 128-byte swizzle
  CUtensorMap out2;   // EPI_BIAS_GELU's G
  int qkv_heads_rows; // EPI_QKV: rows of one of Q/K/V viewed as (B*heads*S, 64)
  int split_rows;     // EPI_F32: rows between split partials (M rounded up to 256)
  int reduce_add;     // EPI_F32: 1 = every split adds its tile into the M-row output (TMA reduce-add)
};

// One GEMM of a pair launch: operand maps, output maps, sizes, epilogue.
struct PairGemm {
  CUtensorMap tmA, tmB;
  OutMaps om;
  TcArgs g;
  EpiParams e;
};

// Which output tiles each CTA pair computes, in order.  Round-robin (one
// GEMM): pair c takes tiles c, c + pairs, ...  Table (two GEMMs in one
// launch, e.g. a weight gradient and an input gradient that read the same
// operand): entry = gemm * 32768 + tile, planned on the host so that every
// pair gets about the same number of K blocks (longest tiles first, each to
// the pair that frees up first), which fills the pairs a lone GEMM would
// leave idle in its last wave.
constexpr int kMaxPairs = 80;
constexpr int kMaxItems = 24;
struct PairSched {
  int table;
  uint16_t n[kMaxPairs];
  uint16_t item[kMaxPairs][kMaxItems];
};

template <bool GROUP>
struct SchedIter {
  const PairSched& s;
  int cid, i, t, step, total;
  __device__ SchedIter(const PairSched& s_, const TcArgs& g0, int cid_, int ncl)
      : s(s_), cid(cid_), i(0), t(cid_), step(ncl), total(g0.tiles_m * g0.tiles_n * g0.splits) {}
  __device__ bool next(int& gi, int& tile) {
    if (!GROUP || !s.table) {
      if (t >= total) return false;
      gi = 0;
      tile = t;
      t += step;
      return true;
    }
    if (i >= s.n[cid]) return false;
    const int v = s.item[cid][i++];
    gi = v >> 15;
    tile = v & 32767;
    return true;
  }
};

// Epilogue of one tile for epilogue warp (quarter, part) of this CTA:
// TMEM accumulator `acc` -> fused epilogue -> staging box -> TMA store.  The
// warp has one staging box (32 rows x 64 bytes), reused chunk by chunk: each
// write to it first waits until the box's previous store has read it.
template <typename T, int KIND>
__device__ __forceinline__ bool pair_epilogue_tile(const OutMaps& om, const TcArgs& g, const EpiParams& e, int t,
                                                   int rank, int quarter, int part, int lane, uint32_t tmem, int acc,
                                                   uint32_t aph, uint64_t* tfull,
                                                   const uint32_t (&tempty_leader)[2], uint8_t* box) {
  constexpr int BN = 256;
  constexpr int HALF = 128;
  constexpr int CW = BN / (kPairEpiWarps / 4);              // 64 columns per warp
  constexpr int OUT_ES = epi_base(KIND) == EPI_F32 ? 4 : 2;
  constexpr int SW = 64 / OUT_ES;                          // columns per staging box: 32 (16-bit) or 16 (fp32)
  constexpr int NOUT = epi_two_outputs(KIND) ? 2 : 1;
  const int swz = (lane >> 1) & 3;                         // 64-byte swizzle of this lane's staging row
  int mb, nb, sp;
  decode_tile(g, t, mb, nb, sp);
  const int mrow0 = mb * 256 + rank * HALF + quarter * 32;   // first row of this warp's boxes
  const int m = mrow0 + lane;
  const int nbase = nb * BN + part * CW;
  const bool mrow = m < g.M;
  // The epilogue's (M, N) input (residual, U or GELU'(U)) of this warp's 32
  // rows x 64 columns is loaded row-contiguously (4 lanes per 64-byte row
  // segment, 8 rows per load) while the main loop runs: its first 32 columns
  // into the box, in the swizzled layout the outputs use, its second 32 into
  // registers, copied into the box once the first chunk's store has read it.
  // Each lane reads its own row from the box and the outputs overwrite it in
  // place.  (Row-per-lane 16-byte loads touched 32 lines per instruction.)
  static_assert(!EpiAux<KIND>::kNeeds || (NOUT == 1 && OUT_ES == 2 && CW == 2 * SW), "aux staging layout");
  bool aux_on = false;
  uint4 aux_hi[4];
  const int ach = lane & 3, arow = lane >> 2;              // 16-byte chunk of the row segment, first row
  if constexpr (EpiAux<KIND>::kNeeds) {
    const T* ap = static_cast<const T*>(epi_aux_ptr(e, epi_base(KIND)));
    aux_on = ap != nullptr;
    if (aux_on) {
      if (lane == 0) bulk_wait_read<0>();   // the box's last store has read it
      __syncwarp();
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int rl = arow + 8 * k;        // row within the warp's 32
        const int mm = mrow0 + rl;
        const int n0 = nbase + ach * 8, n1 = n0 + SW;
        const uint4 lo = (mm < g.M && n0 < g.N) ? *reinterpret_cast<const uint4*>(ap + (size_t)mm * e.ldo + n0)
                                                : make_uint4(0u, 0u, 0u, 0u);
        aux_hi[k] = (mm < g.M && n1 < g.N) ? *reinterpret_cast<const uint4*>(ap + (size_t)mm * e.ldo + n1)
                                           : make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4*>(box + rl * 64 + ((ach ^ ((rl >> 1) & 3)) << 4)) = lo;
      }
      __syncwarp();
    }
  }
  // precomputed dropout keep bits of this thread's 64 columns (one byte per 8), loaded early
  uint2 kpre = make_uint2(0u, 0u);
  bool kvalid = false;
  if constexpr (epi_base(KIND) == EPI_BIAS_DROP_RES) {
    const size_t e0 = (size_t)m * e.ldo + nbase;
    if (e.keep8 && mrow && (e0 & 63) == 0 && nbase + CW <= g.N) {
      kpre = *reinterpret_cast<const uint2*>(e.keep8 + (e0 >> 3));
      kvalid = true;
    }
  }
  if (!mbar_wait_warp(&tfull[acc], aph, g.err, 44)) return false;
  tc_fence_after();
  const uint32_t tbase = tmem + ((uint32_t)(quarter * 32) << 16) + acc * BN + part * CW;
#pragma unroll
  for (int c0 = 0; c0 < CW; c0 += SW) {
    float v[SW];
    if constexpr (SW == 32) tmem_ld32(tbase + c0, *reinterpret_cast<float(*)[32]>(v));
    else tmem_ld16(tbase + c0, *reinterpret_cast<float(*)[16]>(v));
    if (c0 + SW == CW) {
      // last TMEM read of this tile: hand the accumulator back to the leader
      tc_fence_before();
      mbar_arrive_cluster(tempty_leader[acc]);
    }
    if (!(aux_on && c0 == 0)) {
      // the box's previous store has read it (the first chunk's aux load waited already)
      if (lane == 0) bulk_wait_read<0>();
      __syncwarp();
    }
    if constexpr (EpiAux<KIND>::kNeeds) {
      if (aux_on && c0 == SW) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int rl = arow + 8 * k;
          *reinterpret_cast<uint4*>(box + rl * 64 + ((ach ^ ((rl >> 1) & 3)) << 4)) = aux_hi[k];
        }
        __syncwarp();
      }
    }
    if constexpr (OUT_ES == 4) {
      // 16 floats = four 16-byte chunks of the 64-byte row
#pragma unroll
      for (int q = 0; q < 4; ++q)
        *reinterpret_cast<float4*>(box + lane * 64 + ((q ^ swz) << 4)) =
            make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    } else {
      float v2[NOUT == 2 ? SW : 1];
#pragma unroll
      for (int q = 0; q < SW / 8; ++q) {
        const int n = nbase + c0 + q * 8;
        float* vq = v + q * 8;
        float aux[8];
        if constexpr (EpiAux<KIND>::kNeeds) {
          if (aux_on) unpack8<T>(*reinterpret_cast<const uint4*>(box + lane * 64 + ((q ^ swz) << 4)), aux);
          else {
#pragma unroll
            for (int i = 0; i < 8; ++i) aux[i] = 0.0f;
          }
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) aux[i] = 0.0f;
        }
        uint32_t kb = 0x100u;
        if constexpr (epi_base(KIND) == EPI_BIAS_DROP_RES) {
          const int j = (c0 >> 3) + q;
          if (kvalid) kb = ((j < 4 ? kpre.x : kpre.y) >> (8 * (j & 3))) & 0xFFu;
        }
        float w2[8];
        if (mrow && n < g.N) epi_compute8<T, KIND>(e, m, n, *reinterpret_cast<float(*)[8]>(vq), w2, aux, kb);
        store8<T>(reinterpret_cast<T*>(box + lane * 64 + ((q ^ swz) << 4)), *reinterpret_cast<float(*)[8]>(vq));
        if constexpr (NOUT == 2) {
#pragma unroll
          for (int i = 0; i < 8; ++i) v2[q * 8 + i] = w2[i];
        }
      }
      if constexpr (epi_sums_columns(KIND) && SW == 32) {
        // bias gradient of the FFN1 Linear fused in: column sums of the
        // stored (rounded) values of this warp's 32 rows, by a shuffle
        // reduction in registers (a read-back from the staging box instead
        // made the dW2|dU launch 3.5 us slower: it competes with the main
        // loop for shared-memory bandwidth)
        if (e.colsum) {
          float cs[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) cs[i] = (mrow && nbase + c0 + i < g.N) ? round_f<T>(v[i]) : 0.0f;
          const float tot = warp_colsum32(cs);
          const int col = nbase + c0 + lane;
          if (col < g.N) {
            if (e.accumulate) atomicAdd(e.colsum + col, tot);
            else e.colsum[(size_t)((mb * 2 + rank) * 4 + quarter) * g.N + col] = tot;
          }
        }
      }
      if constexpr (NOUT == 2) {
        // the first output leaves, then the second takes the box
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          const int x = nbase + c0;
          if (mrow0 < g.M && x < g.N) tma_store_2d(&om.out, box, x, mrow0);
          bulk_commit();
          bulk_wait_read<0>();
        }
        __syncwarp();
#pragma unroll
        for (int q = 0; q < SW / 8; ++q)
          store8<T>(reinterpret_cast<T*>(box + lane * 64 + ((q ^ swz) << 4)), *reinterpret_cast<float(*)[8]>(v2 + q * 8));
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      const int x = nbase + c0;
      if constexpr (epi_base(KIND) == EPI_QKV) {
        if (mrow0 < g.M && x < g.N) {
          const int which = (x >= e.hidden) + (x >= 2 * e.hidden);
          const int c = x - which * e.hidden;
          const int bb = mrow0 / e.seq, s0 = mrow0 - bb * e.seq;
          const int y = which * om.qkv_heads_rows + (bb * e.heads + (c >> 6)) * e.seq + s0;
          tma_store_2d(&om.out, box, c & 63, y);
        }
      } else if constexpr (epi_base(KIND) == EPI_F32) {
        if (mrow0 < g.M && x < g.N) {
          if (om.reduce_add) tma_reduce_add_2d(&om.out, box, x, mrow0);
          else tma_store_2d(&om.out, box, x, sp * om.split_rows + mrow0);
        }
      } else if constexpr (NOUT == 2) {
        if (e.out2 && mrow0 < g.M && x < g.N) tma_store_2d(&om.out2, box, x, mrow0);
      } else if (mrow0 < g.M && x < g.N) {
        tma_store_2d(&om.out, box, x, mrow0);
      }
      bulk_commit();
    }
  }
  return true;
}

// Per-item scalars of whichever GEMM a scheduled tile belongs to.
struct ItemArgs {
  int tiles_m, tiles_n, kb_per_split, kblocks, a_mn, b_mn, bf16, b_early;
};
__device__ __forceinline__ ItemArgs item_args(const TcArgs& g0, const TcArgs& g1, int gi) {
  ItemArgs a;
  a.tiles_m = gi ? g1.tiles_m : g0.tiles_m;
  a.tiles_n = gi ? g1.tiles_n : g0.tiles_n;
  a.kb_per_split = gi ? g1.kb_per_split : g0.kb_per_split;
  a.kblocks = gi ? g1.kblocks : g0.kblocks;
  a.a_mn = gi ? g1.a_mn : g0.a_mn;
  a.b_mn = gi ? g1.b_mn : g0.b_mn;
  a.bf16 = gi ? g1.bf16 : g0.bf16;
  a.b_early = gi ? g1.b_early : g0.b_early;
  return a;
}
__device__ __forceinline__ void decode_item(const ItemArgs& a, int t, int& mb, int& nb, int& kb0, int& kb1) {
  const int per = a.tiles_m * a.tiles_n;
  const int sp = t / per;
  const int r = t - sp * per;
  mb = r / a.tiles_n;
  nb = r - mb * a.tiles_n;
  kb0 = sp * a.kb_per_split;
  kb1 = min(a.kblocks, kb0 + a.kb_per_split);
}

// Kernel parameters are per GEMM and by value (the scheduled item selects
// scalars from them), so every access stays a parameter-space load.
template <typename T, int KA, int KB>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
    gemm_tc_pair_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
                        const __grid_constant__ OutMaps om0, const TcArgs g0, const EpiParams e0,
                        const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
                        const __grid_constant__ OutMaps om1, const TcArgs g1, const EpiParams e1,
                        const __grid_constant__ PairSched sch) {
  constexpr int BN = 256;
  constexpr int HALF = 128;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sout = smem + kPairStages * kPairStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sout + kPairOutBytes);
  uint64_t* empty = full + kPairStages;
  uint64_t* tfull = empty + kPairStages;
  uint64_t* tempty = tfull + 2;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(tempty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  int* const err = g0.err;
  if (threadIdx.x == 32) {
    // the tensor maps are kernel parameters, not the previous kernel's
    // output: fetch them while the setup and the dependency wait run
    prefetch_tensormap(&tmA0);
    prefetch_tensormap(&tmB0);
    prefetch_tensormap(&om0.out);
    if (sch.table) {
      prefetch_tensormap(&tmA1);
      prefetch_tensormap(&tmB1);
      prefetch_tensormap(&om1.out);
    }
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * 32 * kPairEpiWarps);
    }
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc_pair(tslot, 2 * BN);
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  // the TMA producer thread waits for the previous kernel after it has sent
  // the loads that do not depend on it; every other thread waits here
  const bool producer = warp == 0 && lane == 0;
  if (!producer) pdl_wait();
  pdl_launch_dependents();
  const int cid = blockIdx.x >> 1, ncl = gridDim.x >> 1;   // tiles_m counts 256-row pair tiles

  if (warp == 0) {
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      uint32_t issued_phase[kPairStages];
      bool issued[kPairStages];
      for (int i = 0; i < kPairStages; ++i) issued[i] = false;
      SchedIter<KA != KB> it(sch, g0, cid, ncl);
      int gi, t;
      bool have = it.next(gi, t);
      // B of the pair's first tile, when it is not the previous kernel's
      // output (a weight, or an earlier kernel's activation): its first
      // stages (fresh, so their empty barriers need no wait) go out now,
      // riding on the previous kernel's tail.  Measured in the layer step:
      // 0.690 -> 0.653 ms (the eight GEMM launches 595 -> 553 us); timed
      // alone, with no kernel before, the launches do not change.
      int pre = 0;
      if (have) {
        const ItemArgs g = item_args(g0, g1, gi);
        if (g.b_early) {
          const CUtensorMap* mB = gi ? &tmB1 : &tmB0;
          int mb, nb, kb0, kb1;
          decode_item(g, t, mb, nb, kb0, kb1);
          const int n0 = nb * BN + (int)rank * HALF;
          pre = min(kPairStages, kb1 - kb0);
          for (int i = 0; i < pre; ++i) {
            uint8_t* b_dst = smem + i * kPairStageBytes + 128 * BK * 2;
            const uint32_t fb = mapa_shared(smem_u32(&full[i]), 0);
            if (leader) mbar_arrive_expect_tx(&full[i], 2 * kPairStageBytes);
            const int k0 = (kb0 + i) * BK;
            if (!g.b_mn) {
              tma_load_2d_pair(b_dst, mB, fb, k0, n0);
            } else {
              tma_load_2d_pair(b_dst, mB, fb, n0, k0);
              tma_load_2d_pair(b_dst + 8192, mB, fb, n0 + 64, k0);
            }
          }
        }
      }
      pdl_wait();
      for (; ok && have; have = it.next(gi, t)) {
        const ItemArgs g = item_args(g0, g1, gi);
        const CUtensorMap* mA = gi ? &tmA1 : &tmA0;
        const CUtensorMap* mB = gi ? &tmB1 : &tmB0;
        int mb, nb, kb0, kb1;
        decode_item(g, t, mb, nb, kb0, kb1);
        const int m0 = mb * 256 + (int)rank * HALF;
        const int n0 = nb * BN + (int)rank * HALF;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1u, err, 41)) { ok = false; break; }
          uint8_t* a_dst = smem + s * kPairStageBytes;
          uint8_t* b_dst = a_dst + 128 * BK * 2;
          const uint32_t fb = mapa_shared(smem_u32(&full[s]), 0);
          const bool b_sent = pre > 0;   // this stage's B (and byte count) went out before the wait
          if (leader && !b_sent) mbar_arrive_expect_tx(&full[s], 2 * kPairStageBytes);
          const int k0 = kb * BK;
          if (!g.a_mn) {
            tma_load_2d_pair(a_dst, mA, fb, k0, m0);
          } else {
            tma_load_2d_pair(a_dst, mA, fb, m0, k0);
            tma_load_2d_pair(a_dst + 8192, mA, fb, m0 + 64, k0);
          }
          if (b_sent) {
            --pre;
          } else if (!g.b_mn) {
            tma_load_2d_pair(b_dst, mB, fb, k0, n0);
          } else {
            tma_load_2d_pair(b_dst, mB, fb, n0, k0);
            tma_load_2d_pair(b_dst + 8192, mB, fb, n0 + 64, k0);
          }
          issued[s] = true;
          issued_phase[s] = ph;
          if (++s == kPairStages) { s = 0; ph ^= 1u; }
        }
      }
      if (!ok && leader) {
        for (int i = 0; i < kPairStages; ++i)
          if (issued[i]) mbar_wait(&full[i], issued_phase[i], nullptr, 0);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      int s = 0;
      uint32_t ph = 0;
      int acc = 0;
      uint32_t aph = 0;
      bool ok = true;
      SchedIter<KA != KB> it(sch, g0, cid, ncl);
      int gi, t;
      while (ok && it.next(gi, t)) {
        const ItemArgs g = item_args(g0, g1, gi);
        const uint32_t idesc = idesc_f16(256, BN, g.bf16 != 0, g.a_mn != 0, g.b_mn != 0);
        int mb, nb, kb0, kb1;
        decode_item(g, t, mb, nb, kb0, kb1);
        if (!mbar_wait_cluster(&tempty[acc], aph ^ 1u, err, 42)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem + acc * BN;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[s], ph, err, 43)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + s * kPairStageBytes);
          const uint32_t b_base = a_base + 128 * BK * 2;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t ad = g.a_mn ? smem_desc_sw128(a_base + k * 2048, 8192, 1024)
                                       : smem_desc_sw128(a_base + k * 32, 16, 1024);
            const uint64_t bd = g.b_mn ? smem_desc_sw128(b_base + k * 2048, 8192, 1024)
                                       : smem_desc_sw128(b_base + k * 32, 16, 1024);
            mma_f16_pair(d, ad, bd, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
          }
          mma_commit_pair(&empty[s]);
          if (++s == kPairStages) { s = 0; ph ^= 1u; }
        }
        if (!ok) break;
        mma_commit_pair(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) aph ^= 1u;
      }
    }
  } else {
    // Epilogue warps 2..17: warp w reads TMEM lanes 32*(w%4) .. +31 (rows of
    // this CTA's half tile) and a quarter of the 256 columns.  Results go
    // through a 64-byte-swizzled staging box (32 rows x 64 bytes) and leave by
    // TMA store, so global writes are whole lines.
    const int quarter = warp & 3;
    const int part = (warp - 2) >> 2;
    uint8_t* box = sout + (warp - 2) * kStageOut;
    const uint32_t tempty_leader[2] = {mapa_shared(smem_u32(&tempty[0]), 0), mapa_shared(smem_u32(&tempty[1]), 0)};
    int acc = 0;
    uint32_t aph = 0;
    SchedIter<KA != KB> it(sch, g0, cid, ncl);
    int gi, t;
    while (it.next(gi, t)) {
      bool ok;
      if constexpr (KA == KB)
        ok = pair_epilogue_tile<T, KA>(om0, g0, e0, t, (int)rank, quarter, part, lane, tmem, acc, aph, tfull,
                                       tempty_leader, box);
      else
        ok = gi ? pair_epilogue_tile<T, KB>(om1, g1, e1, t, (int)rank, quarter, part, lane, tmem, acc, aph, tfull,
                                            tempty_leader, box)
                : pair_epilogue_tile<T, KA>(om0, g0, e0, t, (int)rank, quarter, part, lane, tmem, acc, aph, tfull,
                                            tempty_leader, box);
      if (!ok) break;
      acc ^= 1;
      if (acc == 0) aph ^= 1u;
    }
    if constexpr (KA == KB) {
      if (e0.gen_keep) {
        // pairs without a tile in the last round draw dropout keep bits
        // while the other pairs finish it (consecutive lanes, consecutive bytes)
        const int total = g0.tiles_m * g0.tiles_n * g0.splits;
        const int rem = total % ncl;
        if (rem != 0 && cid >= rem) {
          const uint64_t nthr = (uint64_t)(ncl - rem) * 2 * 32 * kPairEpiWarps;
          const uint64_t n = e0.gen_keep2 ? 2 * e0.gen_n8 : e0.gen_n8;
          for (uint64_t u = ((uint64_t)((cid - rem) * 2 + (int)rank) * kPairEpiWarps + (warp - 2)) * 32 + lane;
               u < n; u += nthr) {
            const bool second = u >= e0.gen_n8;
            const uint64_t e8 = second ? u - e0.gen_n8 : u;
            (second ? e0.gen_keep2 : e0.gen_keep)[e8] =
                (uint8_t)dropout_bits8(e0.gen_drop, e0.gen_site + (second ? 1 : 0), e8);
          }
        }
      }
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem, 2 * BN);
}

__global__ void splitk_reduce_kernel(const float* __restrict__ part, int splits, size_t stride, size_t n4,
                                     float* __restrict__ out) {
  pdl_wait();
  pdl_launch_dependents();
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n4; i += (size_t)gridDim.x * blockDim.x) {
    float4 s = reinterpret_cast<const float4*>(part)[i];
    for (int k = 1; k < splits; ++k) {
      const float4 v = reinterpret_cast<const float4*>(part + k * stride)[i];
      s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
    }
    reinterpret_cast<float4*>(out)[i] = s;
  }
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

// 2-D map over a row-major (outer, inner) matrix with row stride ld elements;
// box = box_bytes of the inner dimension (swizzled to match) x box_outer rows.
bool make_map_t(CUtensorMap* m, const void* ptr, CUtensorMapDataType dt, int es_bytes, uint64_t inner, uint64_t outer,
                uint64_t ld, uint32_t box_outer, int box_bytes = 128) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {ld * (uint64_t)es_bytes};
  cuuint32_t box[2] = {(cuuint32_t)(box_bytes / es_bytes), box_outer};
  cuuint32_t es[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            box_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map(CUtensorMap* m, const void* ptr, bool bf16, uint64_t inner, uint64_t outer, uint64_t ld,
              uint32_t box_outer) {
  return make_map_t(m, ptr, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, inner, outer,
                    ld, box_outer);
}

int num_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

// Error word of the GEMM kernels' bounded waits: four ints, [0] the error
// code, [2..3] the host-set wait limit in ns (0 = the default; sm100.cuh).
int* error_word() {
  static int* p = nullptr;
  if (!p) cudaMalloc(&p, 4 * sizeof(int)), cudaMemset(p, 0, 4 * sizeof(int));
  return p;
}

template <typename T, int BN, int KIND>
int launch_tc(const GemmDesc& gd, const EpiParams& e, int splits, cudaStream_t s) {
  using C = TileCfg<BN>;
  const bool bf16 = sizeof(T) == 2 && std::is_same<T, bf16_t>::value;
  CUtensorMap ma, mb;
  bool ok;
  if (gd.a_kmajor) ok = make_map(&ma, gd.A, bf16, gd.K, gd.M, gd.lda, BM);
  else ok = make_map(&ma, gd.A, bf16, gd.M, gd.K, gd.lda, 64);
  if (ok) {
    if (gd.b_kmajor) ok = make_map(&mb, gd.B, bf16, gd.K, gd.N, gd.ldb, BN);
    else ok = make_map(&mb, gd.B, bf16, gd.N, gd.K, gd.ldb, 64);
  }
  if (!ok) return 1;
  TcArgs g;
  g.M = gd.M; g.N = gd.N; g.K = gd.K;
  g.a_mn = gd.a_kmajor ? 0 : 1;
  g.b_mn = gd.b_kmajor ? 0 : 1;
  g.bf16 = bf16 ? 1 : 0;
  g.b_early = gd.b_early ? 1 : 0;
  g.tiles_m = (gd.M + BM - 1) / BM;
  g.tiles_n = (gd.N + BN - 1) / BN;
  g.kblocks = (gd.K + BK - 1) / BK;
  g.kb_per_split = (g.kblocks + splits - 1) / splits;
  g.splits = (g.kblocks + g.kb_per_split - 1) / g.kb_per_split;
  g.split_stride = (size_t)gd.M * gd.N;
  g.err = error_word();
  const int total = g.tiles_m * g.tiles_n * g.splits;
  const int grid = std::min(total, num_sms());
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(gemm_tc_kernel<T, BN, KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    attr = true;
  }
  launch_pdl(gemm_tc_kernel<T, BN, KIND>, grid, kThreads, C::kSmem, s, ma, mb, g, e);
  count_launch();
  return 0;
}

bool aligned16(const void* p, int ld) {
  return (reinterpret_cast<uintptr_t>(p) & 15) == 0 && ((size_t)ld * 2) % 16 == 0;
}

// Fills the operand maps, output maps and sizes of one pair-kernel GEMM.
template <typename T, int KIND>
bool build_pair_gemm(PairGemm& P, const GemmDesc& gd, const EpiParams& e, int splits) {
  const bool bf16 = std::is_same<T, bf16_t>::value;
  std::memset(&P, 0, sizeof(P));
  bool ok;
  if (gd.a_kmajor) ok = make_map(&P.tmA, gd.A, bf16, gd.K, gd.M, gd.lda, 128);
  else ok = make_map(&P.tmA, gd.A, bf16, gd.M, gd.K, gd.lda, 64);
  if (ok) {
    if (gd.b_kmajor) ok = make_map(&P.tmB, gd.B, bf16, gd.K, gd.N, gd.ldb, 128);
    else ok = make_map(&P.tmB, gd.B, bf16, gd.N, gd.K, gd.ldb, 64);
  }
  if (!ok) return false;
  TcArgs& g = P.g;
  g.M = gd.M; g.N = gd.N; g.K = gd.K;
  g.a_mn = gd.a_kmajor ? 0 : 1;
  g.b_mn = gd.b_kmajor ? 0 : 1;
  g.bf16 = bf16 ? 1 : 0;
  g.b_early = gd.b_early ? 1 : 0;
  g.tiles_m = (gd.M + 255) / 256;
  g.tiles_n = (gd.N + 255) / 256;
  g.kblocks = (gd.K + BK - 1) / BK;
  g.kb_per_split = (g.kblocks + splits - 1) / splits;
  g.splits = (g.kblocks + g.kb_per_split - 1) / g.kb_per_split;
  g.err = error_word();
  OutMaps& om = P.om;
  om.split_rows = g.tiles_m * 256;
  g.split_stride = (size_t)om.split_rows * gd.N;
  const CUtensorMapDataType t16 = bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  if constexpr (epi_base(KIND) == EPI_F32) {
    // split partials live in a workspace padded to whole 256-row tiles; the
    // unsplit output (or the one the splits add into) is exactly M rows, so
    // clipping keeps stores inside it
    om.reduce_add = g.splits > 1 && e.accumulate ? 1 : 0;
    const uint64_t rows = g.splits > 1 && !om.reduce_add ? (uint64_t)g.splits * om.split_rows : (uint64_t)gd.M;
    ok = make_map_t(&om.out, e.out, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, gd.N, rows, e.ldo, 32, 64);
  } else if constexpr (epi_base(KIND) == EPI_QKV) {
    om.qkv_heads_rows = e.tokens * (e.hidden / 64);
    ok = make_map_t(&om.out, e.out, t16, 2, 64, (uint64_t)3 * om.qkv_heads_rows, 64, 32, 64);
  } else {
    ok = make_map_t(&om.out, e.out, t16, 2, gd.N, gd.M, e.ldo, 32, 64);
    if (ok && epi_two_outputs(KIND) && e.out2) ok = make_map_t(&om.out2, e.out2, t16, 2, gd.N, gd.M, e.ldo, 32, 64);
  }
  P.e = e;
  return ok;
}

// Plans a table schedule for two GEMMs on `pairs` CTA pairs: tiles sorted by
// estimated cost (longest first, then GEMM and tile order), each given to
// the pair with the least work so far (lowest index on ties).  False if a
// pair would get more than kMaxItems tiles.
// Estimated cost of a tile in tenths of a 64-wide K block of main loop:
// its K blocks, weighted by the epilogue (the dGELU epilogue keeps the
// epilogue warps busier than the main loop of its K = 1024 tiles, measured
// ~1.45x per K block; the multiply-and-column-sum epilogue ~1.1x), plus a
// fixed per-tile fill/drain of ~4 K blocks.
int tile_cost10(int kb, int kind) {
  const int w = epi_base(kind) == EPI_DGELU ? 145 : epi_base(kind) == EPI_MUL ? 110 : 100;
  return w * kb / 10 + 40;
}

bool plan_pair_table(PairSched& sch, const TcArgs& g0, int kind0, const TcArgs& g1, int kind1, int pairs) {
  struct Item { int kb, gi, tile; };
  std::vector<Item> items;
  for (int gi = 0; gi < 2; ++gi) {
    const TcArgs& g = gi ? g1 : g0;
    const int total = g.tiles_m * g.tiles_n * g.splits;
    for (int t = 0; t < total; ++t) {
      const int sp = t / (g.tiles_m * g.tiles_n);
      const int kb0 = sp * g.kb_per_split;
      items.push_back({tile_cost10(std::min(g.kblocks, kb0 + g.kb_per_split) - kb0, gi ? kind1 : kind0), gi, t});
    }
  }
  if (items.empty() || items.size() > (size_t)pairs * kMaxItems) return false;
  std::stable_sort(items.begin(), items.end(), [](const Item& a, const Item& b) { return a.kb > b.kb; });
  std::memset(&sch, 0, sizeof(sch));
  sch.table = 1;
  std::vector<long long> load(pairs, 0);
  for (const Item& it : items) {
    int best = 0;
    for (int p = 1; p < pairs; ++p)
      if (load[p] < load[best]) best = p;
    if (sch.n[best] >= kMaxItems || it.tile >= 32768) return false;
    sch.item[best][sch.n[best]++] = (uint16_t)(it.gi * 32768 + it.tile);
    load[best] += it.kb;
  }
  return true;
}

template <typename T, int KA, int KB>
void launch_pair(const PairGemm& pa, const PairGemm& pb, const PairSched& sch, int grid, cudaStream_t s) {
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(gemm_tc_pair_kernel<T, KA, KB>, cudaFuncAttributeMaxDynamicSharedMemorySize, kPairSmem);
    attr = true;
  }
  launch_pdl(gemm_tc_pair_kernel<T, KA, KB>, grid, kPairThreads, kPairSmem, s, pa.tmA, pa.tmB, pa.om, pa.g, pa.e,
             pb.tmA, pb.tmB, pb.om, pb.g, pb.e, sch);
  count_launch();
}

// Launch cache.  The tensor maps, sizes and tile table of a pair launch
// depend only on its operands, outputs, sizes and epilogue parameters; a
// call that repeats them (every training step of a layer) reuses what the
// first one built instead of encoding the tensor maps and planning the tile
// table again.  Keyed by every field of the GEMM descriptors and epilogue
// parameters (and the device); bounded, emptied when full.
struct PairLaunch {
  PairGemm a, b;
  PairSched sch;
  int grid;
  bool grouped;   // false: a group whose table did not fit runs as two launches
};

struct LaunchKey {
  uint64_t w[96];
  int n = 0;
  void add(uint64_t v) { w[n++] = v; }
  void addp(const void* p) { add(static_cast<uint64_t>(reinterpret_cast<uintptr_t>(p))); }
  void addf(float f) {
    uint32_t u;
    std::memcpy(&u, &f, 4);
    add(u);
  }
  std::string str() const { return std::string(reinterpret_cast<const char*>(w), n * sizeof(uint64_t)); }
};

static_assert(sizeof(EpiParams) == 192 && sizeof(GemmDesc) == 80 && sizeof(DropoutParams) == 24,
              "a field was added: the launch-cache key must list it");

void key_drop(LaunchKey& k, const DropoutParams& d) {
  k.add(d.seed);
  k.add(d.offset);
  k.add(d.thr);
  k.addf(d.scale);
}

void key_gemm(LaunchKey& k, const GemmDesc& g, const EpiParams& e, int kind, int splits) {
  k.add(kind); k.add(splits);
  k.add(g.M); k.add(g.N); k.add(g.K);
  k.addp(g.A); k.add(g.lda); k.add(g.a_kmajor);
  k.addp(g.B); k.add(g.ldb); k.add(g.b_kmajor); k.add(g.b_early);
  k.add(e.kind); k.addp(e.bias); k.addp(e.res); k.addp(e.aux); k.addp(e.out); k.addp(e.out2); k.add(e.ldo);
  key_drop(k, e.drop);
  k.add(e.site); k.addp(e.keep8);
  k.add(e.seq); k.add(e.hidden); k.add(e.head_dim); k.add(e.heads); k.add(e.tokens); k.add(e.gelu_tanh);
  k.addp(e.gen_keep); k.addp(e.gen_keep2); k.add(e.gen_site); k.add(e.gen_n8);
  key_drop(k, e.gen_drop);
  k.addp(e.colsum); k.add(e.accumulate);
}

std::mutex g_launch_mu;
std::unordered_map<std::string, PairLaunch>& launch_cache() {
  static std::unordered_map<std::string, PairLaunch> m;
  return m;
}
constexpr size_t kLaunchCacheMax = 4096;

// The cached launch for `key`, built by `build` on a miss (nullptr if the
// build fails).  Call with g_launch_mu held.
template <typename Build>
const PairLaunch* cached_launch(LaunchKey& key, Build build) {
  int dev = 0;
  cudaGetDevice(&dev);
  key.add(dev);
  auto& m = launch_cache();
  const std::string ks = key.str();
  auto it = m.find(ks);
  if (it != m.end()) return &it->second;
  PairLaunch pl;
  if (!build(pl)) return nullptr;
  if (m.size() >= kLaunchCacheMax) m.clear();
  return &m.emplace(ks, pl).first->second;
}

template <typename T, int KIND>
int launch_tc_pair(const GemmDesc& gd, const EpiParams& e, int splits, cudaStream_t s) {
  LaunchKey key;
  key.add(1);
  key.add(std::is_same<T, bf16_t>::value);
  key_gemm(key, gd, e, KIND, splits);
  std::lock_guard<std::mutex> lk(g_launch_mu);
  const PairLaunch* pl = cached_launch(key, [&](PairLaunch& L) {
    if (!build_pair_gemm<T, KIND>(L.a, gd, e, splits)) return false;
    std::memset(&L.sch, 0, sizeof(L.sch));   // round-robin
    const int total = L.a.g.tiles_m * L.a.g.tiles_n * L.a.g.splits;
    L.grid = 2 * std::min(total, num_sms() / 2);
    L.grouped = false;
    return true;
  });
  if (!pl) return 1;
  launch_pair<T, KIND, KIND>(pl->a, pl->a, pl->sch, pl->grid, s);
  return 0;
}

// Two independent GEMMs in one launch on a planned table (falls back to two
// launches when the plan does not fit the table).
template <typename T, int KA, int KB>
int launch_tc_pair_group(const GemmDesc& ga, const EpiParams& ea, int splits_a, const GemmDesc& gb,
                         const EpiParams& eb, cudaStream_t s) {
  LaunchKey key;
  key.add(2);
  key.add(std::is_same<T, bf16_t>::value);
  key_gemm(key, ga, ea, KA, splits_a);
  key_gemm(key, gb, eb, KB, 1);
  bool grouped = false;
  {
    std::lock_guard<std::mutex> lk(g_launch_mu);
    const PairLaunch* pl = cached_launch(key, [&](PairLaunch& L) {
      if (!build_pair_gemm<T, KA>(L.a, ga, ea, splits_a) || !build_pair_gemm<T, KB>(L.b, gb, eb, 1)) return false;
      const int pairs = std::min(num_sms() / 2, kMaxPairs);
      L.grouped = plan_pair_table(L.sch, L.a.g, KA, L.b.g, KB, pairs);
      L.grid = 2 * pairs;
      return true;
    });
    if (!pl) return 1;
    grouped = pl->grouped;
    if (grouped) launch_pair<T, KA, KB>(pl->a, pl->b, pl->sch, pl->grid, s);
  }
  if (!grouped) {
    int rc = launch_tc_pair<T, KA>(ga, ea, splits_a, s);
    return rc ? rc : launch_tc_pair<T, KB>(gb, eb, 1, s);
  }
  return 0;
}

// Split count of a weight-gradient GEMM on CTA-pair tiles (256 x 256).
int splitk_count_pair(int M, int N, int K) {
  const int tiles = ((M + 255) / 256) * ((N + 255) / 256);
  const int kblocks = (K + BK - 1) / BK;
  const int clusters = num_sms() / 2;
  if (tiles >= (3 * clusters) / 4) return 1;
  return std::max(1, std::min(std::min(4, kblocks / 8), clusters / tiles));
}

// Split count and workspace use of a float32 weight-gradient GEMM.
int f32_splits(const GemmDesc& g) {
  const size_t rows_pad = (size_t)((g.M + 255) / 256) * 256;
  int splits = g.splitk_ws ? splitk_count_pair(g.M, g.N, g.K) : 1;
  while (splits > 1 && (size_t)splits * rows_pad * g.N > g.splitk_ws_floats) --splits;
  return splits;
}

// Sums the split partials of a float32 GEMM in split order into e.out.
void f32_split_reduce(const GemmDesc& g, const EpiParams& e, int splits, cudaStream_t s) {
  const size_t rows_pad = (size_t)((g.M + 255) / 256) * 256;
  const int kblocks = (g.K + BK - 1) / BK;
  const int kb_per = (kblocks + splits - 1) / splits;
  const int real = (kblocks + kb_per - 1) / kb_per;
  const size_t n4 = (size_t)g.M * g.N / 4;
  const size_t n = (size_t)g.M * g.N;
  if (g.defer && g.defer->n < kMaxFinalizeJobs && n % 4 == 0 && n < (1ull << 31) &&
      (reinterpret_cast<uintptr_t>(e.out) & 15) == 0) {
    g.defer->job[g.defer->n++] = {g.splitk_ws, static_cast<float*>(e.out), real, (int)n, rows_pad * g.N};
    return;
  }
  launch_pdl(splitk_reduce_kernel, (int)std::min<size_t>((n4 + 255) / 256, 148 * 8), 256, 0, s,
             static_cast<const float*>(g.splitk_ws), real, rows_pad * g.N, n4, static_cast<float*>(e.out));
  count_launch();
}

template <typename T>
int run_t(const GemmDesc& g, const EpiParams& e, cudaStream_t s) {
  if (!aligned16(g.A, g.lda) || !aligned16(g.B, g.ldb)) return 2;
  if (e.kind == EPI_F32) {
    const int splits = f32_splits(g);
    if (splits > 1 && !e.accumulate) {
      EpiParams ep = e;
      ep.out = g.splitk_ws;
      int rc = launch_tc_pair<T, EPI_F32>(g, ep, splits, s);
      if (rc) return rc;
      f32_split_reduce(g, e, splits, s);
      return 0;
    }
    return launch_tc_pair<T, EPI_F32>(g, e, splits, s);   // one split, or splits adding into e.out
  }
  switch (e.kind) {
    case EPI_QKV:
      // the staged head-split store needs whole 64-wide heads and 32-row boxes inside one sequence
      if (e.head_dim == 64 && e.seq % 32 == 0 && e.hidden % 64 == 0) return launch_tc_pair<T, EPI_QKV>(g, e, 1, s);
      return g.N > 128 ? launch_tc<T, 256, EPI_QKV>(g, e, 1, s) : launch_tc<T, 128, EPI_QKV>(g, e, 1, s);
    case EPI_BIAS_DROP_RES: return launch_tc_pair<T, EPI_BIAS_DROP_RES>(g, e, 1, s);
    case EPI_BIAS_GELU:
      return e.gelu_tanh ? launch_tc_pair<T, EPI_BIAS_GELU | EPI_TANH>(g, e, 1, s)
                         : launch_tc_pair<T, EPI_BIAS_GELU>(g, e, 1, s);
    case EPI_DGELU:
      return e.gelu_tanh ? launch_tc_pair<T, EPI_DGELU | EPI_TANH>(g, e, 1, s) : launch_tc_pair<T, EPI_DGELU>(g, e, 1, s);
    case EPI_BIAS_GELU_D:
      return e.gelu_tanh ? launch_tc_pair<T, EPI_BIAS_GELU_D | EPI_TANH>(g, e, 1, s)
                         : launch_tc_pair<T, EPI_BIAS_GELU_D>(g, e, 1, s);
    case EPI_MUL: return launch_tc_pair<T, EPI_MUL>(g, e, 1, s);
    case EPI_STORE: return launch_tc_pair<T, EPI_STORE>(g, e, 1, s);
  }
  return 1;
}

// A float32 weight gradient (ga) and an input gradient (gb, EPI_DGELU,
// EPI_MUL or EPI_STORE) in one launch.
template <typename T>
int run2_t(const GemmDesc& ga, const EpiParams& ea, const GemmDesc& gb, const EpiParams& eb, cudaStream_t s) {
  const bool groupable = ea.kind == EPI_F32 && (eb.kind == EPI_DGELU || eb.kind == EPI_MUL || eb.kind == EPI_STORE) &&
                         aligned16(ga.A, ga.lda) && aligned16(ga.B, ga.ldb) && aligned16(gb.A, gb.lda) &&
                         aligned16(gb.B, gb.ldb);
  if (!groupable) {
    const int rc = run_t<T>(ga, ea, s);
    return rc ? rc : run_t<T>(gb, eb, s);
  }
  const int splits = f32_splits(ga);
  EpiParams ep = ea;
  const bool ws = splits > 1 && !ea.accumulate;   // partials to the workspace, summed after
  if (ws) ep.out = ga.splitk_ws;
  const int rc =
      eb.kind == EPI_STORE   ? launch_tc_pair_group<T, EPI_F32, EPI_STORE>(ga, ep, splits, gb, eb, s)
      : eb.kind == EPI_MUL   ? launch_tc_pair_group<T, EPI_F32, EPI_MUL>(ga, ep, splits, gb, eb, s)
      : eb.gelu_tanh         ? launch_tc_pair_group<T, EPI_F32, EPI_DGELU | EPI_TANH>(ga, ep, splits, gb, eb, s)
                             : launch_tc_pair_group<T, EPI_F32, EPI_DGELU>(ga, ep, splits, gb, eb, s);
  if (rc) return rc;
  if (ws) f32_split_reduce(ga, ea, splits, s);
  return 0;
}

template <typename T>
int run_pair_t(const GemmDesc& g, const EpiParams& e, int splits, cudaStream_t s) {
  if (!aligned16(g.A, g.lda) || !aligned16(g.B, g.ldb)) return 2;
  switch (e.kind) {
    case EPI_QKV: return launch_tc_pair<T, EPI_QKV>(g, e, 1, s);
    case EPI_BIAS_DROP_RES: return launch_tc_pair<T, EPI_BIAS_DROP_RES>(g, e, 1, s);
    case EPI_BIAS_GELU:
      return e.gelu_tanh ? launch_tc_pair<T, EPI_BIAS_GELU | EPI_TANH>(g, e, 1, s)
                         : launch_tc_pair<T, EPI_BIAS_GELU>(g, e, 1, s);
    case EPI_DGELU:
      return e.gelu_tanh ? launch_tc_pair<T, EPI_DGELU | EPI_TANH>(g, e, 1, s) : launch_tc_pair<T, EPI_DGELU>(g, e, 1, s);
    case EPI_BIAS_GELU_D:
      return e.gelu_tanh ? launch_tc_pair<T, EPI_BIAS_GELU_D | EPI_TANH>(g, e, 1, s)
                         : launch_tc_pair<T, EPI_BIAS_GELU_D>(g, e, 1, s);
    case EPI_MUL: return launch_tc_pair<T, EPI_MUL>(g, e, 1, s);
    case EPI_STORE: return launch_tc_pair<T, EPI_STORE>(g, e, 1, s);
    case EPI_F32: return launch_tc_pair<T, EPI_F32>(g, e, splits, s);
  }
  return 1;
}

}  // namespace

int gemm_tc_bubble_pairs(int dtype, int M, int N, const EpiParams& e) {
  if (dtype == DT_F32) return 0;
  if (e.kind == EPI_QKV && !(e.head_dim == 64 && e.seq % 32 == 0 && e.hidden % 64 == 0)) return 0;
  if (e.kind != EPI_QKV && e.kind != EPI_BIAS_DROP_RES) return 0;
  const int total = ((M + 255) / 256) * ((N + 255) / 256);   // launch_tc_pair's round-robin grid
  const int ncl = std::min(total, num_sms() / 2);
  const int rem = total % ncl;
  return rem ? ncl - rem : 0;
}

// The CTA-pair GEMM directly (splits > 1 only for EPI_F32, writing split
// partials to e.out as laid out for splitk_reduce).
int gemm_tc_pair_run(int dtype, const GemmDesc& g, const EpiParams& e, int splits, cudaStream_t s) {
  return dtype == DT_F16 ? run_pair_t<half_t>(g, e, splits, s) : run_pair_t<bf16_t>(g, e, splits, s);
}

int gemm_tc_run(int dtype, const GemmDesc& g, const EpiParams& e, cudaStream_t s) {
  return dtype == DT_F16 ? run_t<half_t>(g, e, s) : run_t<bf16_t>(g, e, s);
}

int gemm_tc_run2(int dtype, const GemmDesc& ga, const EpiParams& ea, const GemmDesc& gb, const EpiParams& eb,
                 cudaStream_t s) {
  return dtype == DT_F16 ? run2_t<half_t>(ga, ea, gb, eb, s) : run2_t<bf16_t>(ga, ea, gb, eb, s);
}

size_t gemm_tc_splitk_ws_floats(int M, int N, int K) {
  const int sp = splitk_count_pair(M, N, K);
  return sp > 1 ? (size_t)sp * ((M + 255) / 256) * 256 * N : 0;
}

// Sets the wait limit (ns, 0 = default) the GEMM kernels' waits read.
void gemm_tc_set_wait_limit(uint64_t ns) {
  cudaMemcpy(error_word() + 2, &ns, sizeof(ns), cudaMemcpyHostToDevice);
}

// One thread waits, with the library's bounded wait and the GEMM error word,
// on an mbarrier that nothing ever arrives on: the wait runs out after the
// limit and records code 99.  Nothing asynchronous is in flight meanwhile.
__global__ void wait_probe_kernel(int* err) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, err, 99);
  __syncthreads();
}

void gemm_tc_wait_probe(cudaStream_t s) {
  wait_probe_kernel<<<1, 32, 0, s>>>(error_word());
  count_launch();
}

// Reads and clears the bounded-wait error word of the tensor-core kernels.
int gemm_tc_take_error() {
  int v = 0;
  int* p = error_word();
  cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost);
  if (v) cudaMemset(p, 0, sizeof(int));
  return v;
}

}  // namespace tlp
