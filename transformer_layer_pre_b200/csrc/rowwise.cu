// rowwise.cu — bandwidth-bound kernels over (rows, H) activations:
// LayerNorm forward/backward, dropout backward, column sums, GELU, mask dump.
//
// LayerNorm is per token over the hidden axis with the biased variance and
// eps inside the square root; statistics are float32 ("AI-infra engineers and
// the Transformer", section 3.2: LayerNorm kept in fp32).  A block owns a
// contiguous range of rows, streamed into shared memory by bulk asynchronous
// copies, and each thread 8 consecutive columns of them, so column sums (bias
// and LayerNorm-parameter gradients) accumulate in the owning thread's
// registers in row order and leave as one partial row per block, summed by
// tlp::colsum_finalize_run in block order: deterministic.  (With the
// stochastic-mode flag of a launch, each block instead adds its row into the
// gradient itself with atomics.)
#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "profile.h"
#include "sm100.cuh"

namespace tlp {

namespace {

// Row-block kernels: a block owns a contiguous range of rows; thread t owns
// columns 8t .. 8t+7 of every row of that range.  Thread 0 streams the rows
// into shared memory kRowsPer rows at a time with bulk asynchronous copies,
// kStages groups ahead, so DRAM stays busy while the block computes; the
// other threads read their columns from shared memory.  Row statistics are
// block reductions (one per group); column sums stay in the owning thread's
// registers and leave as one partial row per block.
constexpr int kStages = 4;
constexpr int kMaxBlocks = 296;        // 2 blocks per SM
// error word of the row kernels' bounded waits (layout in sm100.cuh)
__device__ __align__(16) int g_row_err[4];

__host__ __device__ inline int row_threads(int H) { return ((H / 8 + 31) / 32) * 32; }

// Rows per pipeline group: a group of one tensor is at most 8 KB.
__host__ __device__ inline int group_rows(int H, int es) {
  const int r = 8192 / (H * es);
  return r >= 4 ? 4 : (r >= 2 ? 2 : 1);
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   sm100::smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(sm100::smem_u32(bar))
               : "memory");
}

// Sums v[r] over the whole block; red holds (warps, KR) floats.
template <int KR>
__device__ __forceinline__ void block_sum(float (&v)[KR], float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int r = 0; r < KR; ++r) v[r] = warp_sum(v[r]);
  if (lane == 0) {
#pragma unroll
    for (int r = 0; r < KR; ++r) red[warp * KR + r] = v[r];
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < KR; ++r) {
    float s = 0.0f;
    for (int w = 0; w < nw; ++w) s += red[w * KR + r];
    v[r] = s;
  }
  __syncthreads();
}

__device__ __forceinline__ void row_range(int rows, int& r0, int& r1) {
  const int per = (rows + gridDim.x - 1) / gridDim.x;
  r0 = blockIdx.x * per;
  r1 = min(rows, r0 + per);
}

// A block's column sums of 8 columns: its own row of `part` (summed later in
// a fixed order) or, with add, added into row 0 (arrival order).
__device__ __forceinline__ void store_part(float* part, int H, int col, const float (&acc)[8], int add) {
  if (add) {
#pragma unroll
    for (int i = 0; i < 8; ++i) atomicAdd(part + col + i, acc[i]);
    return;
  }
  float* p = part + (size_t)blockIdx.x * H + col;
  reinterpret_cast<float4*>(p)[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
}

// Pipeline of row groups: NT tensors of row stride H elements, KR rows per
// group, kStages groups in flight.  Layout per stage: NT x [KR][H].
template <typename T, int KR, int NT>
struct RowPipe {
  uint8_t* buf;
  uint64_t* full;
  const T* src[NT];
  int H, r0, r1, ngroups;

  __device__ size_t tensor_bytes() const { return (size_t)KR * H * sizeof(T); }
  __device__ size_t stage_bytes() const { return NT * tensor_bytes(); }

  __device__ void init(uint8_t* smem, int H_, int r0_, int r1_) {
    H = H_; r0 = r0_; r1 = r1_;
    ngroups = (r1 - r0 + KR - 1) / KR;
    buf = smem;
    full = reinterpret_cast<uint64_t*>(smem + kStages * stage_bytes());
    if (threadIdx.x == 0) {
      for (int s = 0; s < kStages; ++s) sm100::mbar_init(&full[s], 1);
      sm100::fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0)
      for (int g = 0; g < kStages && g < ngroups; ++g) issue(g);
  }
  // thread 0: copy group g into its stage
  __device__ void issue(int g) {
    const int s = g % kStages;
    const int row = r0 + g * KR;
    const uint32_t bytes = (uint32_t)(min(KR, r1 - row) * (size_t)H * sizeof(T));
    uint8_t* dst = buf + s * stage_bytes();
    sm100::mbar_arrive_expect_tx(&full[s], NT * bytes);
#pragma unroll
    for (int t = 0; t < NT; ++t) bulk_load(dst + t * tensor_bytes(), src[t] + (size_t)row * H, bytes, &full[s]);
  }
  // every thread: wait for group g; false if the wait gave up
  __device__ bool wait(int g) {
    return sm100::mbar_wait(&full[g % kStages], (uint32_t)((g / kStages) & 1), g_row_err, 1);
  }
  __device__ const T* row(int g, int t, int r) const {
    return reinterpret_cast<const T*>(buf + (g % kStages) * stage_bytes() + t * tensor_bytes()) + (size_t)r * H;
  }
  // after every thread is done with group g (block barrier): refill its stage
  __device__ void release(int g) {
    if (threadIdx.x == 0 && g + kStages < ngroups) {
      sm100::fence_proxy_async_smem();
      issue(g + kStages);
    }
  }
  // an abandoned pipeline still has copies in flight: let them land
  __device__ void drain(int g) {
    if (threadIdx.x == 0)
      for (int k = g; k < ngroups && k < g + kStages; ++k) sm100::mbar_wait(&full[k % kStages], (k / kStages) & 1, nullptr, 0);
  }
};

template <typename T, int KR, int NT>
size_t pipe_smem(int H) {
  return (size_t)kStages * NT * KR * H * sizeof(T) + kStages * sizeof(uint64_t) + 32 * 2 * KR * sizeof(float);
}

// ------------------------------------------------------------------ LayerNorm forward
// One warp per row, lane-interleaved chunks of 8 columns (16-byte vectors),
// shuffle-only reductions, no shared memory and no block barrier: a warp
// issues its rows' loads first (streaming, not kept in L1) and gamma/beta
// through the read-only path (every warp reads the same H values, so they
// stay cached).  NCH = chunks of 8 per lane (H <= 256*NCH).
constexpr int kFwdWarps = 4;

__device__ __forceinline__ uint4 ldg_stream16(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}
template <typename T> __device__ __forceinline__ Raw8<T> raw8_stream(const T* p) {
  Raw8<T> r;
  r.a = ldg_stream16(p);
  return r;
}
template <> __device__ __forceinline__ Raw8<float> raw8_stream<float>(const float* p) {
  Raw8<float> r;
  const uint4 a = ldg_stream16(p), b = ldg_stream16(p + 4);
  r.a = make_float4(__uint_as_float(a.x), __uint_as_float(a.y), __uint_as_float(a.z), __uint_as_float(a.w));
  r.b = make_float4(__uint_as_float(b.x), __uint_as_float(b.y), __uint_as_float(b.z), __uint_as_float(b.w));
  return r;
}
template <typename T> __device__ __forceinline__ void load8_ro(const T* p, float (&v)[8]) {
  Raw8<T> r;
  r.a = __ldg(reinterpret_cast<const uint4*>(p));
  raw8_unpack<T>(r, v);
}
template <> __device__ __forceinline__ void load8_ro<float>(const float* p, float (&v)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p)), b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

template <typename T, int NCH, int RPW>
__global__ void __launch_bounds__(kFwdWarps * 32) ln_fwd_kernel(const T* __restrict__ x, const T* __restrict__ gamma,
                                                                const T* __restrict__ beta, T* __restrict__ y,
                                                                float* __restrict__ mean_out,
                                                                float* __restrict__ rstd_out, int rows, int H,
                                                                float eps, uint8_t* __restrict__ keep_out,
                                                                DropoutParams dp, int site, AttnKeepGen ak) {
  pdl_wait();
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  // a warp owns RPW consecutive rows; every load of all of them is issued
  // before the first row's arithmetic, so RPW rows' bytes are in flight
  const int row0 = (blockIdx.x * kFwdWarps + (threadIdx.x >> 5)) * RPW;
  if (row0 >= rows) return;
  Raw8<T> raw[RPW][NCH];
#pragma unroll
  for (int q = 0; q < RPW; ++q) {
    const int row = row0 + q;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      const int col = (lane + 32 * c) * 8;
      raw[q][c] = (row < rows && col < H) ? raw8_stream<T>(x + (size_t)row * H + col) : raw8_zero<T>();
    }
  }
  if (keep_out) {
    // dropout keep bits of these rows for a downstream kernel (element index
    // row*H + col), drawn while the rows' loads are in flight
#pragma unroll
    for (int q = 0; q < RPW; ++q) {
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
        const int col = (lane + 32 * c) * 8;
        if (row0 + q < rows && col < H) {
          const uint64_t e8 = ((uint64_t)(row0 + q) * H + col) >> 3;
          keep_out[e8] = (uint8_t)dropout_bits8(dp, site, e8);
        }
      }
    }
  }
  if (ak.keep) {
    // the attention-probability keep bits of the queries these rows are (site
    // 0): 16 bytes per head, 8 per lane and step, drawn while the loads are in flight
#pragma unroll
    for (int q = 0; q < RPW; ++q) {
      const int row = row0 + q;
      if (row < rows) {
        const int b = row / ak.S, sq = row - b * ak.S;
        for (int c = lane; c < ak.nh * 2; c += 32) {
          const int h = c >> 1, q0 = (c & 1) * 8;
          const uint64_t e8 = ((((uint64_t)(b * ak.nh + h)) * ak.S + sq) * ak.S >> 3) + q0;
          uint32_t w0 = 0, w1 = 0;
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            w0 |= dropout_bits8(ak.dp, 0, e8 + g) << (8 * g);
            w1 |= dropout_bits8(ak.dp, 0, e8 + 4 + g) << (8 * g);
          }
          *reinterpret_cast<uint2*>(ak.keep + ((size_t)(b * ak.nh + h) * 128 + sq) * 16 + q0) = make_uint2(w0, w1);
        }
      }
    }
  }
  const float inv_h = 1.0f / (float)H;
#pragma unroll
  for (int q = 0; q < RPW; ++q) {
    const int row = row0 + q;
    if (row >= rows) break;
    float v[NCH][8];
    float s = 0.0f;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      raw8_unpack<T>(raw[q][c], v[c]);
#pragma unroll
      for (int i = 0; i < 8; ++i) s += v[c][i];
    }
    const float mean = warp_sum(s) * inv_h;
    float ss = 0.0f;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      if ((lane + 32 * c) * 8 < H) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float d = v[c][i] - mean;
          ss += d * d;
        }
      }
    }
    const float rstd = 1.0f / sqrtf(warp_sum(ss) * inv_h + eps);
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      const int col = (lane + 32 * c) * 8;
      if (col < H) {
        float g[8], b[8], o[8];
        load8_ro<T>(gamma + col, g);
        load8_ro<T>(beta + col, b);
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] = g[i] * ((v[c][i] - mean) * rstd) + b[i];
        store8<T>(y + (size_t)row * H + col, o);
      }
    }
    if (lane == 0) {
      mean_out[row] = mean;
      rstd_out[row] = rstd;
    }
  }
}

// ------------------------------------------------------------------ LayerNorm backward
// Pipeline tensors: 0 dy, 1 x (or y when invertible), 2 res (when given).
template <typename T, bool INV, bool RES, int KR>
__global__ void __launch_bounds__(512) ln_bwd_kernel(LnBwdArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int NT = RES ? 3 : 2;
  const int H = a.H;
  const int col = threadIdx.x * 8;
  const bool act = col < H;
  float gm[8], bt[8];
  float dg[8], db[8], ds[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) dg[i] = db[i] = ds[i] = 0.0f;
  if (act) {
    load8<T>(static_cast<const T*>(a.gamma) + col, gm);
    if constexpr (INV) load8<T>(static_cast<const T*>(a.beta) + col, bt);
  }
  const float inv_h = 1.0f / (float)H;
  const float sc = a.drop.thr ? a.drop.scale : 1.0f;
  int r0, r1;
  row_range(a.rows, r0, r1);
  RowPipe<T, KR, NT> pipe;
  pipe.src[0] = static_cast<const T*>(a.dy);
  pipe.src[1] = static_cast<const T*>(INV ? a.y : a.x);
  if constexpr (RES) pipe.src[2] = static_cast<const T*>(a.res);
  pipe.init(smem, H, r0, r1);
  float* red = reinterpret_cast<float*>(pipe.full + kStages);
  for (int gi = 0; gi < pipe.ngroups; ++gi) {
    const bool ok = pipe.wait(gi);
    if (__syncthreads_or(!ok)) { pipe.drain(gi); return; }
    const int base = r0 + gi * KR;
    float g[KR][8], xh[KR][8], s1[KR], s2[KR], rs[KR];
#pragma unroll
    for (int r = 0; r < KR; ++r) {
      s1[r] = s2[r] = 0.0f;
      const int row = base + r;
      rs[r] = row < r1 ? a.rstd[row] : 0.0f;
      if (act && row < r1) {
        float dy[8], xv[8];
        load8<T>(pipe.row(gi, 0, r) + col, dy);
        load8<T>(pipe.row(gi, 1, r) + col, xv);
        if constexpr (INV) {
#pragma unroll
          for (int i = 0; i < 8; ++i) xh[r][i] = (xv[i] - bt[i]) / gm[i];
        } else {
          const float mean = a.mean[row];
#pragma unroll
          for (int i = 0; i < 8; ++i) xh[r][i] = (xv[i] - mean) * rs[r];
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          g[r][i] = dy[i] * gm[i];
          s1[r] += g[r][i];
          s2[r] += g[r][i] * xh[r][i];
          dg[i] += dy[i] * xh[r][i];
          db[i] += dy[i];
        }
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) g[r][i] = xh[r][i] = 0.0f;
      }
    }
    float s12[2 * KR];
#pragma unroll
    for (int r = 0; r < KR; ++r) {
      s12[r] = s1[r];
      s12[KR + r] = s2[r];
    }
    block_sum<2 * KR>(s12, red);
#pragma unroll
    for (int r = 0; r < KR; ++r) {
      const int row = base + r;
      if (!act || row >= r1) continue;
      const size_t off = (size_t)row * H + col;
      const float m1 = s12[r] * inv_h, m2 = s12[KR + r] * inv_h;
      float o[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = rs[r] * (g[r][i] - m1 - xh[r][i] * m2);
      if constexpr (RES) {
        float rv[8];
        load8<T>(pipe.row(gi, 2, r) + col, rv);
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] += rv[i];
      }
      store8<T>(static_cast<T*>(a.dx) + off, o);
      if (a.drop_out) {
        const uint32_t bits = a.keep8 ? (uint32_t)a.keep8[off >> 3]
                                      : (a.drop.thr ? dropout_bits8(a.drop, a.site, off >> 3) : 0xFFu);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          o[i] = round_f<T>(((bits >> i) & 1u) ? round_f<T>(o[i]) * sc : 0.0f);
          ds[i] += o[i];
        }
        store8<T>(static_cast<T*>(a.drop_out) + off, o);
      }
    }
    __syncthreads();
    pipe.release(gi);
  }
  if (act) {
    store_part(a.part_dgamma, H, col, dg, a.part_acc);
    store_part(a.part_dbeta, H, col, db, a.part_acc);
    if (a.part_dsum) store_part(a.part_dsum, H, col, ds, a.part_acc);
  }
}

// LayerNorm backward for H <= 1024: two warps per row (64 lanes, lane L owns
// the 8-column chunks L, L+64, ...; NC chunks), no block-wide barrier inside
// the row loop.  A block owns a contiguous range of rows; its kLnbPairs warp
// pairs take every kLnbPairs-th row and load the pair's next row before
// working on the current one.  The row sums of the two warps meet in shared
// memory behind a 64-thread named barrier.  Each lane keeps the column sums
// (dgamma, dbeta and, with a dropout copy, the dropped gradient) of its own
// columns in registers; at the end the block adds its pairs' sums in shared
// memory in pair order, leaving one partial row per block.
constexpr int kLnbPairs = 4;

template <typename T, bool INV, bool RES, bool DROP, int NC>
__global__ void __launch_bounds__(kLnbPairs * 64, (sizeof(T) == 4 || (INV && DROP)) ? 1 : 2) ln_bwd_warp_kernel(LnBwdArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  extern __shared__ __align__(16) float red[];   // [kLnbPairs][H]; row exchange after it
  float* xch = red + kLnbPairs * a.H;            // [pair][row parity][half][2]
  const int H = a.H;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int pair = warp >> 1, half = warp & 1;
  const int L = half * 32 + lane;
  const float inv_h = 1.0f / (float)H;
  const float sc = a.drop.thr ? a.drop.scale : 1.0f;
  const T* dyp = static_cast<const T*>(a.dy);
  const T* xp = static_cast<const T*>(INV ? a.y : a.x);
  const T* rp = static_cast<const T*>(a.res);
  float dg[NC][8], db[NC][8], ds[DROP ? NC : 1][8];
#pragma unroll
  for (int c = 0; c < NC; ++c)
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      dg[c][i] = db[c][i] = 0.0f;
      if constexpr (DROP) ds[c][i] = 0.0f;
    }
  int r0, r1;
  row_range(a.rows, r0, r1);
  Raw8<T> rdy[NC], rx[NC];
  float rs_n = 0.0f, mean_n = 0.0f;   // the fetched row's rstd and mean
  auto fetch = [&](int row) {
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      const int col = (L + 64 * c) * 8;
      const bool in = row < r1 && col < H;
      const size_t off = (size_t)row * H + col;
      rdy[c] = in ? raw8_stream<T>(dyp + off) : raw8_zero<T>();
      rx[c] = in ? raw8_stream<T>(xp + off) : raw8_zero<T>();
    }
    if (row < r1) {
      rs_n = __ldg(a.rstd + row);
      if constexpr (!INV) mean_n = __ldg(a.mean + row);
    }
  };
  int row = r0 + pair;
  fetch(row);
  for (int k = 0; row < r1; row += kLnbPairs, ++k) {
    float dy[NC][8], xh[NC][8];
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      raw8_unpack<T>(rdy[c], dy[c]);
      raw8_unpack<T>(rx[c], xh[c]);
    }
    const float rs = rs_n;
    const float mean = INV ? 0.0f : mean_n;
    fetch(row + kLnbPairs);
    Raw8<T> rr[RES ? NC : 1];
    if constexpr (RES) {
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        const int col = (L + 64 * c) * 8;
        rr[c] = col < H ? raw8_stream<T>(rp + (size_t)row * H + col) : raw8_zero<T>();
      }
    }
    // keep bits of the dropout copy, loaded with the residual (consumed after the row sums)
    uint32_t kb[DROP ? NC : 1];
    if constexpr (DROP) {
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        const int col = (L + 64 * c) * 8;
        kb[c] = a.keep8 && col < H ? (uint32_t)__ldg(a.keep8 + (((size_t)row * H + col) >> 3)) : 0xFFu;
      }
    }
    float s1 = 0.0f, s2 = 0.0f;
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      const int col = (L + 64 * c) * 8;
      if (col >= H) continue;
      float gm[8];
      load8_ro<T>(static_cast<const T*>(a.gamma) + col, gm);
      if constexpr (INV) {
        float bt[8];
        load8_ro<T>(static_cast<const T*>(a.beta) + col, bt);
#pragma unroll
        for (int i = 0; i < 8; ++i) xh[c][i] = (xh[c][i] - bt[i]) / gm[i];
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) xh[c][i] = (xh[c][i] - mean) * rs;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        dg[c][i] += dy[c][i] * xh[c][i];
        db[c][i] += dy[c][i];
        dy[c][i] *= gm[i];                 // g = dy * gamma from here on
        s1 += dy[c][i];
        s2 += dy[c][i] * xh[c][i];
      }
    }
    s1 = warp_sum(s1);
    s2 = warp_sum(s2);
    float* xr = xch + (pair * 2 + (k & 1)) * 4;
    if (lane == 0) {
      xr[half * 2] = s1;
      xr[half * 2 + 1] = s2;
    }
    sm100::named_barrier(1 + pair, 64);
    const float m1 = (xr[0] + xr[2]) * inv_h, m2 = (xr[1] + xr[3]) * inv_h;
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      const int col = (L + 64 * c) * 8;
      if (col >= H) continue;
      const size_t off = (size_t)row * H + col;
      float o[8];
      float rv[8];
      if constexpr (RES) raw8_unpack<T>(rr[c], rv);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        o[i] = rs * (dy[c][i] - m1 - xh[c][i] * m2);
        if constexpr (RES) o[i] += rv[i];
      }
      store8<T>(static_cast<T*>(a.dx) + off, o);
      if constexpr (DROP) {
        const uint32_t bits = a.keep8 ? kb[c] : (a.drop.thr ? dropout_bits8(a.drop, a.site, off >> 3) : 0xFFu);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          o[i] = round_f<T>(((bits >> i) & 1u) ? round_f<T>(o[i]) * sc : 0.0f);
          ds[c][i] += o[i];
        }
        store8<T>(static_cast<T*>(a.drop_out) + off, o);
      }
    }
  }
  // block sums in pair order, one tensor at a time
  auto reduce = [&](float (*acc)[8], float* part) {
    __syncthreads();
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      const int col = (L + 64 * c) * 8;
      if (col < H) {
        float* d = red + pair * H + col;
        reinterpret_cast<float4*>(d)[0] = make_float4(acc[c][0], acc[c][1], acc[c][2], acc[c][3]);
        reinterpret_cast<float4*>(d)[1] = make_float4(acc[c][4], acc[c][5], acc[c][6], acc[c][7]);
      }
    }
    __syncthreads();
    for (int col = threadIdx.x; col < H; col += blockDim.x) {
      float t = 0.0f;
#pragma unroll
      for (int w = 0; w < kLnbPairs; ++w) t += red[w * H + col];
      if (a.part_acc) atomicAdd(part + col, t);
      else part[(size_t)blockIdx.x * H + col] = t;
    }
  };
  reduce(dg, a.part_dgamma);
  reduce(db, a.part_dbeta);
  if constexpr (DROP) reduce(ds, a.part_dsum);
}

// ------------------------------------------------------------------ dropout of rows
template <typename T, int KR>
__global__ void __launch_bounds__(512) dropout_rows_kernel(const T* __restrict__ in, T* __restrict__ out,
                                                           DropoutParams dp, int site, int rows, int H,
                                                           float* __restrict__ part,
                                                           const uint8_t* __restrict__ keep8, int padd) {
  pdl_wait();
  pdl_launch_dependents();
  extern __shared__ __align__(128) uint8_t smem[];
  const int col = threadIdx.x * 8;
  const bool act = col < H;
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  const float sc = dp.thr ? dp.scale : 1.0f;
  int r0, r1;
  row_range(rows, r0, r1);
  RowPipe<T, KR, 1> pipe;
  pipe.src[0] = in;
  pipe.init(smem, H, r0, r1);
  for (int gi = 0; gi < pipe.ngroups; ++gi) {
    const bool ok = pipe.wait(gi);
    if (__syncthreads_or(!ok)) { pipe.drain(gi); return; }
    const int base = r0 + gi * KR;
#pragma unroll
    for (int r = 0; r < KR; ++r) {
      const int row = base + r;
      if (!act || row >= r1) continue;
      const size_t off = (size_t)row * H + col;
      float v[8];
      load8<T>(pipe.row(gi, 0, r) + col, v);
      const uint32_t bits = keep8 ? (uint32_t)keep8[off >> 3] : (dp.thr ? dropout_bits8(dp, site, off >> 3) : 0xFFu);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        v[i] = round_f<T>(((bits >> i) & 1u) ? v[i] * sc : 0.0f);
        acc[i] += v[i];
      }
      store8<T>(out + off, v);
    }
    __syncthreads();
    pipe.release(gi);
  }
  if (act) store_part(part, H, col, acc, padd);
}

// Dropout backward for H <= 1024 with precomputed keep bits: one warp per
// row (lane-interleaved 8-column chunks, NCH per lane), the next row's data
// and keep bytes loaded before the current row is written; column sums in
// registers, added over the block's 8 warps in warp order at the end (one
// partial row per block, like the row-block kernel above).
constexpr int kDropWarps = 8;

template <typename T, int NCH>
__global__ void __launch_bounds__(kDropWarps * 32) dropout_rows_warp_kernel(const T* __restrict__ in,
                                                                            T* __restrict__ out, float scale,
                                                                            int rows, int H, float* __restrict__ part,
                                                                            const uint8_t* __restrict__ keep8,
                                                                            int padd) {
  pdl_wait();
  pdl_launch_dependents();
  extern __shared__ __align__(16) float dred[];   // [kDropWarps][H]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float acc[NCH][8];
#pragma unroll
  for (int c = 0; c < NCH; ++c)
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[c][i] = 0.0f;
  int r0, r1;
  row_range(rows, r0, r1);
  Raw8<T> rv[NCH];
  uint32_t kb[NCH];
  auto fetch = [&](int row) {
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      const int col = (lane + 32 * c) * 8;
      const bool ok = row < r1 && col < H;
      const size_t off = (size_t)row * H + col;
      rv[c] = ok ? raw8_stream<T>(in + off) : raw8_zero<T>();
      kb[c] = ok ? (uint32_t)keep8[off >> 3] : 0u;
    }
  };
  int row = r0 + warp;
  fetch(row);
  for (; row < r1; row += kDropWarps) {
    float v[NCH][8];
    uint32_t bits[NCH];
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      raw8_unpack<T>(rv[c], v[c]);
      bits[c] = kb[c];
    }
    fetch(row + kDropWarps);
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      const int col = (lane + 32 * c) * 8;
      if (col >= H) continue;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        v[c][i] = round_f<T>(((bits[c] >> i) & 1u) ? v[c][i] * scale : 0.0f);
        acc[c][i] += v[c][i];
      }
      store8<T>(out + (size_t)row * H + col, v[c]);
    }
  }
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    const int col = (lane + 32 * c) * 8;
    if (col < H) {
      float* d = dred + warp * H + col;
      reinterpret_cast<float4*>(d)[0] = make_float4(acc[c][0], acc[c][1], acc[c][2], acc[c][3]);
      reinterpret_cast<float4*>(d)[1] = make_float4(acc[c][4], acc[c][5], acc[c][6], acc[c][7]);
    }
  }
  __syncthreads();
  for (int col = threadIdx.x; col < H; col += blockDim.x) {
    float t = 0.0f;
#pragma unroll
    for (int w = 0; w < kDropWarps; ++w) t += dred[w * H + col];
    if (padd) atomicAdd(part + col, t);
    else part[(size_t)blockIdx.x * H + col] = t;
  }
}

// ------------------------------------------------------------------ column sums
constexpr int kColParts = 64;

template <typename T>
__global__ void __launch_bounds__(256) colsum_kernel(const T* __restrict__ X, int rows, int cols,
                                                     float* __restrict__ part, int padd) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ float red[8][256 + 8];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int c0 = (blockIdx.x * 32 + tx) * 8;
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  if (c0 < cols) {
    for (int r = blockIdx.y * 8 + ty; r < rows; r += 8 * gridDim.y) {
      float v[8];
      load8<T>(X + (size_t)r * cols + c0, v);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += v[i];
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) red[ty][tx * 8 + i] = acc[i];
  __syncthreads();
  const int c = blockIdx.x * 256 + threadIdx.x;
  if (c < cols) {
    float s = 0.0f;
    for (int w = 0; w < 8; ++w) s += red[w][threadIdx.x];
    if (padd) atomicAdd(part + c, s);
    else part[(size_t)blockIdx.y * cols + c] = s;
  }
}

// The closing sums of a backward pass, in one launch.  Blocks are numbered
// over all jobs (first[j] = the first block of job j).  A column-sum job
// gives each block 32 columns: 8 column groups of 4 (float4 loads) x 32
// part lanes, lane l summing partial rows l, l+32, ..., then the 32 lane sums
// in lane order (a fixed order).  (Up to ten loads per thread, all issued
// before the first add, so a block waits about one memory latency, not one
// per load.)  A split-K job sums its partial matrices element-wise, four
// floats a thread, partials in increasing order.
constexpr int kFinCols = 32;
constexpr int kFinLanes = 32;
constexpr int kFinThreads = 256;
static_assert(kFinLanes * (kFinCols / 4) == kFinThreads, "one thread per (part lane, column group)");

struct FinalizeGrid {
  FinalizeList fl;
  int first[kMaxFinalizeJobs + 1];
};

__global__ void __launch_bounds__(kFinThreads) colsum_finalize_kernel(const __grid_constant__ FinalizeGrid fg) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ float4 red[kFinLanes][kFinCols / 4 + 1];
  int j = 0;
  while (j + 1 < fg.fl.n && (int)blockIdx.x >= fg.first[j + 1]) ++j;
  const FinalizeJob& job = fg.fl.job[j];
  const int b = (int)blockIdx.x - fg.first[j];
  const int cols = job.cols, nparts = job.nparts;
  if (job.stride) {
    const float4* p = reinterpret_cast<const float4*>(job.part);
    const size_t n4 = (size_t)cols / 4, st4 = job.stride / 4;
    const size_t step = (size_t)(fg.first[j + 1] - fg.first[j]) * kFinThreads;
    for (size_t i = (size_t)b * kFinThreads + threadIdx.x; i < n4; i += step) {
      float4 sum = p[i];
#pragma unroll 4
      for (int k = 1; k < nparts; ++k) {
        const float4 v = p[k * st4 + i];
        sum.x += v.x; sum.y += v.y; sum.z += v.z; sum.w += v.w;
      }
      reinterpret_cast<float4*>(job.out)[i] = sum;
    }
    return;
  }
  const int cg = threadIdx.x % (kFinCols / 4), pl = threadIdx.x / (kFinCols / 4);
  const int c = b * kFinCols + cg * 4;
  float4 s = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  if (c < cols) {
    const float* __restrict__ part = job.part + c;
    int p = pl;
    for (; p + 7 * kFinLanes < nparts; p += 8 * kFinLanes) {
      float4 v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = *reinterpret_cast<const float4*>(part + (size_t)(p + i * kFinLanes) * cols);
#pragma unroll
      for (int i = 0; i < 8; ++i) { s.x += v[i].x; s.y += v[i].y; s.z += v[i].z; s.w += v[i].w; }
    }
    for (; p < nparts; p += kFinLanes) {
      const float4 v = *reinterpret_cast<const float4*>(part + (size_t)p * cols);
      s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
    }
  }
  red[pl][cg] = s;
  __syncthreads();
  if (pl == 0 && c < cols) {
    float4 t = red[0][cg];
#pragma unroll
    for (int w = 1; w < kFinLanes; ++w) {
      const float4 v = red[w][cg];
      t.x += v.x; t.y += v.y; t.z += v.z; t.w += v.w;
    }
    *reinterpret_cast<float4*>(job.out + c) = t;
  }
}

// Scalar column sums for column counts that are not a multiple of 4: 32
// columns x 32 part lanes per block, blockIdx.y the job.
__global__ void __launch_bounds__(1024) colsum_finalize_scalar_kernel(FinalizeList fl) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ float red[32][33];
  const FinalizeJob& job = fl.job[blockIdx.y];
  const int cols = job.cols, nparts = job.nparts;
  if (blockIdx.x * 32 >= cols) return;
  const float* __restrict__ part = job.part;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int c = blockIdx.x * 32 + tx;
  float s = 0.0f;
  if (c < cols) {
#pragma unroll 8
    for (int p = ty; p < nparts; p += 32) s += part[(size_t)p * cols + c];
  }
  red[ty][tx] = s;
  __syncthreads();
  if (ty == 0 && c < cols) {
    float t = 0.0f;
#pragma unroll
    for (int w = 0; w < 32; ++w) t += red[w][tx];
    job.out[c] = t;
  }
}

template <typename T>
__global__ void gelu_kernel(const T* __restrict__ U, T* __restrict__ G, size_t n8, int tanh_form) {
  pdl_wait();
  pdl_launch_dependents();
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n8; i += (size_t)gridDim.x * blockDim.x) {
    float v[8];
    load8<T>(U + i * 8, v);
    gelu8_form(v, tanh_form != 0);
    store8<T>(G + i * 8, v);
  }
}

__global__ void dropout_mask_kernel(DropoutParams dp, int site, uint64_t e0, uint64_t n8, uint8_t* keep) {
  for (uint64_t i = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < n8; i += (uint64_t)gridDim.x * blockDim.x) {
    const uint32_t bits = dropout_bits8(dp, site, (e0 >> 3) + i);
#pragma unroll
    for (int k = 0; k < 8; ++k) keep[i * 8 + k] = (bits >> k) & 1u;
  }
}

// Blocks of the row kernels that keep per-block column sums: at least 16 rows
// a block, at most two blocks per SM, so a large batch fills every SM evenly
// (8192 rows: 296 blocks of <= 28 rows, not 256 blocks of 32 on 148 SMs).
int row_blocks(int rows) { return std::max(1, std::min(kMaxBlocks, (rows + 15) / 16)); }

#define TLP_KR_SWITCH(H, ES, ...)                             \
  switch (group_rows(H, ES)) {                                \
    case 4: { constexpr int KR = 4; __VA_ARGS__; } break;     \
    case 2: { constexpr int KR = 2; __VA_ARGS__; } break;     \
    default: { constexpr int KR = 1; __VA_ARGS__; } break;    \
  }

#define TLP_NCH_SWITCH(H, ...)                                                  \
  switch ((H + 255) / 256) {                                                   \
    case 1: { constexpr int NCH = 1; __VA_ARGS__; } break;                     \
    case 2: { constexpr int NCH = 2; __VA_ARGS__; } break;                     \
    case 3: { constexpr int NCH = 3; __VA_ARGS__; } break;                     \
    case 4: { constexpr int NCH = 4; __VA_ARGS__; } break;                     \
    case 5: case 6: { constexpr int NCH = 6; __VA_ARGS__; } break;             \
    case 7: case 8: { constexpr int NCH = 8; __VA_ARGS__; } break;             \
    case 9: case 10: case 11: case 12: { constexpr int NCH = 12; __VA_ARGS__; } break; \
    default: { constexpr int NCH = 16; __VA_ARGS__; } break;                   \
  }

template <typename T>
void ln_fwd_t(const void* x, const void* g, const void* b, void* y, float* mean, float* rstd, int rows, int H,
              float eps, cudaStream_t s, uint8_t* keep_out, const DropoutParams& dp, int site, const AttnKeepGen& ak) {
  TLP_NCH_SWITCH(H, {
    // one row per warp (two rows per warp, with both rows' loads issued
    // first, measured slower: 16.1 against 15.9 us for 8192 x 1024 fp16)
    constexpr int RPW = 1;
    const int blocks = (rows + kFwdWarps * RPW - 1) / (kFwdWarps * RPW);
    launch_pdl(ln_fwd_kernel<T, NCH, RPW>, blocks, kFwdWarps * 32, 0, s, static_cast<const T*>(x),
               static_cast<const T*>(g), static_cast<const T*>(b), static_cast<T*>(y), mean, rstd, rows, H, eps,
               keep_out, dp, site, ak);
  });
  count_launch();
}

template <typename T, bool INV, bool RES, bool DROP, int NC>
void ln_bwd_warp_launch(const LnBwdArgs& a, int parts, cudaStream_t s) {
  const size_t sm = ((size_t)kLnbPairs * a.H + kLnbPairs * 8) * sizeof(float);
  cudaFuncSetAttribute(ln_bwd_warp_kernel<T, INV, RES, DROP, NC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)sm);
  launch_pdl(ln_bwd_warp_kernel<T, INV, RES, DROP, NC>, parts, kLnbPairs * 64, sm, s, a);
}

template <typename T, bool INV, bool RES>
int ln_bwd_t(const LnBwdArgs& a, cudaStream_t s) {
  const int parts = ln_bwd_parts(a.rows);
  if (a.H <= 512) {
    a.drop_out ? ln_bwd_warp_launch<T, INV, RES, true, 1>(a, parts, s)
               : ln_bwd_warp_launch<T, INV, RES, false, 1>(a, parts, s);
  } else if (a.H <= 1024) {
    a.drop_out ? ln_bwd_warp_launch<T, INV, RES, true, 2>(a, parts, s)
               : ln_bwd_warp_launch<T, INV, RES, false, 2>(a, parts, s);
  } else {
    TLP_KR_SWITCH(a.H, (int)sizeof(T), {
      const size_t sm = pipe_smem<T, KR, RES ? 3 : 2>(a.H);
      cudaFuncSetAttribute(ln_bwd_kernel<T, INV, RES, KR>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
      launch_pdl(ln_bwd_kernel<T, INV, RES, KR>, parts, row_threads(a.H), sm, s, a);
    });
  }
  count_launch();
  return parts;
}

template <typename T>
void dropout_rows_t(const void* in, void* out, const DropoutParams& dp, int site, int rows, int H, float* part,
                    cudaStream_t s, const uint8_t* keep8, int padd) {
  TLP_KR_SWITCH(H, (int)sizeof(T), {
    const size_t sm = pipe_smem<T, KR, 1>(H);
    cudaFuncSetAttribute(dropout_rows_kernel<T, KR>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    launch_pdl(dropout_rows_kernel<T, KR>, rowdrop_parts(rows), row_threads(H), sm, s,
               static_cast<const T*>(in), static_cast<T*>(out), dp, site, rows, H, part, keep8, padd);
  });
  count_launch();
}

}  // namespace

// Hidden sizes served by the row kernels: multiples of 8 up to 4096 (one
// thread per 8 columns, at most 512 threads per block).
bool rowwise_supports_hidden(int H) { return H % 8 == 0 && H <= 4096; }

int ln_bwd_parts(int rows) { return row_blocks(rows); }
int rowdrop_parts(int rows) { return row_blocks(rows); }
int colsum_parts(int rows) { return std::max(1, std::min(kColParts, rows / 64)); }

void ln_fwd_run(int dt, const void* x, const void* g, const void* b, void* y, float* mean, float* rstd, int rows,
                int H, float eps, cudaStream_t s, uint8_t* keep_out, const DropoutParams* dp, int site,
                const AttnKeepGen* akeep) {
  DropoutParams d = {};
  if (keep_out && dp && dp->thr) d = *dp;
  else keep_out = nullptr;
  AttnKeepGen ak = {};
  if (akeep && akeep->keep && akeep->dp.thr) ak = *akeep;
  if (dt == DT_F32) ln_fwd_t<float>(x, g, b, y, mean, rstd, rows, H, eps, s, keep_out, d, site, ak);
  else if (dt == DT_F16) ln_fwd_t<half_t>(x, g, b, y, mean, rstd, rows, H, eps, s, keep_out, d, site, ak);
  else ln_fwd_t<bf16_t>(x, g, b, y, mean, rstd, rows, H, eps, s, keep_out, d, site, ak);
}

template <typename T>
int ln_bwd_dispatch(const LnBwdArgs& a, cudaStream_t s) {
  const bool inv = a.x == nullptr, res = a.res != nullptr;
  if (inv) return res ? ln_bwd_t<T, true, true>(a, s) : ln_bwd_t<T, true, false>(a, s);
  return res ? ln_bwd_t<T, false, true>(a, s) : ln_bwd_t<T, false, false>(a, s);
}

int ln_bwd_run(int dt, const LnBwdArgs& a, cudaStream_t s) {
  if (dt == DT_F32) return ln_bwd_dispatch<float>(a, s);
  if (dt == DT_F16) return ln_bwd_dispatch<half_t>(a, s);
  return ln_bwd_dispatch<bf16_t>(a, s);
}

void rowwise_set_wait_limit(uint64_t ns) { cudaMemcpyToSymbol(g_row_err, &ns, sizeof(ns), 2 * sizeof(int)); }

int rowwise_take_error() {
  int v = 0, z = 0;
  cudaMemcpyFromSymbol(&v, g_row_err, sizeof(int));
  if (v) cudaMemcpyToSymbol(g_row_err, &z, sizeof(int));
  return v;
}

template <typename T>
void dropout_rows_warp_t(const void* in, void* out, float scale, int rows, int H, float* part, cudaStream_t s,
                         const uint8_t* keep8, int padd) {
  const size_t sm = (size_t)kDropWarps * H * sizeof(float);
  TLP_NCH_SWITCH(H, {
    if constexpr (NCH <= 4) {
      cudaFuncSetAttribute(dropout_rows_warp_kernel<T, NCH>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
      launch_pdl(dropout_rows_warp_kernel<T, NCH>, rowdrop_parts(rows), kDropWarps * 32, sm, s,
                 static_cast<const T*>(in), static_cast<T*>(out), scale, rows, H, part, keep8, padd);
    }
  });
  count_launch();
}

void dropout_rows_run(int dt, const void* in, void* out, const DropoutParams& dp, int site, int rows, int H,
                      float* part, cudaStream_t s, const uint8_t* keep8, int acc) {
  const int padd = acc ? 1 : 0;
  if (keep8 && dp.thr && H <= 1024) {
    // keep bits at hand: the warp-per-row form (no Philox, no shared-memory pipeline)
    if (dt == DT_F32) dropout_rows_warp_t<float>(in, out, dp.scale, rows, H, part, s, keep8, padd);
    else if (dt == DT_F16) dropout_rows_warp_t<half_t>(in, out, dp.scale, rows, H, part, s, keep8, padd);
    else dropout_rows_warp_t<bf16_t>(in, out, dp.scale, rows, H, part, s, keep8, padd);
    return;
  }
  if (dt == DT_F32) dropout_rows_t<float>(in, out, dp, site, rows, H, part, s, keep8, padd);
  else if (dt == DT_F16) dropout_rows_t<half_t>(in, out, dp, site, rows, H, part, s, keep8, padd);
  else dropout_rows_t<bf16_t>(in, out, dp, site, rows, H, part, s, keep8, padd);
}

void colsum_run(int dt, const void* X, int rows, int cols, float* part, cudaStream_t s, int acc) {
  dim3 grid((cols + 255) / 256, colsum_parts(rows));
  const int padd = acc ? 1 : 0;
  if (dt == DT_F32)
    launch_pdl(colsum_kernel<float>, grid, 256, 0, s, static_cast<const float*>(X), rows, cols, part, padd);
  else if (dt == DT_F16)
    launch_pdl(colsum_kernel<half_t>, grid, 256, 0, s, static_cast<const half_t*>(X), rows, cols, part, padd);
  else launch_pdl(colsum_kernel<bf16_t>, grid, 256, 0, s, static_cast<const bf16_t*>(X), rows, cols, part, padd);
  count_launch();
}

namespace {

// Zeroes each listed buffer: 16-byte stores where the buffer is 16-byte
// aligned, one float at a time for the rest.
__global__ void __launch_bounds__(256) zero_list_kernel(ZeroList z) {
  pdl_wait();
  pdl_launch_dependents();
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  const size_t tid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  for (int j = 0; j < z.count; ++j) {
    float* p = z.p[j];
    const size_t n = z.n[j];
    size_t head = 0;
    if ((reinterpret_cast<uintptr_t>(p) & 15) == 0) {
      const size_t n4 = n / 4;
      float4* p4 = reinterpret_cast<float4*>(p);
      for (size_t i = tid; i < n4; i += stride) p4[i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      head = n4 * 4;
    }
    for (size_t i = head + tid; i < n; i += stride) p[i] = 0.0f;
  }
}

}  // namespace

void zero_list_run(const ZeroList& z, cudaStream_t s) {
  if (z.count <= 0) return;
  size_t total4 = 0;
  for (int j = 0; j < z.count; ++j) total4 += (z.n[j] + 3) / 4;
  const int blocks = (int)std::max<size_t>(1, std::min<size_t>((total4 + 255) / 256, 148 * 4));
  launch_pdl(zero_list_kernel, blocks, 256, 0, s, z);
  count_launch();
}

void colsum_finalize_list_run(const FinalizeList& fl, cudaStream_t s) {
  if (fl.n <= 0) return;
  bool vec = true;
  for (int i = 0; i < fl.n; ++i) {
    const FinalizeJob& j = fl.job[i];
    if (!j.stride && (j.cols % 4 != 0 || (reinterpret_cast<uintptr_t>(j.part) & 15) != 0 ||
                      (reinterpret_cast<uintptr_t>(j.out) & 15) != 0))
      vec = false;
  }
  if (!vec) {
    // scalar column sums; split-K jobs (always 4-aligned) then go one by one
    FinalizeList cs = fl;
    cs.n = 0;
    int maxc = 0;
    for (int i = 0; i < fl.n; ++i)
      if (!fl.job[i].stride) {
        cs.job[cs.n++] = fl.job[i];
        maxc = std::max(maxc, fl.job[i].cols);
      }
    if (cs.n) {
      launch_pdl(colsum_finalize_scalar_kernel, dim3((maxc + 31) / 32, cs.n), 1024, 0, s, cs);
      count_launch();
    }
    for (int i = 0; i < fl.n; ++i)
      if (fl.job[i].stride) {
        FinalizeList one;
        one.n = 1;
        one.job[0] = fl.job[i];
        colsum_finalize_list_run(one, s);
      }
    return;
  }
  FinalizeGrid fg;
  fg.fl = fl;
  fg.first[0] = 0;
  for (int i = 0; i < fl.n; ++i) {
    const FinalizeJob& j = fl.job[i];
    // split-K sums: up to four blocks per SM, so a thread's partial loads
    // come in about one round (the column-sum jobs fill the rest of the wave)
    const int nb = j.stride ? (int)std::min<size_t>(((size_t)j.cols / 4 + kFinThreads - 1) / kFinThreads, 592)
                            : (j.cols + kFinCols - 1) / kFinCols;
    fg.first[i + 1] = fg.first[i] + std::max(nb, 1);
  }
  launch_pdl(colsum_finalize_kernel, fg.first[fl.n], kFinThreads, 0, s, fg);
  count_launch();
}

void colsum_finalize_run(const float* part, int nparts, int cols, float* out, cudaStream_t s) {
  FinalizeList fl;
  fl.n = 1;
  fl.job[0] = {part, out, nparts, cols};
  colsum_finalize_list_run(fl, s);
}

void colsum_finalize3_run(const float* p0, const float* p1, const float* p2, float* o0, float* o1, float* o2,
                          int nparts, int cols, cudaStream_t s) {
  FinalizeList fl;
  fl.n = 0;
  fl.job[fl.n++] = {p0, o0, nparts, cols};
  if (p1) fl.job[fl.n++] = {p1, o1, nparts, cols};
  if (p2) fl.job[fl.n++] = {p2, o2, nparts, cols};
  colsum_finalize_list_run(fl, s);
}

__global__ void gelu_eval_kernel(const float* __restrict__ u, float* __restrict__ g, float* __restrict__ dg,
                                 uint64_t n, int tanh_form) {
  for (uint64_t i = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < n; i += (uint64_t)gridDim.x * blockDim.x) {
    const float2 v = make_float2(u[i], 0.0f);
    g[i] = tanh_form ? gelu_tanh2(v).x : gelu2(v).x;
    dg[i] = tanh_form ? gelu_tanh_grad2(v).x : gelu_grad2(v).x;
  }
}

void gelu_eval_run(const float* u, float* g, float* dg, uint64_t n, int tanh_form, cudaStream_t s) {
  const int blocks = (int)std::min<uint64_t>((n + 255) / 256, 148 * 16);
  gelu_eval_kernel<<<blocks > 0 ? blocks : 1, 256, 0, s>>>(u, g, dg, n, tanh_form);
  count_launch();
}

void gelu_run(int dt, const void* U, void* G, size_t n, int tanh_form, cudaStream_t s) {
  const size_t n8 = n / 8;
  const int blocks = (int)std::min<size_t>((n8 + 255) / 256, 148 * 16);
  if (dt == DT_F32)
    launch_pdl(gelu_kernel<float>, blocks, 256, 0, s, static_cast<const float*>(U), static_cast<float*>(G), n8, tanh_form);
  else if (dt == DT_F16)
    launch_pdl(gelu_kernel<half_t>, blocks, 256, 0, s, static_cast<const half_t*>(U), static_cast<half_t*>(G), n8, tanh_form);
  else
    launch_pdl(gelu_kernel<bf16_t>, blocks, 256, 0, s, static_cast<const bf16_t*>(U), static_cast<bf16_t*>(G), n8, tanh_form);
  count_launch();
}

void dropout_mask_run(const DropoutParams& dp, int site, uint64_t e0, uint64_t n, uint8_t* keep, cudaStream_t s) {
  const uint64_t n8 = n / 8;
  const int blocks = (int)std::min<uint64_t>((n8 + 255) / 256, 148 * 16);
  dropout_mask_kernel<<<blocks > 0 ? blocks : 1, 256, 0, s>>>(dp, site, e0, n8, keep);
  count_launch();
}

}  // namespace tlp
