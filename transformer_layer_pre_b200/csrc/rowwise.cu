// rowwise.cu — bandwidth-bound kernels over (rows, H) activations:
// LayerNorm forward/backward, dropout backward, column sums, GELU, mask dump.
//
// LayerNorm is per token over the hidden axis with the biased variance and
// eps inside the square root; statistics are float32 ("AI-infra engineers and
// the Transformer", section 3.2: LayerNorm kept in fp32).  A block owns a
// contiguous range of rows and each thread 8 consecutive columns of them, so
// column sums (bias and LayerNorm-parameter gradients) accumulate in the
// owning thread's registers in row order and leave as one partial row per
// block, summed by tlp::colsum_finalize_run in block order: deterministic.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "profile.h"

namespace tlp {

namespace {

// Row-block kernels: a block of ceil(H/8 / 32) warps owns a contiguous range
// of rows; thread t owns columns 8t .. 8t+7 of every row of that range (one
// 16-byte vector for 16-bit storage) and walks the rows kRows at a time.
// Row statistics are block reductions (one per kRows rows); column sums stay
// in the owning thread's registers and leave as one partial row per block.
constexpr int kRows = 4;
constexpr int kMaxBlocks = 592;   // 4 blocks per SM

__host__ __device__ inline int row_threads(int H) { return ((H / 8 + 31) / 32) * 32; }

// Sums v[r] over the whole block; red holds (warps, kRows) floats.
__device__ __forceinline__ void block_sum(float (&v)[kRows], float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int r = 0; r < kRows; ++r) v[r] = warp_sum(v[r]);
  if (lane == 0) {
#pragma unroll
    for (int r = 0; r < kRows; ++r) red[warp * kRows + r] = v[r];
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < kRows; ++r) {
    float s = 0.0f;
    for (int w = 0; w < nw; ++w) s += red[w * kRows + r];
    v[r] = s;
  }
  __syncthreads();
}

__device__ __forceinline__ void row_range(int rows, int& r0, int& r1) {
  const int per = (rows + gridDim.x - 1) / gridDim.x;
  r0 = blockIdx.x * per;
  r1 = min(rows, r0 + per);
}

__device__ __forceinline__ void store_part(float* part, int H, int col, const float (&acc)[8]) {
  float* p = part + (size_t)blockIdx.x * H + col;
  reinterpret_cast<float4*>(p)[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
}

// ------------------------------------------------------------------ LayerNorm forward
template <typename T>
__global__ void __launch_bounds__(512) ln_fwd_kernel(const T* __restrict__ x, const T* __restrict__ gamma,
                                                    const T* __restrict__ beta, T* __restrict__ y,
                                                    float* __restrict__ mean_out, float* __restrict__ rstd_out,
                                                    int rows, int H, float eps) {
  __shared__ float red[16 * kRows];
  const int col = threadIdx.x * 8;
  const bool act = col < H;
  float g[8], b[8];
  if (act) {
    load8<T>(gamma + col, g);
    load8<T>(beta + col, b);
  }
  int r0, r1;
  row_range(rows, r0, r1);
  const float inv_h = 1.0f / (float)H;
  for (int base = r0; base < r1; base += kRows) {
    float v[kRows][8], s[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      s[r] = 0.0f;
      if (act && base + r < r1) {
        load8<T>(x + (size_t)(base + r) * H + col, v[r]);
#pragma unroll
        for (int i = 0; i < 8; ++i) s[r] += v[r][i];
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[r][i] = 0.0f;
      }
    }
    block_sum(s, red);
    float mean[kRows], ss[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      mean[r] = s[r] * inv_h;
      ss[r] = 0.0f;
      if (act) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float d = v[r][i] - mean[r];
          ss[r] += d * d;
        }
      }
    }
    block_sum(ss, red);
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      if (base + r >= r1) continue;
      const float rstd = 1.0f / sqrtf(ss[r] * inv_h + eps);
      if (act) {
        float o[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] = g[i] * ((v[r][i] - mean[r]) * rstd) + b[i];
        store8<T>(y + (size_t)(base + r) * H + col, o);
      }
      if (threadIdx.x == 0) {
        mean_out[base + r] = mean[r];
        rstd_out[base + r] = rstd;
      }
    }
  }
}

// ------------------------------------------------------------------ LayerNorm backward
template <typename T, bool INV>
__global__ void __launch_bounds__(512) ln_bwd_kernel(LnBwdArgs a) {
  __shared__ float red[16 * kRows];
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
  const T* dyp = static_cast<const T*>(a.dy);
  const float inv_h = 1.0f / (float)H;
  const float sc = a.drop.thr ? a.drop.scale : 1.0f;
  int r0, r1;
  row_range(a.rows, r0, r1);
  for (int base = r0; base < r1; base += kRows) {
    float g[kRows][8], xh[kRows][8], s1[kRows], s2[kRows], rs[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      s1[r] = s2[r] = 0.0f;
      const int row = base + r;
      rs[r] = row < r1 ? a.rstd[row] : 0.0f;
      if (act && row < r1) {
        const size_t off = (size_t)row * H + col;
        float dy[8], xv[8];
        load8<T>(dyp + off, dy);
        if constexpr (INV) {
          load8<T>(static_cast<const T*>(a.y) + off, xv);
#pragma unroll
          for (int i = 0; i < 8; ++i) xh[r][i] = (xv[i] - bt[i]) / gm[i];
        } else {
          load8<T>(static_cast<const T*>(a.x) + off, xv);
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
    block_sum(s1, red);
    block_sum(s2, red);
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      const int row = base + r;
      if (!act || row >= r1) continue;
      const size_t off = (size_t)row * H + col;
      const float m1 = s1[r] * inv_h, m2 = s2[r] * inv_h;
      float o[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = rs[r] * (g[r][i] - m1 - xh[r][i] * m2);
      if (a.res) {
        float rv[8];
        load8<T>(static_cast<const T*>(a.res) + off, rv);
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] += rv[i];
      }
      store8<T>(static_cast<T*>(a.dx) + off, o);
      if (a.drop_out) {
        const uint32_t bits = a.drop.thr ? dropout_bits8(a.drop, a.site, off >> 3) : 0xFFu;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          o[i] = round_f<T>(((bits >> i) & 1u) ? round_f<T>(o[i]) * sc : 0.0f);
          ds[i] += o[i];
        }
        store8<T>(static_cast<T*>(a.drop_out) + off, o);
      }
    }
  }
  if (act) {
    store_part(a.part_dgamma, H, col, dg);
    store_part(a.part_dbeta, H, col, db);
    if (a.part_dsum) store_part(a.part_dsum, H, col, ds);
  }
}

// ------------------------------------------------------------------ dropout of rows
template <typename T>
__global__ void __launch_bounds__(512) dropout_rows_kernel(const T* __restrict__ in, T* __restrict__ out,
                                                            DropoutParams dp, int site, int rows, int H,
                                                            float* __restrict__ part) {
  const int col = threadIdx.x * 8;
  if (col >= H) return;
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  const float sc = dp.thr ? dp.scale : 1.0f;
  int r0, r1;
  row_range(rows, r0, r1);
  for (int row = r0; row < r1; ++row) {
    const size_t off = (size_t)row * H + col;
    float v[8];
    load8<T>(in + off, v);
    const uint32_t bits = dp.thr ? dropout_bits8(dp, site, off >> 3) : 0xFFu;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[i] = round_f<T>(((bits >> i) & 1u) ? v[i] * sc : 0.0f);
      acc[i] += v[i];
    }
    store8<T>(out + off, v);
  }
  store_part(part, H, col, acc);
}

// ------------------------------------------------------------------ column sums
constexpr int kColParts = 64;

template <typename T>
__global__ void __launch_bounds__(256) colsum_kernel(const T* __restrict__ X, int rows, int cols,
                                                     float* __restrict__ part) {
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
    part[(size_t)blockIdx.y * cols + c] = s;
  }
}

// out[c] = sum over p of part[p][c]: 32 columns x 32 part-lanes per block,
// each lane sums every 32nd partial row, then a fixed-order sum over lanes.
__global__ void __launch_bounds__(1024) colsum_finalize_kernel(const float* __restrict__ part, int nparts, int cols,
                                                             float* __restrict__ out) {
  __shared__ float red[32][33];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int c = blockIdx.x * 32 + tx;
  float s = 0.0f;
  if (c < cols) {
#pragma unroll 4
    for (int p = ty; p < nparts; p += 32) s += part[(size_t)p * cols + c];
  }
  red[ty][tx] = s;
  __syncthreads();
  if (ty == 0 && c < cols) {
    float t = 0.0f;
#pragma unroll
    for (int w = 0; w < 32; ++w) t += red[w][tx];
    out[c] = t;
  }
}

template <typename T>
__global__ void gelu_kernel(const T* __restrict__ U, T* __restrict__ G, size_t n8) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n8; i += (size_t)gridDim.x * blockDim.x) {
    float v[8];
    load8<T>(U + i * 8, v);
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = gelu_f(v[k]);
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

int row_blocks(int rows) { return std::max(1, std::min(kMaxBlocks, (rows + 4 * kRows - 1) / (4 * kRows))); }

template <typename T>
void ln_fwd_t(const void* x, const void* g, const void* b, void* y, float* mean, float* rstd, int rows, int H,
              float eps, cudaStream_t s) {
  // one group of kRows rows per block: no column sums, so maximal parallelism
  ln_fwd_kernel<T><<<(rows + kRows - 1) / kRows, row_threads(H), 0, s>>>(static_cast<const T*>(x), static_cast<const T*>(g),
                                                              static_cast<const T*>(b), static_cast<T*>(y), mean,
                                                              rstd, rows, H, eps);
  count_launch();
}

template <typename T, bool INV>
void ln_bwd_t(const LnBwdArgs& a, cudaStream_t s) {
  ln_bwd_kernel<T, INV><<<ln_bwd_parts(a.rows), row_threads(a.H), 0, s>>>(a);
  count_launch();
}

template <typename T>
void dropout_rows_t(const void* in, void* out, const DropoutParams& dp, int site, int rows, int H, float* part,
                    cudaStream_t s) {
  dropout_rows_kernel<T><<<rowdrop_parts(rows), row_threads(H), 0, s>>>(static_cast<const T*>(in),
                                                                       static_cast<T*>(out), dp, site, rows, H, part);
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
                int H, float eps, cudaStream_t s) {
  if (dt == DT_F32) ln_fwd_t<float>(x, g, b, y, mean, rstd, rows, H, eps, s);
  else if (dt == DT_F16) ln_fwd_t<half_t>(x, g, b, y, mean, rstd, rows, H, eps, s);
  else ln_fwd_t<bf16_t>(x, g, b, y, mean, rstd, rows, H, eps, s);
}

void ln_bwd_run(int dt, const LnBwdArgs& a, cudaStream_t s) {
  const bool inv = a.x == nullptr;
  if (dt == DT_F32) inv ? ln_bwd_t<float, true>(a, s) : ln_bwd_t<float, false>(a, s);
  else if (dt == DT_F16) inv ? ln_bwd_t<half_t, true>(a, s) : ln_bwd_t<half_t, false>(a, s);
  else inv ? ln_bwd_t<bf16_t, true>(a, s) : ln_bwd_t<bf16_t, false>(a, s);
}

void dropout_rows_run(int dt, const void* in, void* out, const DropoutParams& dp, int site, int rows, int H,
                      float* part, cudaStream_t s) {
  if (dt == DT_F32) dropout_rows_t<float>(in, out, dp, site, rows, H, part, s);
  else if (dt == DT_F16) dropout_rows_t<half_t>(in, out, dp, site, rows, H, part, s);
  else dropout_rows_t<bf16_t>(in, out, dp, site, rows, H, part, s);
}

void colsum_run(int dt, const void* X, int rows, int cols, float* part, cudaStream_t s) {
  dim3 grid((cols + 255) / 256, colsum_parts(rows));
  if (dt == DT_F32) colsum_kernel<float><<<grid, 256, 0, s>>>(static_cast<const float*>(X), rows, cols, part);
  else if (dt == DT_F16) colsum_kernel<half_t><<<grid, 256, 0, s>>>(static_cast<const half_t*>(X), rows, cols, part);
  else colsum_kernel<bf16_t><<<grid, 256, 0, s>>>(static_cast<const bf16_t*>(X), rows, cols, part);
  count_launch();
}

void colsum_finalize_run(const float* part, int nparts, int cols, float* out, cudaStream_t s) {
  colsum_finalize_kernel<<<(cols + 31) / 32, 1024, 0, s>>>(part, nparts, cols, out);
  count_launch();
}

void gelu_run(int dt, const void* U, void* G, size_t n, cudaStream_t s) {
  const size_t n8 = n / 8;
  const int blocks = (int)std::min<size_t>((n8 + 255) / 256, 148 * 16);
  if (dt == DT_F32) gelu_kernel<float><<<blocks, 256, 0, s>>>(static_cast<const float*>(U), static_cast<float*>(G), n8);
  else if (dt == DT_F16) gelu_kernel<half_t><<<blocks, 256, 0, s>>>(static_cast<const half_t*>(U), static_cast<half_t*>(G), n8);
  else gelu_kernel<bf16_t><<<blocks, 256, 0, s>>>(static_cast<const bf16_t*>(U), static_cast<bf16_t*>(G), n8);
  count_launch();
}

void dropout_mask_run(const DropoutParams& dp, int site, uint64_t e0, uint64_t n, uint8_t* keep, cudaStream_t s) {
  const uint64_t n8 = n / 8;
  const int blocks = (int)std::min<uint64_t>((n8 + 255) / 256, 148 * 16);
  dropout_mask_kernel<<<blocks > 0 ? blocks : 1, 256, 0, s>>>(dp, site, e0, n8, keep);
  count_launch();
}

}  // namespace tlp
