// rowwise.cu — bandwidth-bound kernels over (rows, H) activations:
// LayerNorm forward/backward, dropout backward, column sums, GELU, mask dump.
//
// LayerNorm is per token over the hidden axis with the biased variance and
// eps inside the square root; statistics are float32 ("AI-infra engineers and
// the Transformer", section 3.2: LayerNorm kept in fp32).  One warp owns a
// row; each lane holds chunks of 8 consecutive elements (one 16-byte load for
// 16-bit storage), so a warp reads 512 contiguous bytes per chunk step.
// Column sums (bias and LayerNorm-parameter gradients) are reduced in a fixed
// order: per-warp registers, then per-block shared memory, then one partial
// row per block, then tlp::colsum_finalize_run — the result is deterministic.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "profile.h"

namespace tlp {

namespace {

constexpr int kWarps = 8;  // warps per block of the row kernels
constexpr int kMaxParts = 296;

// ------------------------------------------------------------------ LayerNorm forward
template <typename T, int NCH>
__global__ void __launch_bounds__(kWarps * 32) ln_fwd_kernel(const T* __restrict__ x, const T* __restrict__ gamma,
                                                            const T* __restrict__ beta, T* __restrict__ y,
                                                            float* __restrict__ mean_out, float* __restrict__ rstd_out,
                                                            int rows, int H, float eps) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (row >= rows) return;
  const T* xr = x + (size_t)row * H;
  float v[NCH][8];
  float s = 0.0f;
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    const int col = (lane + 32 * c) * 8;
    if (col < H) {
      load8<T>(xr + col, v[c]);
#pragma unroll
      for (int i = 0; i < 8; ++i) s += v[c][i];
    }
  }
  const float mean = warp_sum(s) / (float)H;
  float ss = 0.0f;
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    const int col = (lane + 32 * c) * 8;
    if (col < H) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float dlt = v[c][i] - mean;
        ss += dlt * dlt;
      }
    }
  }
  const float var = warp_sum(ss) / (float)H;
  const float rstd = 1.0f / sqrtf(var + eps);
  T* yr = y + (size_t)row * H;
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    const int col = (lane + 32 * c) * 8;
    if (col < H) {
      float g[8], b[8], o[8];
      load8<T>(gamma + col, g);
      load8<T>(beta + col, b);
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = g[i] * ((v[c][i] - mean) * rstd) + b[i];
      store8<T>(yr + col, o);
    }
  }
  if (lane == 0) {
    mean_out[row] = mean;
    rstd_out[row] = rstd;
  }
}

// Reduce per-lane column accumulators acc[NCH][8] of every warp of the block
// into one partial row part[blockIdx.x * H + col]; red is (kWarps, H) floats.
template <int NCH>
__device__ __forceinline__ void block_colsum(float (&acc)[NCH][8], float* red, float* part, int H) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    const int col = (lane + 32 * c) * 8;
    if (col < H) {
#pragma unroll
      for (int i = 0; i < 8; ++i) red[warp * H + col + i] = acc[c][i];
    }
  }
  __syncthreads();
  for (int col = threadIdx.x; col < H; col += blockDim.x) {
    float s = 0.0f;
    for (int w = 0; w < kWarps; ++w) s += red[w * H + col];
    part[(size_t)blockIdx.x * H + col] = s;
  }
}

// ------------------------------------------------------------------ LayerNorm backward
template <typename T, int NCH, bool INV>
__global__ void __launch_bounds__(kWarps * 32) ln_bwd_kernel(LnBwdArgs a) {
  extern __shared__ float red[];
  const int lane = threadIdx.x & 31;
  const int H = a.H;
  const int nwarps = gridDim.x * kWarps;
  float dg[NCH][8], db[NCH][8], dsum[NCH][8];
#pragma unroll
  for (int c = 0; c < NCH; ++c)
#pragma unroll
    for (int i = 0; i < 8; ++i) dg[c][i] = db[c][i] = dsum[c][i] = 0.0f;

  const T* dyp = static_cast<const T*>(a.dy);
  const T* gam = static_cast<const T*>(a.gamma);
  for (int row = blockIdx.x * kWarps + (threadIdx.x >> 5); row < a.rows; row += nwarps) {
    const size_t off = (size_t)row * H;
    const float rstd = a.rstd[row];
    float dy[NCH][8], xh[NCH][8];
    float s1 = 0.0f, s2 = 0.0f;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      const int col = (lane + 32 * c) * 8;
      if (col < H) {
        float g[8];
        load8<T>(dyp + off + col, dy[c]);
        load8<T>(gam + col, g);
        if constexpr (INV) {
          float yv[8], bt[8];
          load8<T>(static_cast<const T*>(a.y) + off + col, yv);
          load8<T>(static_cast<const T*>(a.beta) + col, bt);
#pragma unroll
          for (int i = 0; i < 8; ++i) xh[c][i] = (yv[i] - bt[i]) / g[i];
        } else {
          float xv[8];
          load8<T>(static_cast<const T*>(a.x) + off + col, xv);
          const float mean = a.mean[row];
#pragma unroll
          for (int i = 0; i < 8; ++i) xh[c][i] = (xv[i] - mean) * rstd;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float gi = dy[c][i] * g[i];
          s1 += gi;
          s2 += gi * xh[c][i];
          dg[c][i] += dy[c][i] * xh[c][i];
          db[c][i] += dy[c][i];
          dy[c][i] = gi;  // keep g = dy * gamma
        }
      }
    }
    const float m1 = warp_sum(s1) / (float)H;
    const float m2 = warp_sum(s2) / (float)H;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      const int col = (lane + 32 * c) * 8;
      if (col < H) {
        float o[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] = rstd * (dy[c][i] - m1 - xh[c][i] * m2);
        if (a.res) {
          float r[8];
          load8<T>(static_cast<const T*>(a.res) + off + col, r);
#pragma unroll
          for (int i = 0; i < 8; ++i) o[i] += r[i];
        }
        store8<T>(static_cast<T*>(a.dx) + off + col, o);
        if (a.drop_out) {
          uint32_t bits = 0xFFu;
          if (a.drop.thr) bits = dropout_bits8(a.drop, a.site, (off + col) >> 3);
          const float sc = a.drop.thr ? a.drop.scale : 1.0f;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            o[i] = ((bits >> i) & 1u) ? round_f<T>(o[i]) * sc : 0.0f;
            o[i] = round_f<T>(o[i]);
            dsum[c][i] += o[i];
          }
          store8<T>(static_cast<T*>(a.drop_out) + off + col, o);
        }
      }
    }
  }
  block_colsum<NCH>(dg, red, a.part_dgamma, H);
  block_colsum<NCH>(db, red, a.part_dbeta, H);
  if (a.part_dsum) block_colsum<NCH>(dsum, red, a.part_dsum, H);
}

// ------------------------------------------------------------------ dropout of rows
template <typename T, int NCH>
__global__ void __launch_bounds__(kWarps * 32) dropout_rows_kernel(const T* __restrict__ in, T* __restrict__ out,
                                                                  DropoutParams dp, int site, int rows, int H,
                                                                  float* __restrict__ part) {
  extern __shared__ float red[];
  const int lane = threadIdx.x & 31;
  const int nwarps = gridDim.x * kWarps;
  float acc[NCH][8];
#pragma unroll
  for (int c = 0; c < NCH; ++c)
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[c][i] = 0.0f;
  for (int row = blockIdx.x * kWarps + (threadIdx.x >> 5); row < rows; row += nwarps) {
    const size_t off = (size_t)row * H;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      const int col = (lane + 32 * c) * 8;
      if (col < H) {
        float v[8];
        load8<T>(in + off + col, v);
        uint32_t bits = 0xFFu;
        if (dp.thr) bits = dropout_bits8(dp, site, (off + col) >> 3);
        const float sc = dp.thr ? dp.scale : 1.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          v[i] = round_f<T>(((bits >> i) & 1u) ? v[i] * sc : 0.0f);
          acc[c][i] += v[i];
        }
        store8<T>(out + off + col, v);
      }
    }
  }
  block_colsum<NCH>(acc, red, part, H);
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

__global__ void colsum_finalize_kernel(const float* __restrict__ part, int nparts, int cols, float* __restrict__ out) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= cols) return;
  float s = 0.0f;
  for (int p = 0; p < nparts; ++p) s += part[(size_t)p * cols + c];
  out[c] = s;
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

int nch_of(int H) { return (H + 255) / 256; }

#define TLP_NCH_SWITCH(H, ...)                        \
  switch (nch_of(H)) {                                \
    case 1: { constexpr int NCH = 1; __VA_ARGS__; } break; \
    case 2: { constexpr int NCH = 2; __VA_ARGS__; } break; \
    case 3: { constexpr int NCH = 3; __VA_ARGS__; } break; \
    case 4: { constexpr int NCH = 4; __VA_ARGS__; } break; \
    case 5: { constexpr int NCH = 5; __VA_ARGS__; } break; \
    case 6: { constexpr int NCH = 6; __VA_ARGS__; } break; \
    case 7: { constexpr int NCH = 7; __VA_ARGS__; } break; \
    case 8: { constexpr int NCH = 8; __VA_ARGS__; } break; \
    case 12: { constexpr int NCH = 12; __VA_ARGS__; } break; \
    case 16: { constexpr int NCH = 16; __VA_ARGS__; } break; \
    default: break;                                   \
  }

template <typename T>
void ln_fwd_t(const void* x, const void* g, const void* b, void* y, float* mean, float* rstd, int rows, int H,
              float eps, cudaStream_t s) {
  const int blocks = (rows + kWarps - 1) / kWarps;
  TLP_NCH_SWITCH(H, ln_fwd_kernel<T, NCH><<<blocks, kWarps * 32, 0, s>>>(
                        static_cast<const T*>(x), static_cast<const T*>(g), static_cast<const T*>(b),
                        static_cast<T*>(y), mean, rstd, rows, H, eps));
  count_launch();
}

template <typename T, bool INV>
void ln_bwd_t(const LnBwdArgs& a, cudaStream_t s) {
  const int blocks = ln_bwd_parts(a.rows);
  const size_t smem = (size_t)kWarps * a.H * sizeof(float);
  TLP_NCH_SWITCH(a.H, {
    cudaFuncSetAttribute(ln_bwd_kernel<T, NCH, INV>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    ln_bwd_kernel<T, NCH, INV><<<blocks, kWarps * 32, smem, s>>>(a);
  });
  count_launch();
}

template <typename T>
void dropout_rows_t(const void* in, void* out, const DropoutParams& dp, int site, int rows, int H, float* part,
                    cudaStream_t s) {
  const int blocks = rowdrop_parts(rows);
  const size_t smem = (size_t)kWarps * H * sizeof(float);
  TLP_NCH_SWITCH(H, {
    cudaFuncSetAttribute(dropout_rows_kernel<T, NCH>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    dropout_rows_kernel<T, NCH><<<blocks, kWarps * 32, smem, s>>>(static_cast<const T*>(in), static_cast<T*>(out),
                                                                  dp, site, rows, H, part);
  });
  count_launch();
}

}  // namespace

// Hidden sizes served by the row kernels: multiples of 8 up to 4096 whose
// 256-column chunk count has an instantiation above.
bool rowwise_supports_hidden(int H) {
  const int n = nch_of(H);
  return H % 8 == 0 && H <= 4096 && (n <= 8 || n == 12 || n == 16);
}

int ln_bwd_parts(int rows) { return std::max(1, std::min(kMaxParts, (rows + kWarps - 1) / kWarps)); }
int rowdrop_parts(int rows) { return ln_bwd_parts(rows); }
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
  colsum_finalize_kernel<<<(cols + 255) / 256, 256, 0, s>>>(part, nparts, cols, out);
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
