// attn_simt.cu — exact-float32 SIMT attention, forward and backward.
//
// Scaled dot-product attention of every (sequence, head): scores
// S = Q K^T * (1/sqrt(d)) + mask (additive over keys), P = softmax over keys,
// dropout on P (site 0), ctx = P_dropped V ("Transformer deployment",
// section 1 pseudo-code: scale after Q K^T, softmax on the last axis; the
// dropout site is the probabilities, "DeepSpeed Transformer Kernel usage
// guide", Step 3: attention dropout is recomputed from the softmax output).
//
// One thread owns one query row (forward, dQ) or one key column (dK, dV);
// scores are never stored: the forward keeps the log-sum-exp per row and the
// backward regenerates P and the dropout bits from it.  This path serves the
// float32 storage type, whose 1e-5 parity bar needs IEEE float32 products.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "profile.h"

namespace tlp {

namespace {

constexpr int kRows = 64;  // rows (threads) per block
constexpr int kTile = 32;  // keys or queries staged per shared-memory tile

template <typename T, int D>
__global__ void __launch_bounds__(kRows) attn_fwd_simt(AttnArgs a) {
  __shared__ float Ks[kTile][D];
  __shared__ float Vs[kTile][D];
  const int S = a.S, H = a.nh * D;
  const int b = blockIdx.z, h = blockIdx.y;
  const int i = blockIdx.x * kRows + threadIdx.x;
  const size_t head = ((size_t)b * a.nh + h) * S;
  const T* Q = static_cast<const T*>(a.q);
  const T* K = static_cast<const T*>(a.k);
  const T* V = static_cast<const T*>(a.v);
  float q[D], o[D];
#pragma unroll
  for (int c = 0; c < D; ++c) {
    q[c] = i < S ? to_f(Q[(head + i) * D + c]) : 0.0f;
    o[c] = 0.0f;
  }
  float m = -INFINITY, l = 0.0f;
  for (int j0 = 0; j0 < S; j0 += kTile) {
    for (int idx = threadIdx.x; idx < kTile * D; idx += kRows) {
      const int jj = idx / D, c = idx % D, j = j0 + jj;
      Ks[jj][c] = j < S ? to_f(K[(head + j) * D + c]) : 0.0f;
      Vs[jj][c] = j < S ? to_f(V[(head + j) * D + c]) : 0.0f;
    }
    __syncthreads();
    if (i < S) {
      float sc[kTile];
      float tmax = -INFINITY;
#pragma unroll
      for (int jj = 0; jj < kTile; ++jj) {
        const int j = j0 + jj;
        float s = -INFINITY;
        if (j < S) {
          float dot = 0.0f;
#pragma unroll
          for (int c = 0; c < D; ++c) dot = fmaf(q[c], Ks[jj][c], dot);
          s = dot * a.scale + (a.mask ? a.mask[(size_t)b * S + j] : 0.0f);
        }
        sc[jj] = s;
        tmax = fmaxf(tmax, s);
      }
      const float mnew = fmaxf(m, tmax);
      if (mnew != -INFINITY) {
        const float corr = (m == -INFINITY) ? 0.0f : expf(m - mnew);
        l *= corr;
#pragma unroll
        for (int c = 0; c < D; ++c) o[c] *= corr;
#pragma unroll 1
        for (int g = 0; g < kTile / 8; ++g) {
          uint32_t bits = 0xFFu;
          if (a.drop.thr) bits = dropout_bits8(a.drop, 0, ((head + i) * S + j0 + g * 8) >> 3);
#pragma unroll 1
          for (int t = 0; t < 8; ++t) {
            const int jj = g * 8 + t;
            const float p = sc[jj] == -INFINITY ? 0.0f : expf(sc[jj] - mnew);
            l += p;
            if ((bits >> t) & 1u) {
              const float w = a.drop.thr ? p * a.drop.scale : p;
#pragma unroll
              for (int c = 0; c < D; ++c) o[c] = fmaf(w, Vs[jj][c], o[c]);
            }
          }
        }
        m = mnew;
      }
    }
    __syncthreads();
  }
  if (i < S) {
    T* ctx = static_cast<T*>(a.ctx) + ((size_t)b * S + i) * H + h * D;
    const float inv = l > 0.0f ? 1.0f / l : 0.0f;
#pragma unroll
    for (int c = 0; c < D; ++c) ctx[c] = from_f<T>(o[c] * inv);
    a.lse[head + i] = l > 0.0f ? m + logf(l) : INFINITY;
  }
}

// dvec[b, h, i] = sum_c dctx[t, h*d + c] * ctx[t, h*d + c]   (= sum_j P dP)
template <typename T>
__global__ void attn_dvec_kernel(AttnArgs a) {
  const size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
  const size_t total = (size_t)a.B * a.nh * a.S;
  if (idx >= total) return;
  const int i = idx % a.S;
  const int h = (idx / a.S) % a.nh;
  const int b = idx / ((size_t)a.S * a.nh);
  const int H = a.nh * a.d;
  const size_t off = ((size_t)b * a.S + i) * H + (size_t)h * a.d;
  const T* dO = static_cast<const T*>(a.dctx) + off;
  const T* O = static_cast<const T*>(a.ctx) + off;
  float s = 0.0f;
  for (int c = 0; c < a.d; c += 8) {
    float x[8], y[8];
    load8<T>(dO + c, x);
    load8<T>(O + c, y);
#pragma unroll
    for (int k = 0; k < 8; ++k) s = fmaf(x[k], y[k], s);
  }
  a.dvec[idx] = s;
}

template <typename T, int D>
__global__ void __launch_bounds__(kRows) attn_bwd_dq_simt(AttnArgs a) {
  __shared__ float Ks[kTile][D];
  __shared__ float Vs[kTile][D];
  const int S = a.S, H = a.nh * D;
  const int b = blockIdx.z, h = blockIdx.y;
  const int i = blockIdx.x * kRows + threadIdx.x;
  const size_t head = ((size_t)b * a.nh + h) * S;
  const T* Q = static_cast<const T*>(a.q);
  const T* K = static_cast<const T*>(a.k);
  const T* V = static_cast<const T*>(a.v);
  const T* dO = static_cast<const T*>(a.dctx);
  float q[D], dov[D], dq[D];
  const size_t trow = (size_t)b * S + i;
#pragma unroll
  for (int c = 0; c < D; ++c) {
    q[c] = i < S ? to_f(Q[(head + i) * D + c]) : 0.0f;
    dov[c] = i < S ? to_f(dO[trow * H + h * D + c]) : 0.0f;
    dq[c] = 0.0f;
  }
  const float lse = i < S ? a.lse[head + i] : INFINITY;
  const float Di = i < S ? a.dvec[head + i] : 0.0f;
  for (int j0 = 0; j0 < S; j0 += kTile) {
    for (int idx = threadIdx.x; idx < kTile * D; idx += kRows) {
      const int jj = idx / D, c = idx % D, j = j0 + jj;
      Ks[jj][c] = j < S ? to_f(K[(head + j) * D + c]) : 0.0f;
      Vs[jj][c] = j < S ? to_f(V[(head + j) * D + c]) : 0.0f;
    }
    __syncthreads();
    if (i < S) {
#pragma unroll 1
      for (int g = 0; g < kTile / 8; ++g) {
        if (j0 + g * 8 >= S) break;
        uint32_t bits = 0xFFu;
        if (a.drop.thr) bits = dropout_bits8(a.drop, 0, ((head + i) * S + j0 + g * 8) >> 3);
#pragma unroll 1
        for (int t = 0; t < 8; ++t) {
          const int jj = g * 8 + t, j = j0 + jj;
          float dot = 0.0f, dpd = 0.0f;
#pragma unroll
          for (int c = 0; c < D; ++c) {
            dot = fmaf(q[c], Ks[jj][c], dot);
            dpd = fmaf(dov[c], Vs[jj][c], dpd);
          }
          const float s = dot * a.scale + (a.mask ? a.mask[(size_t)b * S + j] : 0.0f);
          const float p = s == -INFINITY ? 0.0f : expf(s - lse);
          const float dp = ((bits >> t) & 1u) ? (a.drop.thr ? dpd * a.drop.scale : dpd) : 0.0f;
          const float ds = p * (dp - Di);
#pragma unroll
          for (int c = 0; c < D; ++c) dq[c] = fmaf(ds, Ks[jj][c], dq[c]);
        }
      }
    }
    __syncthreads();
  }
  if (i < S) {
    T* out = static_cast<T*>(a.dqkv) + trow * 3 * H + h * D;
#pragma unroll
    for (int c = 0; c < D; ++c) out[c] = from_f<T>(dq[c] * a.scale);
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kRows) attn_bwd_dkdv_simt(AttnArgs a) {
  __shared__ float Qs[kTile][D];
  __shared__ float dOs[kTile][D];
  __shared__ float Ls[kTile], Ds[kTile];
  const int S = a.S, H = a.nh * D;
  const int b = blockIdx.z, h = blockIdx.y;
  const int j = blockIdx.x * kRows + threadIdx.x;
  const size_t head = ((size_t)b * a.nh + h) * S;
  const T* Q = static_cast<const T*>(a.q);
  const T* K = static_cast<const T*>(a.k);
  const T* V = static_cast<const T*>(a.v);
  const T* dO = static_cast<const T*>(a.dctx);
  float k[D], v[D], dk[D], dv[D];
#pragma unroll
  for (int c = 0; c < D; ++c) {
    k[c] = j < S ? to_f(K[(head + j) * D + c]) : 0.0f;
    v[c] = j < S ? to_f(V[(head + j) * D + c]) : 0.0f;
    dk[c] = dv[c] = 0.0f;
  }
  const float mj = (j < S && a.mask) ? a.mask[(size_t)b * S + j] : 0.0f;
  for (int i0 = 0; i0 < S; i0 += kTile) {
    for (int idx = threadIdx.x; idx < kTile * D; idx += kRows) {
      const int ii = idx / D, c = idx % D, i = i0 + ii;
      Qs[ii][c] = i < S ? to_f(Q[(head + i) * D + c]) : 0.0f;
      dOs[ii][c] = i < S ? to_f(dO[((size_t)b * S + i) * H + h * D + c]) : 0.0f;
    }
    for (int ii = threadIdx.x; ii < kTile; ii += kRows) {
      Ls[ii] = i0 + ii < S ? a.lse[head + i0 + ii] : INFINITY;
      Ds[ii] = i0 + ii < S ? a.dvec[head + i0 + ii] : 0.0f;
    }
    __syncthreads();
    if (j < S && mj != -INFINITY) {
#pragma unroll 1
      for (int ii = 0; ii < kTile && i0 + ii < S; ++ii) {
        const int i = i0 + ii;
        float dot = 0.0f, dpd = 0.0f;
#pragma unroll
        for (int c = 0; c < D; ++c) {
          dot = fmaf(Qs[ii][c], k[c], dot);
          dpd = fmaf(dOs[ii][c], v[c], dpd);
        }
        const float s = dot * a.scale + mj;
        const float p = expf(s - Ls[ii]);
        bool keep = true;
        if (a.drop.thr) {
          const uint64_t e = (head + i) * S + j;
          keep = (dropout_bits8(a.drop, 0, e >> 3) >> (e & 7)) & 1u;
        }
        const float sc = a.drop.thr ? a.drop.scale : 1.0f;
        const float pd = keep ? p * sc : 0.0f;
        const float dp = keep ? dpd * sc : 0.0f;
        const float ds = p * (dp - Ds[ii]);
#pragma unroll
        for (int c = 0; c < D; ++c) {
          dv[c] = fmaf(pd, dOs[ii][c], dv[c]);
          dk[c] = fmaf(ds, Qs[ii][c], dk[c]);
        }
      }
    }
    __syncthreads();
  }
  if (j < S) {
    T* out = static_cast<T*>(a.dqkv) + ((size_t)b * S + j) * 3 * H + h * D;
#pragma unroll
    for (int c = 0; c < D; ++c) {
      out[H + c] = from_f<T>(dk[c] * a.scale);
      out[2 * H + c] = from_f<T>(dv[c]);
    }
  }
}

template <typename T, int D>
void fwd_t(const AttnArgs& a, cudaStream_t s) {
  dim3 grid((a.S + kRows - 1) / kRows, a.nh, a.B);
  attn_fwd_simt<T, D><<<grid, kRows, 0, s>>>(a);
  count_launch();
}

template <typename T, int D>
void bwd_t(const AttnArgs& a, cudaStream_t s) {
  const size_t rows = (size_t)a.B * a.nh * a.S;
  attn_dvec_kernel<T><<<(unsigned)((rows + 255) / 256), 256, 0, s>>>(a);
  dim3 grid((a.S + kRows - 1) / kRows, a.nh, a.B);
  attn_bwd_dq_simt<T, D><<<grid, kRows, 0, s>>>(a);
  attn_bwd_dkdv_simt<T, D><<<grid, kRows, 0, s>>>(a);
  count_launch(3);
}

template <typename T>
void dispatch(bool fwd, const AttnArgs& a, cudaStream_t s) {
  switch (a.d) {
    case 16: fwd ? fwd_t<T, 16>(a, s) : bwd_t<T, 16>(a, s); break;
    case 32: fwd ? fwd_t<T, 32>(a, s) : bwd_t<T, 32>(a, s); break;
    case 64: fwd ? fwd_t<T, 64>(a, s) : bwd_t<T, 64>(a, s); break;
    case 128: fwd ? fwd_t<T, 128>(a, s) : bwd_t<T, 128>(a, s); break;
  }
}

}  // namespace

void dvec_launch(int dt, const AttnArgs& a, cudaStream_t s) {
  const size_t rows = (size_t)a.B * a.nh * a.S;
  const unsigned blocks = (unsigned)((rows + 255) / 256);
  if (dt == DT_F32) attn_dvec_kernel<float><<<blocks, 256, 0, s>>>(a);
  else if (dt == DT_F16) attn_dvec_kernel<half_t><<<blocks, 256, 0, s>>>(a);
  else attn_dvec_kernel<bf16_t><<<blocks, 256, 0, s>>>(a);
  count_launch();
}

void attn_simt_fwd_run(int dt, const AttnArgs& a, cudaStream_t s) {
  if (dt == DT_F32) dispatch<float>(true, a, s);
  else if (dt == DT_F16) dispatch<half_t>(true, a, s);
  else dispatch<bf16_t>(true, a, s);
}

void attn_simt_bwd_run(int dt, const AttnArgs& a, cudaStream_t s) {
  if (dt == DT_F32) dispatch<float>(false, a, s);
  else if (dt == DT_F16) dispatch<half_t>(false, a, s);
  else dispatch<bf16_t>(false, a, s);
}

}  // namespace tlp
