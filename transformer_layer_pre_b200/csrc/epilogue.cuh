// epilogue.cuh — fused GEMM epilogues, applied to 8 consecutive columns
// (n % 8 == 0) of one output row m, with v holding the float32 accumulators.
//
//  EPI_QKV            bias + head split: column n of the fused [Q|K|V]
//                     projection goes to tensor n/H, head (n%H)/d, lane n%d,
//                     laid out (B, heads, S, d) so attention reads contiguous
//                     (S, d) blocks ("AI-infra engineers and the Transformer",
//                     section 2.1 Steps 2-3: Linear(D, 3D), then view and
//                     permute to (B, H, S, D/H)).
//  EPI_BIAS_DROP_RES  out = res + dropout(acc + bias) (the output projection
//                     and FFN2 sites, "DeepSpeed Transformer Kernel usage
//                     guide", Step 2 hidden_dropout_ratio).
//  EPI_BIAS_GELU      U = acc + bias stored; G = GELU(U as stored) so that a
//                     backward that recomputes G from U gets identical bits.
//  EPI_DGELU          out = acc * GELU'(U).
//  EPI_STORE          out = acc (+ res).
//  EPI_F32            float32 out = acc.
#pragma once

#include "common.cuh"
#include "kernels.h"

namespace tlp {

template <typename T, int KIND>
__device__ __forceinline__ void epi_apply8(const EpiParams& e, int m, int n, float (&v)[8]) {
  if constexpr (KIND == EPI_F32) {
    float* o = static_cast<float*>(e.out) + (size_t)m * e.ldo + n;
    store8<float>(o, v);
  } else if constexpr (KIND == EPI_STORE) {
    if (e.res) {
      float r[8];
      load8<T>(static_cast<const T*>(e.res) + (size_t)m * e.ldo + n, r);
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] += r[i];
    }
    store8<T>(static_cast<T*>(e.out) + (size_t)m * e.ldo + n, v);
  } else if constexpr (KIND == EPI_QKV) {
    float b[8];
    load8<T>(static_cast<const T*>(e.bias) + n, b);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] += b[i];
    const int which = n / e.hidden;
    const int c = n - which * e.hidden;
    const int h = c / e.head_dim;
    const int lane = c - h * e.head_dim;
    const int bb = m / e.seq;
    const int s = m - bb * e.seq;
    const size_t dst = (size_t)which * e.tokens * e.hidden +
                       ((size_t)(bb * e.heads + h) * e.seq + s) * e.head_dim + lane;
    store8<T>(static_cast<T*>(e.out) + dst, v);
  } else if constexpr (KIND == EPI_BIAS_DROP_RES) {
    float b[8], r[8];
    load8<T>(static_cast<const T*>(e.bias) + n, b);
    load8<T>(static_cast<const T*>(e.res) + (size_t)m * e.ldo + n, r);
    uint32_t bits = 0xFFu;
    if (e.drop.thr) bits = dropout_bits8(e.drop, e.site, ((uint64_t)m * e.ldo + n) >> 3);
    const float sc = e.drop.thr ? e.drop.scale : 1.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = r[i] + (((bits >> i) & 1u) ? (v[i] + b[i]) * sc : 0.0f);
    store8<T>(static_cast<T*>(e.out) + (size_t)m * e.ldo + n, v);
  } else if constexpr (KIND == EPI_BIAS_GELU) {
    float b[8];
    load8<T>(static_cast<const T*>(e.bias) + n, b);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = round_f<T>(v[i] + b[i]);
    store8<T>(static_cast<T*>(e.out) + (size_t)m * e.ldo + n, v);
    if (e.out2) {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = gelu_f(v[i]);
      store8<T>(static_cast<T*>(e.out2) + (size_t)m * e.ldo + n, v);
    }
  } else if constexpr (KIND == EPI_DGELU) {
    float u[8];
    load8<T>(static_cast<const T*>(e.aux) + (size_t)m * e.ldo + n, u);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] *= gelu_grad_f(u[i]);
    store8<T>(static_cast<T*>(e.out) + (size_t)m * e.ldo + n, v);
  }
}

}  // namespace tlp
