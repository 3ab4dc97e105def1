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
//                     backward that recomputes G from U gets identical bits
//                     (erf form, or the tanh form for KIND | EPI_TANH).
//  EPI_DGELU          out = acc * GELU'(U), GELU'(U) rounded to the storage type
//                     first, as EPI_BIAS_GELU_D stores it (both paths give the
//                     same bits).
//  EPI_BIAS_GELU_D    U = acc + bias rounded to storage (not stored);
//                     out = GELU'(U), out2 = G = GELU(U), both from one
//                     evaluation of the normal density and tail (or of tanh).
//                     The backward then needs no special function:
//  EPI_MUL            out = acc * aux (aux = the stored GELU'(U)).
//  EPI_STORE          out = acc (+ res).
//  EPI_F32            float32 out = acc.
//
// `aux` carries the 8 residual (EPI_BIAS_DROP_RES, EPI_STORE with res), U
// (EPI_DGELU) or factor (EPI_MUL) values of the chunk, loaded by the caller
// ahead of time.
#pragma once

#include "common.cuh"
#include "kernels.h"

namespace tlp {

// Flag bit on a kernel's compile-time epilogue kind: GELU (EPI_BIAS_GELU,
// EPI_BIAS_GELU_D, EPI_DGELU) in its tanh form (EpiParams.gelu_tanh at run time).  The low
// bits are the EpiKind.
constexpr int EPI_TANH = 16;
constexpr int epi_base(int kind) { return kind & (EPI_TANH - 1); }

// Whether a kind reads a per-element auxiliary input (and which pointer).
template <int KIND> struct EpiAux {
  static constexpr bool kNeeds =
      epi_base(KIND) == EPI_BIAS_DROP_RES || epi_base(KIND) == EPI_DGELU || epi_base(KIND) == EPI_STORE ||
      epi_base(KIND) == EPI_MUL;
};
__device__ __forceinline__ const void* epi_aux_ptr(const EpiParams& e, int kind) {
  return kind == EPI_DGELU || kind == EPI_MUL ? e.aux : e.res;
}
// Kinds with two stored outputs (out and out2).
constexpr bool epi_two_outputs(int kind) {
  return epi_base(kind) == EPI_BIAS_GELU || epi_base(kind) == EPI_BIAS_GELU_D;
}
// Kinds whose tensor-core epilogue can also sum the stored output's columns.
constexpr bool epi_sums_columns(int kind) { return epi_base(kind) == EPI_DGELU || epi_base(kind) == EPI_MUL; }

// v *= GELU'(u) with GELU'(u) rounded to the storage type T (the value
// EPI_BIAS_GELU_D stores for EPI_MUL), over 8 lanes.
template <typename T>
__device__ __forceinline__ void mul_stored_gelu_grad8(float (&v)[8], const float (&u)[8], bool tanh_form) {
  float g[8], d[8];
  gelu_and_grad8_form(u, g, d, tanh_form);
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] *= round_f<T>(d[i]);
}

// Row-dependent part of the EPI_QKV destination, computed once per row.
__device__ __forceinline__ size_t qkv_row_base(const EpiParams& e, int m) {
  const int bb = m / e.seq;
  const int s = m - bb * e.seq;
  return ((size_t)bb * e.heads * e.seq + s) * e.head_dim;
}

template <typename T, int KIND>
__device__ __forceinline__ void epi_apply8(const EpiParams& e, int m, int n, float (&v)[8], const float (&aux)[8],
                                           size_t row_base) {
  if constexpr (epi_base(KIND) == EPI_F32) {
    float* o = static_cast<float*>(e.out) + (size_t)m * e.ldo + n;
    store8<float>(o, v);
  } else if constexpr (epi_base(KIND) == EPI_STORE) {
    if (e.res) {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] += aux[i];
    }
    store8<T>(static_cast<T*>(e.out) + (size_t)m * e.ldo + n, v);
  } else if constexpr (epi_base(KIND) == EPI_QKV) {
    float b[8];
    load8<T>(static_cast<const T*>(e.bias) + n, b);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] += b[i];
    // which of Q, K, V; head and lane by shifts (head_dim is a power of two)
    const int which = (n >= e.hidden) + (n >= 2 * e.hidden);
    const int c = n - which * e.hidden;
    const int sh = __ffs(e.head_dim) - 1;
    const int h = c >> sh;
    const int lane = c & (e.head_dim - 1);
    const size_t dst = (size_t)which * e.tokens * e.hidden + row_base + ((size_t)h * e.seq << sh) + lane;
    store8<T>(static_cast<T*>(e.out) + dst, v);
  } else if constexpr (epi_base(KIND) == EPI_BIAS_DROP_RES) {
    float b[8];
    load8<T>(static_cast<const T*>(e.bias) + n, b);
    uint32_t bits = 0xFFu;
    if (e.keep8) bits = e.keep8[((uint64_t)m * e.ldo + n) >> 3];
    else if (e.drop.thr) bits = dropout_bits8(e.drop, e.site, ((uint64_t)m * e.ldo + n) >> 3);
    const float sc = e.drop.thr ? e.drop.scale : 1.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = aux[i] + (((bits >> i) & 1u) ? (v[i] + b[i]) * sc : 0.0f);
    store8<T>(static_cast<T*>(e.out) + (size_t)m * e.ldo + n, v);
  } else if constexpr (epi_base(KIND) == EPI_BIAS_GELU) {
    float b[8];
    load8<T>(static_cast<const T*>(e.bias) + n, b);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = round_f<T>(v[i] + b[i]);
    store8<T>(static_cast<T*>(e.out) + (size_t)m * e.ldo + n, v);
    if (e.out2) {
      gelu8_form(v, (KIND & EPI_TANH) != 0);
      store8<T>(static_cast<T*>(e.out2) + (size_t)m * e.ldo + n, v);
    }
  } else if constexpr (epi_base(KIND) == EPI_DGELU) {
    mul_stored_gelu_grad8<T>(v, aux, (KIND & EPI_TANH) != 0);
    store8<T>(static_cast<T*>(e.out) + (size_t)m * e.ldo + n, v);
  } else if constexpr (epi_base(KIND) == EPI_BIAS_GELU_D) {
    float b[8], g[8], d[8];
    load8<T>(static_cast<const T*>(e.bias) + n, b);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = round_f<T>(v[i] + b[i]);
    gelu_and_grad8_form(v, g, d, (KIND & EPI_TANH) != 0);
    store8<T>(static_cast<T*>(e.out) + (size_t)m * e.ldo + n, d);
    store8<T>(static_cast<T*>(e.out2) + (size_t)m * e.ldo + n, g);
  } else if constexpr (epi_base(KIND) == EPI_MUL) {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] *= aux[i];
    store8<T>(static_cast<T*>(e.out) + (size_t)m * e.ldo + n, v);
  }
}

// Epilogue arithmetic without the store: v becomes the (first) output chunk,
// v2 the second one (the G of EPI_BIAS_GELU and EPI_BIAS_GELU_D).  Used by the tensor-core GEMM, whose
// stores go through shared memory and TMA.
// kbits: the 8 dropout keep bits of this chunk when the caller already has
// them (EPI_BIAS_DROP_RES), or a value above 0xFF to look them up here.
template <typename T, int KIND>
__device__ __forceinline__ void epi_compute8(const EpiParams& e, int m, int n, float (&v)[8], float (&v2)[8],
                                             const float (&aux)[8], uint32_t kbits = 0x100u) {
  if constexpr (epi_base(KIND) == EPI_STORE) {
    if (e.res) {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] += aux[i];
    }
  } else if constexpr (epi_base(KIND) == EPI_QKV) {
    float b[8];
    load8<T>(static_cast<const T*>(e.bias) + n, b);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] += b[i];
  } else if constexpr (epi_base(KIND) == EPI_BIAS_DROP_RES) {
    float b[8];
    load8<T>(static_cast<const T*>(e.bias) + n, b);
    uint32_t bits = 0xFFu;
    if (kbits <= 0xFFu) bits = kbits;
    else if (e.keep8) bits = e.keep8[((uint64_t)m * e.ldo + n) >> 3];
    else if (e.drop.thr) bits = dropout_bits8(e.drop, e.site, ((uint64_t)m * e.ldo + n) >> 3);
    const float sc = e.drop.thr ? e.drop.scale : 1.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = aux[i] + (((bits >> i) & 1u) ? (v[i] + b[i]) * sc : 0.0f);
  } else if constexpr (epi_base(KIND) == EPI_BIAS_GELU) {
    float b[8];
    load8<T>(static_cast<const T*>(e.bias) + n, b);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[i] = round_f<T>(v[i] + b[i]);
      v2[i] = v[i];
    }
    gelu8_form(v2, (KIND & EPI_TANH) != 0);
  } else if constexpr (epi_base(KIND) == EPI_DGELU) {
    mul_stored_gelu_grad8<T>(v, aux, (KIND & EPI_TANH) != 0);
  } else if constexpr (epi_base(KIND) == EPI_BIAS_GELU_D) {
    float b[8], u[8];
    load8<T>(static_cast<const T*>(e.bias) + n, b);
#pragma unroll
    for (int i = 0; i < 8; ++i) u[i] = round_f<T>(v[i] + b[i]);
    gelu_and_grad8_form(u, v2, v, (KIND & EPI_TANH) != 0);
  } else if constexpr (epi_base(KIND) == EPI_MUL) {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] *= aux[i];
  }
}

// Convenience form that loads the auxiliary values itself (SIMT GEMM).
template <typename T, int KIND>
__device__ __forceinline__ void epi_apply8(const EpiParams& e, int m, int n, float (&v)[8]) {
  float aux[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  if constexpr (EpiAux<KIND>::kNeeds) {
    const void* p = epi_aux_ptr(e, epi_base(KIND));
    if (p) load8<T>(static_cast<const T*>(p) + (size_t)m * e.ldo + n, aux);
  }
  size_t rb = 0;
  if constexpr (epi_base(KIND) == EPI_QKV) rb = qkv_row_base(e, m);
  epi_apply8<T, KIND>(e, m, n, v, aux, rb);
}

}  // namespace tlp
