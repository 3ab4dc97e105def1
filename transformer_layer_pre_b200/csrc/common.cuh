// common.cuh — storage types, 8-wide vector I/O, Philox dropout bits.
//
// Every kernel of the layer keeps activations in the storage type T
// (float, __half or __nv_bfloat16) and computes in float32.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace tlp {

typedef __half half_t;
typedef __nv_bfloat16 bf16_t;

// ------------------------------------------------------------------ programmatic dependent launch
// Kernels of the layer are launched with programmatic stream serialization
// (launch_pdl in kernels.h): a kernel may be scheduled while the previous
// kernel of the stream is still finishing, runs its local setup (barriers,
// tensor memory, descriptor prefetch), and then pdl_wait() blocks until that
// previous kernel has completed and its memory is visible.  No global memory
// is read or written before pdl_wait().  pdl_launch_dependents() lets the
// next kernel start being scheduled (it still waits for this one to finish).
// Both are no-ops for an ordinary launch.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ------------------------------------------------------------------ scalar conversion
__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(half_t v) { return __half2float(v); }
__device__ __forceinline__ float to_f(bf16_t v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ half_t from_f<half_t>(float v) { return __float2half_rn(v); }
template <> __device__ __forceinline__ bf16_t from_f<bf16_t>(float v) { return __float2bfloat16_rn(v); }

// Round a float32 value to T and back (what storing and re-loading yields).
template <typename T> __device__ __forceinline__ float round_f(float v) { return to_f(from_f<T>(v)); }

// ------------------------------------------------------------------ 8-wide vectors
// p must be 16-byte aligned for 16-bit T and 32-byte aligned for float.
template <typename T> struct Vec8Io;

template <> struct Vec8Io<float> {
  static __device__ __forceinline__ void load(const float* p, float (&v)[8]) {
    float4 a = reinterpret_cast<const float4*>(p)[0];
    float4 b = reinterpret_cast<const float4*>(p)[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
  static __device__ __forceinline__ void store(float* p, const float (&v)[8]) {
    reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
};

template <typename T2, typename T> struct Vec8Io16 {
  static __device__ __forceinline__ void load(const T* p, float (&v)[8]) {
    uint4 r = *reinterpret_cast<const uint4*>(p);
    const T2* h = reinterpret_cast<const T2*>(&r);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = to_f(h[i].x);
      v[2 * i + 1] = to_f(h[i].y);
    }
  }
  static __device__ __forceinline__ void store(T* p, const float (&v)[8]) {
    uint4 r;
    T* h = reinterpret_cast<T*>(&r);
#pragma unroll
    for (int i = 0; i < 8; ++i) h[i] = from_f<T>(v[i]);
    *reinterpret_cast<uint4*>(p) = r;
  }
};
template <> struct Vec8Io<half_t> : Vec8Io16<__half2, half_t> {};
template <> struct Vec8Io<bf16_t> : Vec8Io16<__nv_bfloat162, bf16_t> {};

template <typename T> __device__ __forceinline__ void load8(const T* p, float (&v)[8]) { Vec8Io<T>::load(p, v); }

// 8 16-bit values held in a uint4 (as loaded by a 16-byte vector load) to float.
template <typename T> __device__ __forceinline__ void unpack8(const uint4& r, float (&v)[8]) {
  const T* h = reinterpret_cast<const T*>(&r);
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = to_f(h[i]);
}
// 8 floats rounded to the 16-bit type T, packed as a 16-byte vector (the
// inverse of unpack8).
template <typename T> __device__ __forceinline__ uint4 pack8(const float (&v)[8]) {
  uint4 r;
  T* h = reinterpret_cast<T*>(&r);
#pragma unroll
  for (int i = 0; i < 8; ++i) h[i] = from_f<T>(v[i]);
  return r;
}
// Raw 8-element chunk as loaded from memory (16 bytes for 16-bit types, 32
// for float), so a load can be issued early and converted later.
template <typename T> struct Raw8 { uint4 a; };
template <> struct Raw8<float> { float4 a, b; };

template <typename T> __device__ __forceinline__ Raw8<T> raw8_load(const T* p) {
  Raw8<T> r;
  r.a = *reinterpret_cast<const uint4*>(p);
  return r;
}
template <> __device__ __forceinline__ Raw8<float> raw8_load<float>(const float* p) {
  Raw8<float> r;
  r.a = reinterpret_cast<const float4*>(p)[0];
  r.b = reinterpret_cast<const float4*>(p)[1];
  return r;
}
template <typename T> __device__ __forceinline__ Raw8<T> raw8_zero() {
  Raw8<T> r;
  r.a = make_uint4(0u, 0u, 0u, 0u);
  return r;
}
template <> __device__ __forceinline__ Raw8<float> raw8_zero<float>() {
  Raw8<float> r;
  r.a = r.b = make_float4(0.f, 0.f, 0.f, 0.f);
  return r;
}
template <typename T> __device__ __forceinline__ void raw8_unpack(const Raw8<T>& r, float (&v)[8]) { unpack8<T>(r.a, v); }
template <> __device__ __forceinline__ void raw8_unpack<float>(const Raw8<float>& r, float (&v)[8]) {
  v[0] = r.a.x; v[1] = r.a.y; v[2] = r.a.z; v[3] = r.a.w; v[4] = r.b.x; v[5] = r.b.y; v[6] = r.b.z; v[7] = r.b.w;
}

template <typename T> __device__ __forceinline__ void store8(T* p, const float (&v)[8]) { Vec8Io<T>::store(p, v); }

// ------------------------------------------------------------------ Philox4x32-10
// Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3"
// (SC'11): ten rounds; each multiplies counter words 0 and 2 by fixed odd
// constants, swaps the halves of the products across the words and XORs in
// the key, which is advanced by a Weyl sequence between rounds.
struct Philox4 {
  uint32_t x, y, z, w;
};

__device__ __forceinline__ Philox4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3,
                                                 uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint32_t hi0 = __umulhi(0xD2511F53u, c0), lo0 = 0xD2511F53u * c0;
    const uint32_t hi1 = __umulhi(0xCD9E8D57u, c2), lo1 = 0xCD9E8D57u * c2;
    const uint32_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
    c0 = n0; c1 = lo1; c2 = n2; c3 = lo0;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  Philox4 o = {c0, c1, c2, c3};
  return o;
}

// Dropout contract (shared by every kernel that drops or regenerates a
// mask): flat element e of site s uses counter (e/8 lo, e/8 hi, s, offset)
// and key (seed lo, seed hi); lane e%8 = k is the 16-bit half (k&1) of word
// k>>1; the element is kept when that lane >= thr = floor(p*65536).
struct DropoutParams {
  uint64_t seed;
  uint64_t offset;
  uint32_t thr;   // 0 disables dropout
  float scale;    // 1/(1-p)
};

// Keep bits of the 8 elements e8*8 .. e8*8+7 (bit k = lane k).
__device__ __forceinline__ uint32_t dropout_bits8(const DropoutParams& dp, int site, uint64_t e8) {
  const Philox4 r = philox4x32_10((uint32_t)e8, (uint32_t)(e8 >> 32), (uint32_t)site, (uint32_t)dp.offset,
                                  (uint32_t)dp.seed, (uint32_t)(dp.seed >> 32));
  const uint32_t w[4] = {r.x, r.y, r.z, r.w};
  uint32_t bits = 0;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t lane = (w[k >> 1] >> (16 * (k & 1))) & 0xFFFFu;
    bits |= (lane >= dp.thr ? 1u : 0u) << k;
  }
  return bits;
}

// ------------------------------------------------------------------ GELU (erf form)
// GELU(u) = u * Phi(u), Phi the standard normal distribution function.  Phi
// comes from the normal upper-tail approximation of Abramowitz & Stegun,
// "Handbook of Mathematical Functions", formula 26.2.17 (after Hastings):
// for z >= 0
//   Q(z) = 1 - Phi(z) = phi(z) (b1 t + b2 t^2 + b3 t^3 + b4 t^4 + b5 t^5) + e(z),
//   t = 1 / (1 + p z),   |e(z)| < 7.5e-8,
// phi the normal density; Phi(u) = 1 - Q(u) for u >= 0, Q(-u) otherwise, and
// GELU'(u) = Phi(u) + u phi(u).  Lanes are evaluated in pairs with the packed
// float32 FMA/multiply of sm_100, plus one reciprocal and one base-2
// exponential per element on the special-function unit.  Every step is an
// explicit single-rounded operation (nothing left to FMA contraction), so
// each kernel that evaluates GELU gets the same bits for the same input.
__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ float ex2_approx(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ float2 f2(float a) { return make_float2(a, a); }

// phi(|u|) and Q(|u|) of a pair of lanes.
__device__ __forceinline__ void normal_tail2(float2 u, float2& phi, float2& q) {
  constexpr float kP = 0.2316419f;
  constexpr float kB1 = 0.319381530f, kB2 = -0.356563782f, kB3 = 1.781477937f, kB4 = -1.821255978f,
                  kB5 = 1.330274429f;
  constexpr float kInvSqrt2Pi = 0.398942280401432678f;
  constexpr float kNegHalfLog2e = -0.721347520444481703f;   // exp(-z^2/2) = 2^(z^2 * kNegHalfLog2e)
  const float2 z = make_float2(fabsf(u.x), fabsf(u.y));
  float2 t = __ffma2_rn(z, f2(kP), f2(1.0f));
  t = make_float2(rcp_approx(t.x), rcp_approx(t.y));
  float2 s = __ffma2_rn(t, f2(kB5), f2(kB4));
  s = __ffma2_rn(t, s, f2(kB3));
  s = __ffma2_rn(t, s, f2(kB2));
  s = __ffma2_rn(t, s, f2(kB1));
  s = __fmul2_rn(s, t);
  const float2 a = __fmul2_rn(__fmul2_rn(z, f2(kNegHalfLog2e)), z);
  phi = __fmul2_rn(make_float2(ex2_approx(a.x), ex2_approx(a.y)), f2(kInvSqrt2Pi));
  q = __fmul2_rn(phi, s);
}
__device__ __forceinline__ float2 normal_cdf2(float2 u, float2 q) {
  return make_float2(u.x >= 0.0f ? __fsub_rn(1.0f, q.x) : q.x, u.y >= 0.0f ? __fsub_rn(1.0f, q.y) : q.y);
}
__device__ __forceinline__ float2 gelu2(float2 u) {
  float2 phi, q;
  normal_tail2(u, phi, q);
  return __fmul2_rn(u, normal_cdf2(u, q));
}
__device__ __forceinline__ float2 gelu_grad2(float2 u) {
  float2 phi, q;
  normal_tail2(u, phi, q);
  return __ffma2_rn(u, phi, normal_cdf2(u, q));
}
// In-place over 8 lanes.
__device__ __forceinline__ void gelu8(float (&v)[8]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 g = gelu2(make_float2(v[2 * i], v[2 * i + 1]));
    v[2 * i] = g.x;
    v[2 * i + 1] = g.y;
  }
}

// GELU in its tanh approximation ("AI-infra engineers and the Transformer",
// section 2.3): GELU(u) = u (1 + tanh(z)) / 2 with z = sqrt(2/pi) (u + 0.044715 u^3),
// GELU'(u) = (1 + t)/2 + u (1 - t^2) sqrt(2/pi) (1 + 3 * 0.044715 u^2) / 2, t = tanh(z).
// tanh(|z|) = (1 - e) / (1 + e) with e = exp(-2|z|) (one base-2 exponential and
// one reciprocal per element), the sign restored from z.
__device__ __forceinline__ float2 tanh_gelu_arg2(float2 u) {
  constexpr float kS = 0.797884560802865356f;      // sqrt(2/pi)
  constexpr float kC = 0.044715f;
  constexpr float kM2Log2e = -2.88539008177792682f;   // exp(-2a) = 2^(a * kM2Log2e)
  const float2 z = __fmul2_rn(__fmul2_rn(u, f2(kS)), __ffma2_rn(__fmul2_rn(u, u), f2(kC), f2(1.0f)));
  const float2 a = __fmul2_rn(make_float2(fabsf(z.x), fabsf(z.y)), f2(kM2Log2e));
  const float2 e = make_float2(ex2_approx(a.x), ex2_approx(a.y));
  const float2 den = __fadd2_rn(e, f2(1.0f));
  const float2 t = __fmul2_rn(__ffma2_rn(e, f2(-1.0f), f2(1.0f)), make_float2(rcp_approx(den.x), rcp_approx(den.y)));
  return make_float2(copysignf(t.x, z.x), copysignf(t.y, z.y));
}
__device__ __forceinline__ float2 gelu_tanh2(float2 u) {
  const float2 t = tanh_gelu_arg2(u);
  return __fmul2_rn(__fmul2_rn(u, f2(0.5f)), __fadd2_rn(t, f2(1.0f)));
}
__device__ __forceinline__ float2 gelu_tanh_grad2(float2 u) {
  constexpr float kS = 0.797884560802865356f;
  constexpr float kC3 = 3.0f * 0.044715f;
  const float2 t = tanh_gelu_arg2(u);
  const float2 sech2 = __ffma2_rn(t, make_float2(-t.x, -t.y), f2(1.0f));                  // 1 - t^2
  const float2 dz = __fmul2_rn(__ffma2_rn(__fmul2_rn(u, u), f2(kC3), f2(1.0f)), f2(kS));  // dz/du
  const float2 half_u = __fmul2_rn(u, f2(0.5f));
  return __ffma2_rn(__fmul2_rn(half_u, sech2), dz, __fmul2_rn(__fadd2_rn(t, f2(1.0f)), f2(0.5f)));
}
// GELU(u) and GELU'(u) of 8 lanes from one evaluation of phi and Q (erf form)
// or of tanh (tanh form): g = GELU(u), d = GELU'(u).
__device__ __forceinline__ void gelu_and_grad8_form(const float (&u)[8], float (&g)[8], float (&d)[8], bool tanh_form) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 x = make_float2(u[2 * i], u[2 * i + 1]);
    float2 gv, dv;
    if (!tanh_form) {
      float2 phi, q;
      normal_tail2(x, phi, q);
      const float2 cdf = normal_cdf2(x, q);
      gv = __fmul2_rn(x, cdf);
      dv = __ffma2_rn(x, phi, cdf);
    } else {
      constexpr float kS = 0.797884560802865356f;
      constexpr float kC3 = 3.0f * 0.044715f;
      const float2 t = tanh_gelu_arg2(x);
      const float2 half_u = __fmul2_rn(x, f2(0.5f));
      const float2 onep = __fadd2_rn(t, f2(1.0f));
      gv = __fmul2_rn(half_u, onep);
      const float2 sech2 = __ffma2_rn(t, make_float2(-t.x, -t.y), f2(1.0f));
      const float2 dz = __fmul2_rn(__ffma2_rn(__fmul2_rn(x, x), f2(kC3), f2(1.0f)), f2(kS));
      dv = __ffma2_rn(__fmul2_rn(half_u, sech2), dz, __fmul2_rn(onep, f2(0.5f)));
    }
    g[2 * i] = gv.x; g[2 * i + 1] = gv.y;
    d[2 * i] = dv.x; d[2 * i + 1] = dv.y;
  }
}
// In-place over 8 lanes, either form.
__device__ __forceinline__ void gelu8_form(float (&v)[8], bool tanh_form) {
  if (!tanh_form) {
    gelu8(v);
    return;
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 g = gelu_tanh2(make_float2(v[2 * i], v[2 * i + 1]));
    v[2 * i] = g.x;
    v[2 * i + 1] = g.y;
  }
}

// ------------------------------------------------------------------ warp reductions
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
// Column sums of a warp's 32 x 32 block: v holds 32 values of this lane's
// row; lane l returns the sum over the 32 lanes of v[l].  Recursive halving:
// at each step a lane keeps one half of its values and adds the partner
// lane's copy of that half (31 shuffles), in a fixed order.
__device__ __forceinline__ float warp_colsum32(float (&v)[32]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int k = 16; k >= 1; k >>= 1) {
    const bool upper = (lane & k) != 0;
#pragma unroll
    for (int i = 0; i < k; ++i) {
      const float send = upper ? v[i] : v[i + k];
      const float keep = upper ? v[i + k] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, k);
    }
  }
  return v[0];
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

}  // namespace tlp
