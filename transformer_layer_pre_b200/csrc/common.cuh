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
__device__ __forceinline__ float gelu_f(float u) { return 0.5f * u * (1.0f + erff(u * 0.70710678118654752f)); }
__device__ __forceinline__ float gelu_grad_f(float u) {
  return fmaf(u * 0.39894228040143268f, __expf(-0.5f * u * u), 0.5f * (1.0f + erff(u * 0.70710678118654752f)));
}

// ------------------------------------------------------------------ warp reductions
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

}  // namespace tlp
