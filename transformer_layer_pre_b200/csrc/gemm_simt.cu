// gemm_simt.cu — exact-float32 SIMT GEMM with the fused epilogues.
//
// Serves the float32 storage type, whose parity bar (max relative error
// 1e-5 against the float64 oracle) rules out TF32 tensor cores: every product
// is an IEEE float32 FMA.  64x64 output tiles, K in steps of 16 staged in
// shared memory, 256 threads with 2 rows x 8 columns each.
#include "epilogue.cuh"
#include "kernels.h"
#include "profile.h"

namespace tlp {

namespace {

constexpr int BM = 64, BN = 64, BK = 16;

template <typename T>
__device__ __forceinline__ void load_tile(float (*dst)[BM + 4], const T* src, int ld, bool kmajor, int r0, int k0,
                                          int R, int K, int tid) {
  // dst[k][r] = src(r0 + r, k0 + k), zero outside the matrix
#pragma unroll
  for (int i = 0; i < (BM * BK) / 256; ++i) {
    const int idx = tid + i * 256;
    int r, k;
    if (kmajor) { r = idx / BK; k = idx % BK; } else { k = idx / BM; r = idx % BM; }
    const int gr = r0 + r, gk = k0 + k;
    float v = 0.0f;
    if (gr < R && gk < K) v = to_f(kmajor ? src[(size_t)gr * ld + gk] : src[(size_t)gk * ld + gr]);
    dst[k][r] = v;
  }
}

template <typename T, int KIND>
__global__ void __launch_bounds__(256) gemm_simt_kernel(GemmDesc g, EpiParams e) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  const int tid = threadIdx.x;
  const int tx = tid % 8, ty = tid / 8;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  const T* A = static_cast<const T*>(g.A);
  const T* B = static_cast<const T*>(g.B);
  float acc[2][8];
#pragma unroll
  for (int r = 0; r < 2; ++r)
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[r][c] = 0.0f;

  for (int k0 = 0; k0 < g.K; k0 += BK) {
    load_tile<T>(As, A, g.lda, g.a_kmajor, m0, k0, g.M, g.K, tid);
    load_tile<T>(Bs, B, g.ldb, g.b_kmajor, n0, k0, g.N, g.K, tid);
    __syncthreads();
#pragma unroll
    for (int k = 0; k < BK; ++k) {
      const float a0 = As[k][ty * 2], a1 = As[k][ty * 2 + 1];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const float b = Bs[k][tx * 8 + c];
        acc[0][c] = fmaf(a0, b, acc[0][c]);
        acc[1][c] = fmaf(a1, b, acc[1][c]);
      }
    }
    __syncthreads();
  }
  const int n = n0 + tx * 8;
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int m = m0 + ty * 2 + r;
    if (m < g.M && n < g.N) epi_apply8<T, KIND>(e, m, n, acc[r]);
  }
}

template <typename T>
void launch(const GemmDesc& g, const EpiParams& e, cudaStream_t s) {
  dim3 grid((g.N + BN - 1) / BN, (g.M + BM - 1) / BM);
  switch (e.kind) {
    case EPI_QKV: gemm_simt_kernel<T, EPI_QKV><<<grid, 256, 0, s>>>(g, e); break;
    case EPI_BIAS_DROP_RES: gemm_simt_kernel<T, EPI_BIAS_DROP_RES><<<grid, 256, 0, s>>>(g, e); break;
    case EPI_BIAS_GELU:
      if (e.gelu_tanh) gemm_simt_kernel<T, EPI_BIAS_GELU | EPI_TANH><<<grid, 256, 0, s>>>(g, e);
      else gemm_simt_kernel<T, EPI_BIAS_GELU><<<grid, 256, 0, s>>>(g, e);
      break;
    case EPI_DGELU:
      if (e.gelu_tanh) gemm_simt_kernel<T, EPI_DGELU | EPI_TANH><<<grid, 256, 0, s>>>(g, e);
      else gemm_simt_kernel<T, EPI_DGELU><<<grid, 256, 0, s>>>(g, e);
      break;
    case EPI_BIAS_GELU_D:
      if (e.gelu_tanh) gemm_simt_kernel<T, EPI_BIAS_GELU_D | EPI_TANH><<<grid, 256, 0, s>>>(g, e);
      else gemm_simt_kernel<T, EPI_BIAS_GELU_D><<<grid, 256, 0, s>>>(g, e);
      break;
    case EPI_MUL: gemm_simt_kernel<T, EPI_MUL><<<grid, 256, 0, s>>>(g, e); break;
    case EPI_STORE: gemm_simt_kernel<T, EPI_STORE><<<grid, 256, 0, s>>>(g, e); break;
    case EPI_F32: gemm_simt_kernel<T, EPI_F32><<<grid, 256, 0, s>>>(g, e); break;
  }
  count_launch();
}

}  // namespace

void gemm_simt_run(int dtype, const GemmDesc& g, const EpiParams& e, cudaStream_t s) {
  if (dtype == DT_F32) launch<float>(g, e, s);
  else if (dtype == DT_F16) launch<half_t>(g, e, s);
  else launch<bf16_t>(g, e, s);
}

}  // namespace tlp
