// dispatch.cu — picks the kernel family that serves each dtype: the tcgen05
// tensor-core GEMM for 16-bit storage, the exact-float32 SIMT GEMM for float32.
#include "kernels.h"

namespace tlp {

void gemm_simt_run(int dtype, const GemmDesc& g, const EpiParams& e, cudaStream_t s);
int gemm_tc_run(int dtype, const GemmDesc& g, const EpiParams& e, cudaStream_t s);
int gemm_tc_run2(int dtype, const GemmDesc& ga, const EpiParams& ea, const GemmDesc& gb, const EpiParams& eb,
                 cudaStream_t s);
size_t gemm_tc_splitk_ws_floats(int M, int N, int K);
int gemm_tc_take_error();

int gemm_uses_tensor_cores(int dtype) { return dtype != DT_F32; }

int gemm_run(int dtype, const GemmDesc& g, const EpiParams& e, cudaStream_t s) {
  if (dtype == DT_F32) {
    gemm_simt_run(dtype, g, e, s);
    return 0;
  }
  return gemm_tc_run(dtype, g, e, s);
}

int gemm_run2(int dtype, const GemmDesc& ga, const EpiParams& ea, const GemmDesc& gb, const EpiParams& eb,
              cudaStream_t s) {
  if (dtype == DT_F32) {
    gemm_simt_run(dtype, ga, ea, s);
    gemm_simt_run(dtype, gb, eb, s);
    return 0;
  }
  return gemm_tc_run2(dtype, ga, ea, gb, eb, s);
}

size_t gemm_splitk_ws_floats(int dtype, int M, int N, int K) {
  return dtype == DT_F32 ? 0 : gemm_tc_splitk_ws_floats(M, N, K);
}

int attn_tc_take_error();
int rowwise_take_error();
void gemm_tc_set_wait_limit(uint64_t ns);
void attn_tc_set_wait_limit(uint64_t ns);
void rowwise_set_wait_limit(uint64_t ns);

void device_set_wait_limit(uint64_t ns) {
  gemm_tc_set_wait_limit(ns);
  attn_tc_set_wait_limit(ns);
  rowwise_set_wait_limit(ns);
}

int device_take_error() {
  const int g = gemm_tc_take_error();
  const int a = attn_tc_take_error();
  const int r = rowwise_take_error();
  return g ? g : (a ? a : r);
}

}  // namespace tlp
