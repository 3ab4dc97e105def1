// noalloc.cu — bias-gradient column sum that allocates no device memory.
//
// Some callers cannot call cudaMalloc: their device memory is owned by
// someone else (a framework's caching allocator or a fixed per-process
// budget), or they run inside a stream capture in global mode, where
// allocation is not permitted.  tl_bias_grad_noalloc serves them: the
// partial column sums it needs live in the file-scope array below, which
// every GPU that loads this library holds (2 MiB) until the process exits.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/tlp.h"
#include "kernels.h"

namespace tlp {
namespace {

constexpr int kMaxCols = 8192;
constexpr int kMaxParts = 64;   // >= colsum_parts(rows) for any row count

// Partial column sums, (parts, cols) float32; overwritten by every call.
static __device__ __align__(256) float g_colsum_scratch[kMaxParts * kMaxCols];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
// Per device: the array's device address and the context it was looked up
// in.  A device reset (or any new primary context) gives the module a new
// address, so the address is looked up again when the current context is
// not the one it was taken in.
float* g_scratch_addr[kMaxDevices] = {};
CUcontext g_scratch_ctx[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

CUcontext current_context() {
  static CtxGetCurrentFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  }
  CUcontext c = nullptr;
  if (fn) fn(&c);
  return c;
}

// Device address of the scratch array on the current device (the host-side
// symbol is not a device address).
cudaError_t scratch_address(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_mu);
  const CUcontext ctx = current_context();
  if (!g_scratch_addr[dev] || ctx != g_scratch_ctx[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_colsum_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = static_cast<float*>(p);
    g_scratch_ctx[dev] = ctx;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace tlp

using namespace tlp;

extern "C" tl_status tl_bias_grad_noalloc(int dtype, const void* dz, int rows, int cols, float* db, void* stream) {
  if (dtype < TL_F32 || dtype > TL_BF16 || !dz || !db || rows <= 0 || cols <= 0) return TL_EINVAL;
  if (cols > kMaxCols || cols % 8 != 0) return TL_EINVAL;
  if ((reinterpret_cast<uintptr_t>(dz) & 15) || (reinterpret_cast<uintptr_t>(db) & 15)) return TL_EINVAL;
  const int parts = colsum_parts(rows);
  if (parts > kMaxParts) return TL_EINVAL;
  // an error left pending by an earlier, unrelated call is reported here
  // (and cleared) rather than blamed on this call's launches
  if (cudaGetLastError() != cudaSuccess) return TL_ECUDA;
  float* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return TL_ECUDA;
  // every partial row the finalize step reads is written by the first kernel,
  // so the array needs no clearing between calls
  colsum_run(dtype, dz, rows, cols, scratch, (cudaStream_t)stream);
  if (cudaPeekAtLastError() != cudaSuccess) return TL_ECUDA;
  colsum_finalize_run(scratch, parts, cols, db, (cudaStream_t)stream);
  return cudaPeekAtLastError() == cudaSuccess ? TL_OK : TL_ECUDA;
}
