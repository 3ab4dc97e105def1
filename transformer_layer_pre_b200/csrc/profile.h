// profile.h — launch counting and an opt-in per-launch CUDA-event timer.
#pragma once

#include <cuda_runtime.h>

namespace tlp {

enum ProfClass { PC_GEMM = 0, PC_ATTN_FWD, PC_ATTN_BWD, PC_LN_FWD, PC_LN_BWD, PC_ROWWISE, PC_COUNT };

// Adds n to the library's kernel-launch counter.
void count_launch(int n = 1);

// While profiling is enabled, brackets the launches of its lifetime with a
// pair of events on `s` and books the elapsed time to `cls`.
class ProfScope {
 public:
  ProfScope(int cls, cudaStream_t s);
  ~ProfScope();

 private:
  int slot_;
  cudaStream_t s_;
};

}  // namespace tlp
