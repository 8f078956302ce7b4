// internal.h -- declarations shared by the host-side translation units of libcsa2.so.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/csa2.h"

namespace csa2 {

int fail(int code, const char* fmt, ...);
int cuda_check(cudaError_t e, const char* what);
int* status_ptr();

// Launch bookkeeping: counts every kernel launch and, while the profiler is
// enabled, brackets it with CUDA events on its stream.
struct Launch {
  Launch(const char* name, cudaStream_t st);
  ~Launch();
  const char* name;
  cudaStream_t st;
  int slot;
};

}  // namespace csa2
