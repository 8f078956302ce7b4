// internal.h -- declarations shared by the host-side translation units of libcsa2.so.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/csa2.h"

namespace csa2 {

int fail(int code, const char* fmt, ...);
int cuda_check(cudaError_t e, const char* what);
int* status_ptr();

int launch_scan_tc(const csa2_query_batch* qb, const uint8_t* qc, const uint8_t* qs, const float* w, int H,
                   const csa2_fp4_cache* kc, float* bs, int64_t ld, cudaStream_t st);

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
