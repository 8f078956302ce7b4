// internal.h -- declarations shared by the host-side translation units of libcsa2.so.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/csa2.h"

namespace csa2 {

int fail(int code, const char* fmt, ...);
int cuda_check(cudaError_t e, const char* what);
int* status_ptr();

// hist: per (selector, token) group, counts of the stored scores' keys by
// their top 12 bits (4096 bins, zeroed before the launch), or NULL
int launch_scan_tc(const csa2_query_batch* qb, const uint8_t* qc, const uint8_t* qs, const float* w, int H,
                   const csa2_fp4_cache* kc, float* bs, int64_t ld, uint32_t* hist, cudaStream_t st);

int launch_rescore_tc(const csa2_query_batch* qb, const uint8_t* qc, const uint8_t* qs, const float* const* w,
                      int n_sel, int H, const csa2_fp4_cache* kc, const int32_t* pool, const int32_t* pool_n, int P,
                      float* scores, uint32_t* hist, cudaStream_t st);
bool attend_tc_supported(int D, int Hq, int q_dtype);
// one layer of a multi-layer attention launch
struct AttendLayer {
  const int32_t* idx;    // [T][K] positions chosen by this layer's selector
  const int32_t* idx_n;  // [T]
  const void* q;
  void* out;
  float* lse;
  const csa2_swa_desc* swa;
};
constexpr int kMaxAttLayers = 32;  // layers per attention launch
constexpr int kMaxSel = 8;         // selector layers per rescoring launch
struct SelGroup;
int launch_attend_tc(const csa2_query_batch* qb, int q_dtype, int Hq, const csa2_fp4_cache* kv, int K,
                     const AttendLayer* layers, int n_layers, float scale, int out_dtype, float* part_o,
                     float* part_ml, int* done, int nsplit, cudaStream_t st);

// Launch bookkeeping: counts every kernel launch and, while the profiler is
// enabled, brackets it with CUDA events on its stream.
struct Launch {
  Launch(const char* name, cudaStream_t st);
  ~Launch();
  const char* name;
  cudaStream_t st;
  int slot;
};

// Overlapped launches (programmatic stream serialisation) by kernel kind:
// the quantiser, the scan and attention by default. The selections launch
// plainly (overlapped, they made every decode workload slower), and so does
// the rescoring (faster at four tokens of 1M context and at chunked
// prefill, slower at the four other workloads). The environment variable
// CSA2_OVERLAP, a mask of the kinds below, overrides the default (0: none).
// Every kernel launched this way calls grid_dep_wait() before it touches
// global memory.
enum { kOverlapQuantize = 1, kOverlapScan = 2, kOverlapRescore = 4, kOverlapSelect = 8, kOverlapAttend = 16 };
bool overlap_launches(int kind);
template <typename... KArgs, typename... Args>
cudaError_t launch_overlapped(int kind, void (*k)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args... args) {
  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute at[1];
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = overlap_launches(kind) ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, k, args...);
}

}  // namespace csa2
