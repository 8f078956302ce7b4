// noalloc.cu -- csa2_index_reindex_noalloc: the Reindex call without a
// caller-provided workspace.
//
// Some callers cannot allocate device memory and cannot hand the library a
// workspace either: a serving engine that reserves all device memory for its
// KV pool at start-up and forbids later allocations, or a plug-in interface
// whose operator signature has no workspace argument.  For them this entry
// point keeps its scratch (the rescored pool positions, one fp32 per
// candidate) in a fixed file-scope device array that every GPU which loads the
// library holds until the process exits.  The call allocates nothing: no
// cudaMalloc, no cudaFree, no allocating library routine.
#include "common.cuh"
#include "internal.h"

namespace csa2 {

// fixed scratch: n_tok * P * 8 candidates at most (4 MiB)
constexpr int64_t kNoAllocScratchFloats = int64_t(1) << 20;
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats];

// device address of the array for the current device.  In host code the
// symbol is only a host-side stand-in, so the address is looked up with that
// device current, on every call: a cached address would go stale if the
// device were reset (a new context loads the module again at another
// address).  The lookup allocates nothing.
static float* noalloc_scratch_ptr(int* rc) {
  float* p = nullptr;
  *rc = cuda_check(cudaGetSymbolAddress((void**)&p, g_noalloc_scratch), "cudaGetSymbolAddress(scratch)");
  return *rc ? nullptr : p;
}

int check_index_args(const csa2_query_batch* qb, const uint8_t* qc, const uint8_t* qs, const float* w, int H_I,
                     const csa2_fp4_cache* kc, int P, int K);
int launch_rescore(const csa2_query_batch* qb, const uint8_t* qc, const uint8_t* qs, const float* w, int H,
                   const csa2_fp4_cache* kc, const int32_t* pool, const int32_t* pool_n, int P, float* scores,
                   cudaStream_t st);
int launch_select(const csa2_query_batch* qb, const float* score, int64_t ld, int mode, const int32_t* pool,
                  const int32_t* pool_n, int P, int k_out, int32_t* out, int32_t* out_n, cudaStream_t st);
void clear_last_error();

}  // namespace csa2

using namespace csa2;

extern "C" int csa2_index_reindex_noalloc(const csa2_query_batch* qb, const uint8_t* q_codes, const uint8_t* q_scales,
                                          const float* w, int32_t H_I, const csa2_fp4_cache* k_idx,
                                          const int32_t* pool, const int32_t* pool_n, int32_t P, int32_t K,
                                          int32_t* idx, int32_t* idx_n, void* stream) {
  clear_last_error();
  if (int rc = check_index_args(qb, q_codes, q_scales, w, H_I, k_idx, P, K)) return rc;
  if (!pool || !pool_n || !idx || !idx_n) return fail(CSA2_ERR_INVALID_ARG, "pool/idx buffers must be non-NULL");
  const int64_t need = (int64_t)qb->n_tok * P * kBlock;
  if (need > kNoAllocScratchFloats)
    return fail(CSA2_ERR_WORKSPACE,
                "n_tok * P * 8 = %lld exceeds the fixed scratch of %lld candidates (use csa2_index_reindex)",
                (long long)need, (long long)kNoAllocScratchFloats);
  int rc = CSA2_OK;
  float* scores = noalloc_scratch_ptr(&rc);
  if (rc) return rc;
  // The rescoring kernel writes every candidate slot the selection reads
  // (-inf where a slot holds no visible position), so nothing left in the
  // array by an earlier call is ever read: no clearing is needed.
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (int r = launch_rescore(qb, q_codes, q_scales, w, H_I, k_idx, pool, pool_n, P, scores, st)) return r;
  // no selection scratch either: one CTA per query token, with its own
  // histogram rounds over the scores
  return launch_select(qb, scores, (int64_t)P * kBlock, 1, pool, pool_n, P, K, idx, idx_n, st);
}
