// peak.cu -- tensor-core peak probe: the dense MMA rate this GPU sustains for
// the two instruction kinds the decode path uses, so that the rooflines of
// the scan and rescoring (block-scaled FP4) and of attention (fp16) are
// measured fractions rather than datasheet ratios.
//
// One CTA per SM; two threads (of different warps) each issue back-to-back
// M = 128, N = 256 MMAs from fixed shared-memory operands into their own
// TMEM accumulators, then wait for completion (bounded).  FLOP = 2 M N K per
// MMA (K = 64 for kind::mxf4nvf4, 16 for kind::f16).  Operand values are
// fixed, finite and non-zero; the result is discarded.
#include "internal.h"
#include "tc_common.cuh"

namespace csa2 {
namespace peak {

constexpr int kThreads = 64;
constexpr uint32_t kSmem = 116 * 1024;  // above half an SM's shared memory: one CTA per SM

__global__ void __launch_bounds__(kThreads, 1) k_peak(int fp4, int iters, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  // A [128 rows] at 0, B [256 rows] at 32 KB, scale factors at 64 KB, barriers at 68 KB
  const uint32_t bar = sb + 69632;
  __shared__ uint32_t tmem_h;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // fp16 1/64, E2M1 code 1.0, E4M3 scale 1.0
  for (int i = threadIdx.x; i < 65536 / 4; i += kThreads)
    reinterpret_cast<uint32_t*>(smem)[i] = fp4 ? 0x22222222u : 0x24002400u;
  for (int i = threadIdx.x; i < 4096 / 4; i += kThreads) reinterpret_cast<uint32_t*>(smem + 65536)[i] = 0x38383838u;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 3; ++i) mbar_init(bar + 8 * i, 1);
    tc::fence_barrier_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(smem_u32(&tmem_h), 512);
    tc::tmem_relinquish();
    tc::fence_before_sync();
  }
  tc::fence_proxy_async_smem();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_h;
  bool ok = true;
  if (threadIdx.x == 0 && fp4) {  // scale factors: columns 256..271 of TMEM (A, B)
    for (int c = 0; c < 4; ++c)
      tc::cp_32x128b_warpx4(tmem + 256 + c * 4, tc::smem_desc(sb + 65536 + c * 512, 16, 128, tc::kSwizzleNone));
    tc::commit(bar + 16);
    ok = mbar_wait_bounded(bar + 16, 0, 1000000000ull);
  }
  __syncthreads();
  tc::fence_after_sync();
  if (lane == 0 && ok) {
    // both threads accumulate into columns 0..255 (the values are discarded)
    const uint32_t d = tmem;
    uint64_t ad, bd;
    uint32_t idesc;
    if (fp4) {
      idesc = tc::idesc_mxf4nvf4(128, 256);
      ad = tc::smem_desc(sb + warp * 16384, 16, 512, tc::kSwizzle64B);
      bd = tc::smem_desc(sb + 32768, 16, 512, tc::kSwizzle64B);
    } else {
      idesc = tc::idesc_f16(128, 256, 0, 0);
      ad = tc::smem_desc(sb + warp * 16384, 16, 1024, tc::kSwizzle128B);
      bd = tc::smem_desc(sb + 32768, 16, 1024, tc::kSwizzle128B);
    }
    for (int i = 0; i < iters; ++i) {
      if (fp4)
        tc::mma_mxf4nvf4(d, ad, bd, idesc, tmem + 256, tmem + 264, i > 0 ? 1u : 0u);
      else
        tc::mma_f16(d, ad, bd, idesc, i > 0 ? 1u : 0u);
    }
    tc::commit(bar + 8 * warp);
    if (!mbar_wait_bounded(bar + 8 * warp, 0, 2000000000ull)) set_status(status, CSA2_ERR_TIMEOUT);
  }
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

}  // namespace peak
}  // namespace csa2

using namespace csa2;

extern "C" int csa2_tensor_peak(int32_t kind, int32_t iters, double* tflops, void* stream) {
  if (!tflops || iters < 16 || iters > (1 << 20) || (kind != 0 && kind != 1))
    return fail(CSA2_ERR_INVALID_ARG, "kind must be 0 (fp16) or 1 (FP4), iters in [16, 2^20]");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int dev = 0, sms = 0;
  if (int rc = cuda_check(cudaGetDevice(&dev), "cudaGetDevice")) return rc;
  if (int rc = cuda_check(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev), "SM count")) return rc;
  if (int rc = cuda_check(cudaFuncSetAttribute(peak::k_peak, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)peak::kSmem),
                          "peak smem attribute"))
    return rc;
  cudaEvent_t a = nullptr, b = nullptr;
  if (int rc = cuda_check(cudaEventCreate(&a), "event")) return rc;
  if (int rc = cuda_check(cudaEventCreate(&b), "event")) {
    cudaEventDestroy(a);
    return rc;
  }
  int rc = CSA2_OK;
  float best = 0.0f;
  for (int rep = 0; rep < 3 && rc == CSA2_OK; ++rep) {  // the first run warms the clocks up
    cudaEventRecord(a, st);
    {
      Launch L_("tensor_peak", st);
      peak::k_peak<<<sms, peak::kThreads, peak::kSmem, st>>>(kind, iters, status_ptr());
    }
    cudaEventRecord(b, st);
    rc = cuda_check(cudaEventSynchronize(b), "peak kernel");
    float ms = 0.0f;
    if (rc == CSA2_OK) rc = cuda_check(cudaEventElapsedTime(&ms, a, b), "peak timing");
    if (rc == CSA2_OK && rep > 0 && (best == 0.0f || ms < best)) best = ms;
  }
  cudaEventDestroy(a);
  cudaEventDestroy(b);
  if (rc) return rc;
  const double k = kind == 1 ? 64.0 : 16.0;
  const double flop = 2.0 * 128.0 * 256.0 * k * iters * 2.0 * sms;  // two issuing threads per CTA
  *tflops = flop / (best * 1e-3) / 1e12;
  return CSA2_OK;
}
