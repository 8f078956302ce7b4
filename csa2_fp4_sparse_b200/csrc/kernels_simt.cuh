// kernels_simt.cuh -- the CUDA-core kernels of the CSA2 decode step: the FP4
// quantiser, the stack's index-list copies and the bounded-wait self test.
#pragma once

#include "common.cuh"

namespace csa2 {

// ============================================================================
// K1: FP4 quantiser.  One thread = 8 consecutive elements, 4 threads = one
// 32-element group.  scale = E4M3_rne_satfinite(amax / 6) (one fp32 RN
// division); codes = round-to-nearest-even of the exact |x|/scale on the E2M1
// grid, found by comparing |x| with scale * {.25,.75,1.25,1.75,2.5,3.5,5}
// (products exact in fp32), ties to the even code.
// ============================================================================
// Quantisation jobs of one launch: each a row-major fp32 matrix [rows][dim]
// written as codes [row][dim/2] + scales [row][dim/32], rows remapped through
// `slot` when given (cache append).  A thread takes 8 consecutive elements
// ("unit"); job j owns units [begin[j], begin[j+1]), multiples of 4, so the 4
// threads of a 32-element scale group never straddle two jobs.
constexpr int kQuantJobs = 12;
struct QuantJob {
  const float* x;
  const int64_t* slot;
  uint8_t* codes;
  uint8_t* scales;
  int dim;
};
struct QuantJobs {
  QuantJob job[kQuantJobs];
  int64_t begin[kQuantJobs + 1];
  int n;
};

__global__ void __launch_bounds__(256) k_quantize_fp4(const __grid_constant__ QuantJobs J, int* status) {
  grid_dep_wait();
  grid_dep_launch();
  const int64_t total = J.begin[J.n];
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t base = (int64_t)blockIdx.x * blockDim.x; base < total; base += stride) {
    int64_t i = base + threadIdx.x;
    bool active = i < total;
    float v[8];
    float amax = 0.0f;
    bool bad = false;
    int64_t r = 0, c8 = 0;
    int jb = 0;
    if (active) {
      while (jb + 1 < J.n && i >= J.begin[jb + 1]) ++jb;
      const int64_t per_row = J.job[jb].dim / 8;
      const int64_t li = i - J.begin[jb];
      r = li / per_row;
      c8 = li - r * per_row;
      const float4* xp = reinterpret_cast<const float4*>(J.job[jb].x + r * J.job[jb].dim + c8 * 8);
      float4 a = __ldg(xp), b = __ldg(xp + 1);
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
      v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        float m = fabsf(v[k]);
        bad |= !(m <= 3.402823466e38f);
        amax = fmaxf(amax, m);
      }
    }
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    int badq = __shfl_xor_sync(0xffffffffu, (int)bad, 1) | (int)bad;
    badq |= __shfl_xor_sync(0xffffffffu, badq, 2);
    if (!active) continue;
    const QuantJob& jo = J.job[jb];
    const int dim = jo.dim;
    int64_t orow = jo.slot ? __ldg(jo.slot + r) : r;
    uint32_t packed = 0;
    uint8_t sc = 0;
    if (!badq) {
      float q = __fdiv_rn(amax, 6.0f);
      sc = (uint8_t)__nv_cvt_float_to_fp8(q, __NV_SATFINITE, __NV_E4M3);
      float s = e4m3_to_f32(sc);
      const float t0 = s * 0.25f, t1 = s * 0.75f, t2 = s * 1.25f, t3 = s * 1.75f, t4 = s * 2.5f,
                  t5 = s * 3.5f, t6 = s * 5.0f;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        float a = fabsf(v[k]);
        uint32_t idx = (uint32_t)(a > t0) + (uint32_t)(a >= t1) + (uint32_t)(a > t2) + (uint32_t)(a >= t3) +
                       (uint32_t)(a > t4) + (uint32_t)(a >= t5) + (uint32_t)(a > t6);
        if (s == 0.0f) idx = 0;
        uint32_t nib = idx | ((__float_as_uint(v[k]) >> 28) & 8u);
        packed |= nib << (4 * k);
      }
    } else {
      set_status(status, CSA2_ERR_NONFINITE);
    }
    *reinterpret_cast<uint32_t*>(jo.codes + orow * (dim / 2) + c8 * 4) = packed;
    if ((c8 & 3) == 0) jo.scales[orow * (dim / 32) + c8 / 4] = sc;
  }
}

// copies used by the stack for the optional per-layer outputs
__global__ void k_copy_i32(const int32_t* __restrict__ src, int32_t* __restrict__ dst, int64_t n) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    dst[i] = src[i];
}

// bounded-wait self test: waits on an mbarrier that nothing completes
__global__ void k_selftest_wait(int64_t limit_ns, int* status) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    if (!mbar_wait_bounded(smem_u32(&bar), 0, (uint64_t)limit_ns)) set_status(status, CSA2_ERR_TIMEOUT);
  }
}

}  // namespace csa2
