// common.cuh -- device helpers shared by the CSA2 kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/csa2.h"

namespace csa2 {

constexpr int kBlock = 8;  // positions per indexer block (the pages' 8-position blocks)

// ---------------------------------------------------------------- status word
// First error wins; later errors are dropped so the first cause is reported.
__device__ __forceinline__ void set_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// ---------------------------------------------------------------- formats
// E4M3 ("FN": bias 7, max 448) byte -> fp32, exact.  NaN code is not produced
// by the quantiser; a stored 0x7F/0xFF decodes as 480 (harmless, finite).
__device__ __forceinline__ float e4m3_to_f32(uint32_t b) {
  uint32_t e = (b >> 3) & 15u, m = b & 7u;
  float v = e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : (float)m * 0.001953125f;
  return (b & 0x80u) ? -v : v;
}

// E2M1 nibble -> fp32, exact: magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}
__device__ __forceinline__ float e2m1_to_f32(uint32_t nib) {
  uint32_t i = nib & 7u;
  uint32_t e = i >> 1, m = i & 1u;
  float v = e ? __uint_as_float(((e + 126u) << 23) | (m << 22)) : (m ? 0.5f : 0.0f);
  return (nib & 8u) ? -v : v;
}

// ---------------------------------------------------------------- cache rows
__device__ __forceinline__ int64_t cache_row(const csa2_fp4_cache& c, int b, int64_t t) {
  if (c.page_table) {
    int32_t pg = __ldg(c.page_table + (int64_t)b * c.max_pages + t / c.page_size);
    return (int64_t)pg * c.page_size + t % c.page_size;
  }
  return __ldg(c.seq_base + b) + t;
}

// ---------------------------------------------------------------- timing / waits
__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------- overlapped launches
// A kernel of the decode step is launched with programmatic stream
// serialisation, so that its CTAs can be placed, and can set up their shared
// memory, barriers and tensor memory, while the previous kernel on the stream
// still runs. grid_dep_wait() returns once that kernel has completed and its
// writes are visible (at once when the launch had no such predecessor); every
// thread calls it before its first read or write of global memory.
// grid_dep_launch() lets the next kernel's CTAs be placed; a kernel calls it
// after its own wait, and so after its tensor-memory allocation: a placed
// dependant can then never hold tensor memory that a CTA of an earlier
// kernel still has to allocate. The persistent scoring kernels and attention
// call it when their CTA's work is done (measured faster than at the start:
// the dependants are placed on the SMs the tail frees).
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait with a suspend-time hint: the thread is parked (issuing nothing)
// until the phase completes or about `hint_ns` have passed
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Waits for the phase with the given parity to complete; gives up after
// about limit_ns and returns false (the caller records CSA2_ERR_TIMEOUT).
// Waiting threads are suspended by the hardware between probes (they take no
// issue slots from the warps doing work).  The global timer is read only
// every 64th probe: its reads go through a narrow pipe that a few dozen
// waiting warps reading it on every probe would saturate.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = 0;
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait_sleep(bar, parity, 1000000u)) return true;
    if ((i & 63) == 0) {
      const uint64_t now = globaltimer_ns();
      if (i == 64)
        t0 = now;
      else if (now - t0 > limit_ns)
        return false;
    }
  }
}

// Named barrier `id` over `n` threads (multiple of 32) that also returns the
// AND of `pred` over them.
__device__ __forceinline__ bool named_sync_and(uint32_t id, uint32_t n, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "barrier.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

// Group-wide wait: one thread of the group (`leader`) probes the mbarrier,
// the others are parked on the named barrier `id` (hardware barriers take no
// issue slots and no probe bandwidth); every thread gets the result.  With
// `skip` the leader does not probe and the group gets false.
__device__ __forceinline__ bool mbar_wait_group(uint32_t bar, uint32_t parity, uint64_t limit_ns, bool leader,
                                                bool skip, uint32_t id, uint32_t n) {
  bool ok = true;
  if (leader) ok = !skip && mbar_wait_bounded(bar, parity, limit_ns);
  return named_sync_and(id, n, ok);
}

// Warp-wide wait: only lane 0 probes the barrier (the other lanes are parked
// at the shuffle and take no issue slots); every lane gets the result.
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait_bounded(bar, parity, limit_ns);
  return __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
}

// ---------------------------------------------------------------- reductions
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// exclusive prefix sum over the threads of a CTA (blockDim.x <= 1024, multiple
// of 32); `scratch` holds 32 ints; returns the exclusive prefix, *total = sum
__device__ __forceinline__ int block_exclusive_scan(int v, int* scratch, int* total) {
  int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  __syncthreads();
  if (lane == 31) scratch[wid] = x;
  __syncthreads();
  if (wid == 0) {
    int s = lane < nw ? scratch[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    scratch[lane] = s;  // inclusive over warps
  }
  __syncthreads();
  int warp_before = wid ? scratch[wid - 1] : 0;
  *total = scratch[nw - 1];
  return warp_before + x - v;
}

// key counts that seed a selection: bins of the top 12 key bits
constexpr int kHistBins = 4096;
constexpr int kHistShift = 20;

// order-preserving map of a score to an unsigned key; invalid (-inf marker)
// entries map to 0, below every finite score
__device__ __forceinline__ uint32_t score_key(float f) {
  if (f == -INFINITY || f != f) return 0u;
  uint32_t u = __float_as_uint(f + 0.0f);  // -0 -> +0: equal scores get equal keys
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

}  // namespace csa2
