// Device side of the synthetic input generator (see csa2_synth.h).  Fills
// caller-owned device buffers; bit-identical to synth_host.c.
#include "csa2_synth.h"
#include <cuda_runtime.h>

namespace {

__global__ void k_fill_f32(syn_tensor t, uint32_t row_hi, int64_t pos0, int64_t n, float* out) {
  int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  int64_t total = n * t.dim;
  for (; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    int64_t i = e / t.dim;
    int32_t c = (int32_t)(e - i * t.dim);
    int64_t pos = pos0 + i;
    uint64_t rk = syn_row_key(t.seed, t.stream, syn_row_id(row_hi, pos));
    int nd = syn_is_needle(&t, row_hi, pos);
    out[e] = syn_value(&t, rk, row_hi, pos, c, nd);
  }
}

__global__ void k_fill_bf16(syn_tensor t, uint32_t row_hi, int64_t pos0, int64_t n, uint16_t* out) {
  int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  int64_t total = n * t.dim;
  for (; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    int64_t i = e / t.dim;
    int32_t c = (int32_t)(e - i * t.dim);
    int64_t pos = pos0 + i;
    uint64_t rk = syn_row_key(t.seed, t.stream, syn_row_id(row_hi, pos));
    int nd = syn_is_needle(&t, row_hi, pos);
    out[e] = syn_bf16_rne(syn_value(&t, rk, row_hi, pos, c, nd));
  }
}

// one warp per row
__global__ void k_fill_e4m3(syn_tensor t, uint32_t row_hi, int64_t pos0, int64_t n, int64_t ring,
                            uint8_t* codes, float* scale) {
  int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  int lane = threadIdx.x & 31;
  for (; warp < n; warp += ((int64_t)gridDim.x * blockDim.x) >> 5) {
    int64_t pos = pos0 + warp;
    int64_t slot = ring > 0 ? pos % ring : warp;
    uint64_t rk = syn_row_key(t.seed, t.stream, syn_row_id(row_hi, pos));
    int nd = syn_is_needle(&t, row_hi, pos);
    float amax = 0.0f;
    for (int32_t c = lane; c < t.dim; c += 32) amax = fmaxf(amax, fabsf(syn_value(&t, rk, row_hi, pos, c, nd)));
    for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    float s = amax > 0.0f ? syn_div(amax, 448.0f) : 1.0f;
    if (lane == 0) scale[slot] = s;
    for (int32_t c = lane; c < t.dim; c += 32)
      codes[slot * t.dim + c] = syn_e4m3_code(syn_div(syn_value(&t, rk, row_hi, pos, c, nd), s));
  }
}

int grid_for(int64_t work) {
  int64_t g = (work + 255) / 256;
  if (g > 148 * 16) g = 148 * 16;
  if (g < 1) g = 1;
  return (int)g;
}

}  // namespace

extern "C" {

int syn_dev_fill_f32(const syn_tensor* t, uint32_t row_hi, int64_t pos0, int64_t n, float* out, void* stream) {
  if (n <= 0) return 0;
  k_fill_f32<<<grid_for(n * t->dim), 256, 0, (cudaStream_t)stream>>>(*t, row_hi, pos0, n, out);
  return (int)cudaGetLastError();
}

int syn_dev_fill_bf16(const syn_tensor* t, uint32_t row_hi, int64_t pos0, int64_t n, uint16_t* out, void* stream) {
  if (n <= 0) return 0;
  k_fill_bf16<<<grid_for(n * t->dim), 256, 0, (cudaStream_t)stream>>>(*t, row_hi, pos0, n, out);
  return (int)cudaGetLastError();
}

int syn_dev_fill_e4m3(const syn_tensor* t, uint32_t row_hi, int64_t pos0, int64_t n, int64_t ring,
                      uint8_t* codes, float* scale, void* stream) {
  if (n <= 0) return 0;
  k_fill_e4m3<<<grid_for(n * 32), 256, 0, (cudaStream_t)stream>>>(*t, row_hi, pos0, n, ring, codes, scale);
  return (int)cudaGetLastError();
}

}  // extern "C"
