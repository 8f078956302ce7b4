/* Host side of the synthetic input generator (see csa2_synth.h). */
#include "csa2_synth.h"
#include <math.h>
#include <stddef.h>

/* rows (row_hi, pos0 .. pos0+n-1) of tensor t as fp32, out[n][dim] */
void syn_host_fill_f32(const syn_tensor* t, uint32_t row_hi, int64_t pos0, int64_t n, float* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    int64_t pos = pos0 + i;
    uint64_t rk = syn_row_key(t->seed, t->stream, syn_row_id(row_hi, pos));
    int nd = syn_is_needle(t, row_hi, pos);
    for (int32_t c = 0; c < t->dim; ++c)
      out[i * t->dim + c] = syn_value(t, rk, row_hi, pos, c, nd);
  }
}

/* selected rows only: positions pos[i] of sequence row_hi */
void syn_host_fill_rows_f32(const syn_tensor* t, uint32_t row_hi, const int64_t* pos, int64_t n, float* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    uint64_t rk = syn_row_key(t->seed, t->stream, syn_row_id(row_hi, pos[i]));
    int nd = syn_is_needle(t, row_hi, pos[i]);
    for (int32_t c = 0; c < t->dim; ++c)
      out[i * t->dim + c] = syn_value(t, rk, row_hi, pos[i], c, nd);
  }
}

/* same values rounded to bf16 (bits) */
void syn_host_fill_bf16(const syn_tensor* t, uint32_t row_hi, int64_t pos0, int64_t n, uint16_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    int64_t pos = pos0 + i;
    uint64_t rk = syn_row_key(t->seed, t->stream, syn_row_id(row_hi, pos));
    int nd = syn_is_needle(t, row_hi, pos);
    for (int32_t c = 0; c < t->dim; ++c)
      out[i * t->dim + c] = syn_bf16_rne(syn_value(t, rk, row_hi, pos, c, nd));
  }
}

/* FP8 rows: per-row scale = amax/448 (1 if the row is zero), codes = E4M3 of
 * value/scale.  Row for position p goes to slot p % ring (ring = n for a
 * dense output). */
void syn_host_fill_e4m3(const syn_tensor* t, uint32_t row_hi, int64_t pos0, int64_t n,
                        int64_t ring, uint8_t* codes, float* scale) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    int64_t pos = pos0 + i;
    int64_t slot = ring > 0 ? pos % ring : i;
    uint64_t rk = syn_row_key(t->seed, t->stream, syn_row_id(row_hi, pos));
    int nd = syn_is_needle(t, row_hi, pos);
    float amax = 0.0f;
    for (int32_t c = 0; c < t->dim; ++c) {
      float v = syn_value(t, rk, row_hi, pos, c, nd);
      float a = v < 0.0f ? -v : v;
      if (a > amax) amax = a;
    }
    float s = amax > 0.0f ? syn_div(amax, 448.0f) : 1.0f;
    scale[slot] = s;
    for (int32_t c = 0; c < t->dim; ++c)
      codes[slot * t->dim + c] = syn_e4m3_code(syn_div(syn_value(t, rk, row_hi, pos, c, nd), s));
  }
}

uint8_t syn_host_e4m3_code(float f) { return syn_e4m3_code(f); }
uint16_t syn_host_bf16(float f) { return syn_bf16_rne(f); }
float syn_host_normal(uint64_t seed, uint64_t stream, uint64_t row, uint64_t col) {
  return syn_normal(syn_elem_key(syn_row_key(seed, stream, row), col));
}
