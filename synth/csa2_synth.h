/*
 * csa2_synth.h -- seeded, counter-based synthetic input generator.
 *
 * This header is the whole definition of the synthetic inputs used by the
 * tests and the benchmark.  It is compiled twice: into a host library
 * (libsynth_host.so, plain C) and into a device library (libsynth_dev.so,
 * CUDA).  Both produce bit-identical values for the same (seed, stream, row,
 * col) because every step is integer arithmetic or a single IEEE-754
 * round-to-nearest operation (no fused multiply-add, no transcendental).
 *
 * It contains no arithmetic of the CSA2 method itself: no FP4 quantisation,
 * no scoring, no selection, no attention.  It only draws numbers.
 *
 *   entropy : SplitMix64 finaliser over a counter built from
 *             (seed, stream, row, col)
 *   N(0,1)  : Irwin-Hall sum of twelve 24-bit uniforms, (sum - 6*2^24)*2^-24,
 *             exact in int64, one round-to-nearest int->float conversion
 *   t(3)    : Z / sqrt((Z1^2 + Z2^2 + Z3^2) / 3), each op one IEEE RN op
 *   U[0,1)  : 24-bit uniform * 2^-24 (exact)
 *   bf16    : round-to-nearest-even of an fp32 bit pattern
 *   FP8     : an E4M3 code of an fp32 value (round-to-nearest-even of the
 *             exact value, saturating), used only to synthesise the FP8
 *             sliding-window KV, which the decode path takes as given.
 */
#ifndef CSA2_SYNTH_H
#define CSA2_SYNTH_H

#include <stdint.h>

#if defined(__CUDACC__)
#define SYN_FN __host__ __device__ __forceinline__
#else
#define SYN_FN static inline
#endif

/* stream ids: one per synthetic tensor kind; per-layer tensors add the layer */
enum {
  SYN_S_KIDX = 1,        /* indexer K source, row = (seq<<32)|pos, col = channel */
  SYN_S_KV = 2,          /* main KV latent source */
  SYN_S_IQ = 0x100,      /* + layer: indexer query, row = token, col = h*d_I+c */
  SYN_S_IW = 0x200,      /* + layer: indexer head weight, row = token, col = h */
  SYN_S_QMAIN = 0x300,   /* + layer: main query, row = token, col = h*D+c */
  SYN_S_SWA = 0x400,     /* + layer: SWA KV source, row = (seq<<32)|pos */
  SYN_S_SWASCALE = 0x500 /* + layer: SWA per-token scale exponent */
};

SYN_FN uint64_t syn_mix(uint64_t z) {
  z += 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

/* per-row key; every element of the row derives from it */
SYN_FN uint64_t syn_row_key(uint64_t seed, uint64_t stream, uint64_t row) {
  return syn_mix(syn_mix(syn_mix(seed) + stream) + row);
}

SYN_FN uint64_t syn_elem_key(uint64_t row_key, uint64_t col) {
  return syn_mix(row_key ^ (col * 0xD1B54A32D192ED03ull));
}

/* the i-th 64-bit draw of an element */
SYN_FN uint64_t syn_draw(uint64_t elem_key, uint32_t i) {
  return syn_mix(elem_key + (uint64_t)(i + 1) * 0x632BE59BD9B4E019ull);
}

SYN_FN float syn_i64_to_f32(int64_t v) {
#if defined(__CUDA_ARCH__)
  return __ll2float_rn(v);
#else
  return (float)v; /* cvtsi2ss: round to nearest under the default mode */
#endif
}

SYN_FN float syn_mul(float a, float b) {
#if defined(__CUDA_ARCH__)
  return __fmul_rn(a, b);
#else
  return a * b;
#endif
}
SYN_FN float syn_add(float a, float b) {
#if defined(__CUDA_ARCH__)
  return __fadd_rn(a, b);
#else
  return a + b;
#endif
}
SYN_FN float syn_div(float a, float b) {
#if defined(__CUDA_ARCH__)
  return __fdiv_rn(a, b);
#else
  return a / b;
#endif
}
SYN_FN float syn_sqrt(float a) {
#if defined(__CUDA_ARCH__)
  return __fsqrt_rn(a);
#else
  return __builtin_sqrtf(a);
#endif
}

/* Irwin-Hall N(0,1) from draws [first, first+6) (two 24-bit uniforms each) */
SYN_FN float syn_normal_at(uint64_t elem_key, uint32_t first) {
  int64_t sum = 0;
  for (uint32_t i = 0; i < 6; ++i) {
    uint64_t r = syn_draw(elem_key, first + i);
    sum += (int64_t)(r & 0xFFFFFFull) + (int64_t)((r >> 32) & 0xFFFFFFull);
  }
  /* (sum - 6*2^24) * 2^-24 ; the scale by 2^-24 is exact */
  return syn_mul(syn_i64_to_f32(sum - 100663296LL), 5.9604644775390625e-8f);
}

SYN_FN float syn_normal(uint64_t elem_key) { return syn_normal_at(elem_key, 0); }

/* Student t with 3 degrees of freedom from four independent normals */
SYN_FN float syn_t3(uint64_t elem_key) {
  float z = syn_normal_at(elem_key, 0);
  float z1 = syn_normal_at(elem_key, 6);
  float z2 = syn_normal_at(elem_key, 12);
  float z3 = syn_normal_at(elem_key, 18);
  float s = syn_add(syn_add(syn_mul(z1, z1), syn_mul(z2, z2)), syn_mul(z3, z3));
  s = syn_div(s, 3.0f);
  if (!(s > 0.0f)) return z;
  return syn_div(z, syn_sqrt(s));
}

/* U[0,1) with 24 bits */
SYN_FN float syn_uniform(uint64_t elem_key) {
  uint64_t r = syn_draw(elem_key, 0);
  return syn_mul(syn_i64_to_f32((int64_t)(r & 0xFFFFFFull)), 5.9604644775390625e-8f);
}

SYN_FN uint32_t syn_f32_bits(float f) {
  union { float f; uint32_t u; } v;
  v.f = f;
  return v.u;
}
SYN_FN float syn_bits_f32(uint32_t u) {
  union { float f; uint32_t u; } v;
  v.u = u;
  return v.f;
}

/* fp32 -> bf16 bits, round to nearest even (finite inputs) */
SYN_FN uint16_t syn_bf16_rne(float f) {
  uint32_t u = syn_f32_bits(f);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/* E4M3 (OCP "FN": bias 7, max 448, no infinities) code of a finite fp32 value,
 * round-to-nearest-even of the exact value, saturating at +-448.  Integer
 * only: the value is split into an integer significand and a power of two.  */
SYN_FN uint8_t syn_e4m3_code(float f) {
  uint32_t u = syn_f32_bits(f);
  uint8_t sign = (uint8_t)((u >> 31) << 7);
  uint32_t mag = u & 0x7FFFFFFFu;
  int32_t e = (int32_t)(mag >> 23);
  uint32_t m = mag & 0x7FFFFFu;
  if (e == 0) return sign; /* fp32 subnormals are far below the E4M3 range */
  /* |f| = (2^23 + m) * 2^(e - 150).  Express in units of 2^-9 (the E4M3
   * subnormal step) when below 2^-6, else in units of 2^(E-3) for the
   * E4M3 exponent E. */
  uint32_t sig = 0x800000u | m; /* 24-bit significand */
  int32_t E = e - 127;          /* unbiased exponent */
  int32_t shift;                /* right shift that brings sig to the code grid */
  if (E < -6) {
    /* grid step 2^-9: value/2^-9 = sig * 2^(E - 23 + 9) */
    shift = 23 - 9 - E;         /* >= 23-9+7 = 21 */
  } else {
    shift = 20;                 /* keep 3 mantissa bits */
  }
  uint32_t q;
  if (shift >= 32) {
    q = 0;                      /* below half the smallest step */
  } else {
    uint32_t kept = sig >> shift;
    uint32_t rem = sig & ((1u << shift) - 1u);
    uint32_t half = 1u << (shift - 1);
    q = kept;
    if (rem > half || (rem == half && (kept & 1u))) q += 1u;
  }
  uint32_t code;
  if (E < -6) {
    code = q;                   /* subnormal codes 0..8; 8 is the first normal */
  } else {
    /* q in [8,16]; q == 16 carries into the next exponent */
    int32_t be = E + 7;
    if (q == 16u) { q = 8u; be += 1; }
    if (be > 15 || (be == 15 && q > 14u)) return (uint8_t)(sign | 0x7Eu);
    code = ((uint32_t)be << 3) | (q - 8u);
  }
  return (uint8_t)(sign | code);
}

/* ------------------------------------------------------------------------ */
/* One synthetic tensor: every element is a pure function of its coordinates */

enum { SYN_KIND_NORMAL = 0, SYN_KIND_UNIFORM = 1 };

typedef struct syn_tensor {
  uint64_t seed;
  uint64_t stream;
  int32_t dim;               /* elements per row */
  int32_t kind;              /* SYN_KIND_NORMAL or SYN_KIND_UNIFORM */
  const uint8_t* outlier;    /* [dim], 1 = draw this channel from t(3); or NULL */
  int32_t n_needle;          /* needle blocks per sequence (0 = none) */
  int32_t needle_block;      /* positions per needle block (8) */
  const int32_t* needle_blk; /* [n_seq][n_needle] ascending block ids */
  const float* needle_dir;   /* [n_seq][dim] unit direction */
  float needle_shift;        /* added as shift*dir[c] to every key of a needle block */
} syn_tensor;

/* value of element (row_hi, pos, col); row_hi is the sequence for cache
 * tensors and 0 for per-token tensors */
SYN_FN float syn_value(const syn_tensor* t, uint64_t row_key, uint32_t seq,
                       int64_t pos, int32_t col, int needle) {
  uint64_t ek = syn_elem_key(row_key, (uint64_t)col);
  float v;
  if (t->kind == SYN_KIND_UNIFORM) {
    v = syn_uniform(ek);
  } else if (t->outlier && t->outlier[col]) {
    v = syn_t3(ek);
  } else {
    v = syn_normal(ek);
  }
  if (needle) {
    float d = t->needle_dir[(int64_t)seq * t->dim + col];
    v = syn_add(v, syn_mul(t->needle_shift, d));
  }
  (void)pos;
  return v;
}

SYN_FN int syn_is_needle(const syn_tensor* t, uint32_t seq, int64_t pos) {
  if (t->n_needle <= 0) return 0;
  int64_t blk = pos / t->needle_block;
  const int32_t* list = t->needle_blk + (int64_t)seq * t->n_needle;
  for (int i = 0; i < t->n_needle; ++i)
    if (list[i] == blk) return 1;
  return 0;
}

SYN_FN uint64_t syn_row_id(uint32_t seq, int64_t pos) {
  return ((uint64_t)seq << 32) | (uint64_t)(uint32_t)pos;
}

#endif /* CSA2_SYNTH_H */
