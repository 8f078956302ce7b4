/*
 * oracle.c -- plain, slow CPU definition of the CSA2 decode step.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link or
 * call this file; only the tests, the package's smoke check and the
 * benchmark's CPU baseline use it.  It shares no code with the CUDA library.
 *
 * Everything after the FP4 codes is computed in double precision on the
 * dequantised values, one definition at a time, with no blocking, fusion or
 * reordering beyond what the definition states.  Loops over independent
 * outputs (rows, heads) may run in parallel (OpenMP); no reduction is split.
 *
 * Sources (DeepSeek-V4.1-Flash pages, dbyun.net article 10794, section
 * "KV Cache 成为这一代架构改造的核心"):
 *   - Full / Reindex / Reuse layer modes: a Full layer generates Main KV and
 *     indexer K and re-searches the top-K; Reindex reuses the global KV and
 *     recomputes only which positions matter; Reuse reuses the indices as
 *     well and only runs attention.
 *   - hierarchical indexer: the first Full layer scans the whole visible
 *     context and keeps at most 2048 blocks of 8 positions; later layers pick
 *     the final top-512 inside that pool.
 *   - FP4 for the indexer Q/K and the Main KV; SWA KV stays FP8.
 * The FP4 element format (E2M1 with one E4M3 scale per 32 elements), the
 * indexer score sum_h w_h * ReLU(q_h . k_t), block score = max over the
 * block, and the attention form (MQA, V = K latent, scale 1/sqrt(D)) are
 * synthetic choices of this workload, not values the pages fix.
 *
 * Parity pins live in tests/test_oracle_pins.py.  Functions without an
 * independent pin: none.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* E4M3 ("FN" variant: bias 7, no infinities, S.1111.111 = NaN, max 448)      */

double orc_e4m3_value(uint8_t b) {
  int s = b >> 7, e = (b >> 3) & 15, m = b & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0)
    v = ldexp((double)m, -9);          /* subnormal: m * 2^-9 */
  else
    v = ldexp((double)(8 + m), e - 10); /* (1 + m/8) * 2^(e-7) */
  return s ? -v : v;
}

/* nearest non-negative finite E4M3 code to v >= 0; ties to the even code;
 * values above 448 saturate to 448.  Plain search over all 127 codes. */
uint8_t orc_e4m3_encode_nonneg(double v) {
  int best = 0;
  double best_d = INFINITY;
  if (v >= 448.0) return 0x7E;
  for (int c = 0; c <= 0x7E; ++c) {
    double d = fabs(orc_e4m3_value((uint8_t)c) - v);
    if (d < best_d || (d == best_d && (c & 1) == 0 && (best & 1) == 1)) {
      best = c;
      best_d = d;
    }
  }
  return (uint8_t)best;
}

/* ------------------------------------------------------------------------ */
/* E2M1: 1 sign bit, magnitude index 0..7 -> {0, .5, 1, 1.5, 2, 3, 4, 6}      */

static const double kE2M1[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double orc_e2m1_value(uint8_t nib) {
  double v = kE2M1[nib & 7];
  return (nib & 8) ? -v : v;
}

/* magnitude index of round-to-nearest-even(|x| / s) on the E2M1 grid,
 * saturating at 6.  The distances |x| - s*v_i are compared as exact
 * differences (s*v_i has at most 7 significant bits). */
static int e2m1_index(float ax, double s) {
  int best = 0;
  double best_d = INFINITY;
  for (int i = 0; i < 8; ++i) {
    double d = fabs((double)ax - s * kE2M1[i]);
    if (d < best_d || (d == best_d && (i & 1) == 0 && (best & 1) == 1)) {
      best = i;
      best_d = d;
    }
  }
  return best;
}

/*
 * FP4 quantiser (the storage format named by the pages: indexer Q/K and
 * Main KV in FP4).  For every group of 32 consecutive elements of a row:
 *   amax = max |x_i|                      (exact, fp32)
 *   q    = amax / 6.0f                    (one fp32 round-to-nearest division)
 *   s    = E4M3(q), RNE, saturating at 448; values <= 2^-10 become 0
 *   code = sign(x) | RNE(|x|/s) on the E2M1 grid (saturating at 6); s == 0
 *          gives magnitude 0
 * Codes are packed two per byte (element 2i in the low nibble); scales are
 * stored [row][dim/32].  Returns the number of groups holding a non-finite
 * value (their output is unspecified).
 */
int64_t orc_quantize_fp4(const float* x, int64_t n_rows, int dim, uint8_t* codes, uint8_t* scales) {
  int64_t bad = 0;
  int groups = dim / 32;
#pragma omp parallel for reduction(+ : bad) schedule(static)
  for (int64_t r = 0; r < n_rows; ++r) {
    for (int g = 0; g < groups; ++g) {
      const float* xg = x + r * dim + g * 32;
      float amax = 0.0f;
      int finite = 1;
      for (int i = 0; i < 32; ++i) {
        float a = fabsf(xg[i]);
        if (!isfinite(a)) finite = 0;
        if (a > amax) amax = a;
      }
      if (!finite) {
        ++bad;
        continue;
      }
      volatile float qf = amax / 6.0f; /* fp32 division, round to nearest */
      uint8_t sc = orc_e4m3_encode_nonneg((double)qf);
      double s = orc_e4m3_value(sc);
      scales[r * groups + g] = sc;
      for (int i = 0; i < 32; i += 2) {
        uint8_t nib[2];
        for (int k = 0; k < 2; ++k) {
          float v = xg[i + k];
          int idx = (s == 0.0) ? 0 : e2m1_index(fabsf(v), s);
          nib[k] = (uint8_t)((signbit(v) ? 8 : 0) | idx);
        }
        codes[r * (dim / 2) + (g * 32 + i) / 2] = (uint8_t)(nib[0] | (nib[1] << 4));
      }
    }
  }
  return bad;
}

/* dequantised FP4 rows in double: out[r][c] = e2m1(code) * e4m3(scale) */
void orc_dequant_fp4(const uint8_t* codes, const uint8_t* scales, int64_t n_rows, int dim, double* out) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < n_rows; ++r)
    for (int c = 0; c < dim; ++c) {
      uint8_t byte = codes[r * (dim / 2) + c / 2];
      uint8_t nib = (c & 1) ? (byte >> 4) : (byte & 15);
      out[r * dim + c] = orc_e2m1_value(nib) * orc_e4m3_value(scales[r * (dim / 32) + c / 32]);
    }
}

/* ------------------------------------------------------------------------ */
/* Indexer scores: s_t = sum_h w_h * max(0, sum_c q[h][c] * k[t][c])          */

/* k given as FP4 rows (codes/scales of n rows, dim d); q [H][d] double */
void orc_index_scores_fp4(const double* q, const double* w, int H, int d, const uint8_t* kcodes,
                          const uint8_t* kscales, int64_t n, double* s) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < n; ++t) {
    double kt[1024];
    for (int c = 0; c < d; ++c) {
      uint8_t byte = kcodes[t * (d / 2) + c / 2];
      uint8_t nib = (c & 1) ? (byte >> 4) : (byte & 15);
      kt[c] = orc_e2m1_value(nib) * orc_e4m3_value(kscales[t * (d / 32) + c / 32]);
    }
    double acc = 0.0;
    for (int h = 0; h < H; ++h) {
      double dot = 0.0;
      for (int c = 0; c < d; ++c) dot += q[h * d + c] * kt[c];
      acc += w[h] * (dot > 0.0 ? dot : 0.0);
    }
    s[t] = acc;
  }
}

/* ------------------------------------------------------------------------ */
/* Selection                                                                 */

typedef struct {
  double s;
  int64_t id;
} scored_t;

/* descending score, ties to the lower id */
static int cmp_scored(const void* a, const void* b) {
  const scored_t* x = (const scored_t*)a;
  const scored_t* y = (const scored_t*)b;
  if (x->s > y->s) return -1;
  if (x->s < y->s) return 1;
  return (x->id < y->id) ? -1 : (x->id > y->id);
}

static int cmp_i64(const void* a, const void* b) {
  int64_t x = *(const int64_t*)a, y = *(const int64_t*)b;
  return (x < y) ? -1 : (x > y);
}

/* the k best (score desc, id asc) of n scored ids, returned ascending by id;
 * returns min(k, n) */
int64_t orc_topk(const double* score, const int64_t* ids, int64_t n, int64_t k, int64_t* out) {
  scored_t* v = (scored_t*)malloc(sizeof(scored_t) * (size_t)(n > 0 ? n : 1));
  for (int64_t i = 0; i < n; ++i) {
    v[i].s = score[i];
    v[i].id = ids[i];
  }
  qsort(v, (size_t)n, sizeof(scored_t), cmp_scored);
  int64_t m = n < k ? n : k;
  for (int64_t i = 0; i < m; ++i) out[i] = v[i].id;
  qsort(out, (size_t)m, sizeof(int64_t), cmp_i64);
  free(v);
  return m;
}

/* block scores B_j = max of s_t over the visible positions t <= p of block j
 * (blocks of `blk` positions); returns the number of blocks ceil((p+1)/blk) */
int64_t orc_block_scores(const double* s, int64_t p, int blk, double* bs) {
  int64_t nb = (p + 1 + blk - 1) / blk;
  for (int64_t j = 0; j < nb; ++j) {
    double m = -INFINITY;
    for (int64_t t = j * blk; t < (j + 1) * blk && t <= p; ++t)
      if (s[t] > m) m = s[t];
    bs[j] = m;
  }
  return nb;
}

/* ------------------------------------------------------------------------ */
/* Attention over a set of rows: for each head h,                            */
/*   z_t = scale * q_h . v_t,  o_h = sum_t e^{z_t - m} v_t / sum_t e^{z_t - m} */
/*   lse_h = m + log(sum_t e^{z_t - m})                                      */
/* v [n][D] double (V = K), q [H][D] double, out [H][D]                      */

void orc_attend(const double* q, int H, int D, const double* v, int64_t n, double scale, double* out,
                double* lse) {
#pragma omp parallel for schedule(static)
  for (int h = 0; h < H; ++h) {
    double* z = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    double m = -INFINITY;
    for (int64_t t = 0; t < n; ++t) {
      double dot = 0.0;
      for (int c = 0; c < D; ++c) dot += q[h * D + c] * v[t * D + c];
      z[t] = scale * dot;
      if (z[t] > m) m = z[t];
    }
    double l = 0.0;
    for (int c = 0; c < D; ++c) out[h * D + c] = 0.0;
    for (int64_t t = 0; t < n; ++t) {
      double e = exp(z[t] - m);
      l += e;
      for (int c = 0; c < D; ++c) out[h * D + c] += e * v[t * D + c];
    }
    for (int c = 0; c < D; ++c) out[h * D + c] = n > 0 ? out[h * D + c] / l : 0.0;
    if (lse) lse[h] = n > 0 ? m + log(l) : -INFINITY;
    free(z);
  }
}
