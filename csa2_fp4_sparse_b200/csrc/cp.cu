// cp.cu -- the kernels of the context-parallel decode step: one long
// sequence's positions are split over G GPUs in ascending ranges (each GPU
// holds its slice of the indexer K cache and Main KV), every rank runs the
// decode kernels on its slice, and these kernels turn the ranks' local
// results into the global ones between the caller's all-gathers.
//
// Exactness (hierarchical indexer of the DeepSeek-V4.1-Flash pages, dbyun.net
// article 10794, section "KV Cache 成为这一代架构改造的核心": top-2048 blocks,
// then top-512 positions): the global top-k of a set split into parts lies in
// the union of the parts' local top-k, so merging the ranks' local block
// selections (score, global id) gives the single-GPU pool, ties included
// (every rank lists ascending ids and the ranks own ascending ranges, so
// candidate order is global id order); the pool's positions are rescored by
// the rank that owns them and selected from the combined scores; attention
// over a key set split into parts is the log-sum-exp merge of the parts'
// normalised outputs.
//
//   k_cp_candidates    a rank's selection -> (score, global id) lists for the all-gather
//   k_cp_select        gathered lists [G][T][n] -> global top-k ids (ascending), or
//                      gathered pool-position scores [G][S][T][8P] -> top-k positions
//   k_cp_localize      global ids -> this rank's ids: aligned (-1 where not its own) or compacted
//   k_cp_attend_merge  gathered (o, lse) parts -> one softmax's output
#include "common.cuh"
#include "internal.h"

namespace csa2 {
namespace cp {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kPer = 32;                       // candidates per thread
constexpr int kMaxCand = kThreads * kPer;      // 16384 a token

// (score, global id) of a rank's selected local ids ids[t][i] (-1: none):
// by_id, the score is scores[t][id] (block scores); else scores[t][i]
__global__ void k_cp_candidates(const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ ids,
                                int n, int by_id, int32_t offset, float* __restrict__ out_score,
                                int32_t* __restrict__ out_id) {
  const int t = blockIdx.y;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const int32_t id = __ldg(ids + (int64_t)t * n + i);
    float s = -INFINITY;
    if (id >= 0) s = __ldg(scores + (int64_t)t * ld + (by_id ? id : i));
    out_score[(int64_t)t * n + i] = s;
    out_id[(int64_t)t * n + i] = id >= 0 ? id + offset : -1;
  }
}

// CTA-wide sum (two alternating buffers)
struct Red {
  int* buf;
  int par;
  __device__ int sum(int v) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    v = __reduce_add_sync(0xffffffffu, v);
    int* b = buf + par * kWarps;
    par ^= 1;
    if (lane == 0) b[wid] = v;
    __syncthreads();
    return __reduce_add_sync(0xffffffffu, lane < kWarps ? b[lane] : 0);
  }
};

struct SelArgs {
  // lists mode: candidate c = g*n + i of score/ids [G][T][n]
  // pool mode: candidate c = pool entry (c < pool_n*8) of token t, key the
  //            largest of the G ranks' scores [G][S][T][8P] (a rank holds -inf
  //            where it does not own the position), id = pool[t][c/8]*8 + c%8
  const float* score;
  const int32_t* ids;
  const int32_t* pool;
  const int32_t* pool_n;
  int G, T, n, S, P, k;
  int32_t* out;
  int32_t* out_n;
  int* status;
};

// One CTA per (token, selector): the k best candidates by score, ties to the
// earlier candidate, written as ascending ids, -1 padded; count in out_n.
template <bool kPool>
__global__ void __launch_bounds__(kThreads) k_cp_select(const __grid_constant__ SelArgs A) {
  __shared__ int red_b[2 * kWarps];
  __shared__ int wgt[kWarps], weq[kWarps];
  const int t = blockIdx.x, sel = blockIdx.y, lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int nc = kPool ? min(__ldg(A.pool_n + t), A.P) * kBlock : A.G * A.n;
  Red red{red_b, 0};
  // candidate of (warp, j, lane): c = wid*1024 + j*32 + lane
  uint32_t key[kPer];
  int32_t cid[kPer];
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int c = wid * 32 * kPer + j * 32 + lane;
    key[j] = 0u;
    cid[j] = -1;
    if (c < nc) {
      if (kPool) {
        cid[j] = __ldg(A.pool + (int64_t)t * A.P + c / kBlock) * kBlock + c % kBlock;
        for (int g = 0; g < A.G; ++g) {
          const float s = __ldg(A.score + (((int64_t)g * A.S + sel) * A.T + t) * (A.P * kBlock) + c);
          key[j] = max(key[j], score_key(s));
        }
      } else {
        const int64_t e = ((int64_t)(c / A.n) * A.T + t) * A.n + c % A.n;
        cid[j] = __ldg(A.ids + e);
        key[j] = cid[j] >= 0 ? score_key(__ldg(A.score + e)) : 0u;
      }
      if (cid[j] < 0) key[j] = 0u;
    }
  }
  int valid = 0;
#pragma unroll
  for (int j = 0; j < kPer; ++j) valid += key[j] != 0u;
  valid = red.sum(valid);
  const int k_eff = min(A.k, valid);
  // the k-th largest key, bit by bit from the top
  uint32_t thr = 0u;
  if (k_eff > 0) {
    for (int b = 31; b >= 0; --b) {
      const uint32_t cand = thr | (1u << b);
      int c = 0;
#pragma unroll
      for (int j = 0; j < kPer; ++j) c += key[j] >= cand;
      if (red.sum(c) >= k_eff) thr = cand;
    }
  }
  int above = 0;
#pragma unroll
  for (int j = 0; j < kPer; ++j) above += key[j] > thr;
  const int need_eq = k_eff - red.sum(above);
  // ordered output: (warp, j, lane) order is candidate order
  auto is_gt = [&](uint32_t x) { return x != 0u && x > thr; };
  auto is_eq = [&](uint32_t x) { return k_eff > 0 && x != 0u && x == thr; };
  int wg = 0, we = 0;
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    wg += __popc(__ballot_sync(0xffffffffu, is_gt(key[j])));
    we += __popc(__ballot_sync(0xffffffffu, is_eq(key[j])));
  }
  if (lane == 0) {
    wgt[wid] = wg;
    weq[wid] = we;
  }
  __syncthreads();
  int written = 0, ties = 0;
  for (int w = 0; w < wid; ++w) {
    written += wgt[w] + max(0, min(weq[w], need_eq - ties));
    ties += weq[w];
  }
  int32_t* o = A.out + ((int64_t)sel * A.T + t) * A.k;
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const bool g = is_gt(key[j]);
    const bool e = is_eq(key[j]);
    const uint32_t em = __ballot_sync(0xffffffffu, e);
    const int e_rank = ties + __popc(em & ((1u << lane) - 1u));
    const bool take = g || (e && e_rank < need_eq);
    const uint32_t sm = __ballot_sync(0xffffffffu, take);
    const int at = written + __popc(sm & ((1u << lane) - 1u));
    if (take && at < A.k) o[at] = cid[j];
    written += __popc(sm);
    ties += __popc(em);
  }
  int total = 0, tt = 0;
  for (int w = 0; w < kWarps; ++w) {
    total += wgt[w] + max(0, min(weq[w], need_eq - tt));
    tt += weq[w];
  }
  if (total != k_eff && threadIdx.x == 0) set_status(A.status, CSA2_ERR_RANGE);  // inconsistent counts
  for (int j = k_eff + threadIdx.x; j < A.k; j += kThreads) o[j] = -1;
  if (threadIdx.x == 0) A.out_n[(int64_t)sel * A.T + t] = k_eff;
}

// global id lists [T][k] (ascending, -1 padded, n_in[t] valid) -> this rank's
// ids (id - lo for lo <= id < hi): compact, its entries in order, -1 padded,
// count in out_n; aligned, entry i kept at i (-1 where not its own)
__global__ void __launch_bounds__(kThreads) k_cp_localize(const int32_t* __restrict__ ids,
                                                          const int32_t* __restrict__ n_in, int k, int64_t lo,
                                                          int64_t hi, int compact, int32_t* __restrict__ out,
                                                          int32_t* __restrict__ out_n) {
  __shared__ int wcount[kWarps];
  __shared__ int run_s;
  const int t = blockIdx.x, lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int n = min(__ldg(n_in + t), k);
  if (threadIdx.x == 0) run_s = 0;
  __syncthreads();
  for (int c0 = 0; c0 < k; c0 += kThreads) {
    const int c = c0 + threadIdx.x;
    const int32_t id = c < n ? __ldg(ids + (int64_t)t * k + c) : -1;
    const bool mine = id >= 0 && id >= lo && id < hi;
    if (!compact) {
      if (c < k) out[(int64_t)t * k + c] = mine ? (int32_t)(id - lo) : -1;
      continue;
    }
    const uint32_t m = __ballot_sync(0xffffffffu, mine);
    if (lane == 0) wcount[wid] = __popc(m);
    __syncthreads();
    int before = run_s;
    for (int w = 0; w < wid; ++w) before += wcount[w];
    if (mine) out[(int64_t)t * k + before + __popc(m & ((1u << lane) - 1u))] = (int32_t)(id - lo);
    __syncthreads();
    if (threadIdx.x == 0) {
      int tot = 0;
      for (int w = 0; w < kWarps; ++w) tot += wcount[w];
      run_s += tot;
    }
    __syncthreads();
  }
  if (!compact) {
    if (threadIdx.x == 0) out_n[t] = n;
    return;
  }
  const int cnt = run_s;
  for (int j = cnt + threadIdx.x; j < k; j += kThreads) out[(int64_t)t * k + j] = -1;
  if (threadIdx.x == 0) out_n[t] = cnt;
}

// gathered parts: part g at o_parts + g*o_stride [T][Hq][D] fp32 (normalised
// over its part of the key set) and lse_parts + g*lse_stride [T][Hq] (natural
// log; -inf: empty part) -> the output
// of one softmax over the union: o = sum_g e^(lse_g - L) o_g, L = log sum_g e^lse_g
__global__ void k_cp_attend_merge(const float* __restrict__ o_parts, const float* __restrict__ lse_parts, int G,
                                  int64_t o_stride, int64_t lse_stride, int T, int Hq, int D, void* __restrict__ out,
                                  int out_f32, float* __restrict__ lse) {
  const int h = blockIdx.x, t = blockIdx.y;
  float m = -INFINITY;
  for (int g = 0; g < G; ++g) m = fmaxf(m, __ldg(lse_parts + g * lse_stride + (int64_t)t * Hq + h));
  float wsum = 0.0f;
  for (int g = 0; g < G; ++g) {
    const float l = __ldg(lse_parts + g * lse_stride + (int64_t)t * Hq + h);
    wsum += (l == -INFINITY) ? 0.0f : expf(l - m);
  }
  const float inv = wsum > 0.0f ? 1.0f / wsum : 0.0f;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float acc = 0.0f;
    for (int g = 0; g < G; ++g) {
      const float l = __ldg(lse_parts + g * lse_stride + (int64_t)t * Hq + h);
      if (l == -INFINITY) continue;
      acc += expf(l - m) * __ldg(o_parts + g * o_stride + ((int64_t)t * Hq + h) * D + d);
    }
    const int64_t oi = ((int64_t)t * Hq + h) * D + d;
    if (out_f32)
      reinterpret_cast<float*>(out)[oi] = acc * inv;
    else
      reinterpret_cast<__nv_bfloat16*>(out)[oi] = __float2bfloat16_rn(acc * inv);
  }
  if (lse && threadIdx.x == 0) lse[(int64_t)t * Hq + h] = wsum > 0.0f ? m + logf(wsum) : -INFINITY;
}

}  // namespace cp

int launch_rescore(const csa2_query_batch* qb, const uint8_t* qc, const uint8_t* qs, const float* w, int H,
                   const csa2_fp4_cache* kc, const int32_t* pool, const int32_t* pool_n, int P, float* scores,
                   cudaStream_t st);
int check_index_args(const csa2_query_batch* qb, const uint8_t* qc, const uint8_t* qs, const float* w, int H_I,
                     const csa2_fp4_cache* kc, int P, int K);
void clear_last_error();

}  // namespace csa2

using namespace csa2;

extern "C" {

int csa2_cp_candidates(const float* scores, int64_t ld, const int32_t* ids, int32_t n_tok, int32_t n, int32_t by_id,
                       int32_t offset, float* out_score, int32_t* out_id, void* stream) {
  clear_last_error();
  if (!scores || !ids || !out_score || !out_id || n_tok < 1 || n < 1 || n_tok > 65535 || ld < 1)
    return fail(CSA2_ERR_INVALID_ARG, "bad arguments");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Launch L_("cp_candidates", st);
  cp::k_cp_candidates<<<dim3((n + 255) / 256, n_tok), 256, 0, st>>>(scores, ld, ids, n, by_id, offset, out_score,
                                                                     out_id);
  return cuda_check(cudaGetLastError(), "k_cp_candidates");
}

int csa2_cp_merge(const float* score, const int32_t* ids, int32_t n_ranks, int32_t n_tok, int32_t n, int32_t k,
                  int32_t* out, int32_t* out_n, void* stream) {
  clear_last_error();
  if (!score || !ids || !out || !out_n || n_ranks < 1 || n_tok < 1 || n < 1 || k < 1 || n_tok > 65535)
    return fail(CSA2_ERR_INVALID_ARG, "bad arguments");
  if ((int64_t)n_ranks * n > cp::kMaxCand) return fail(CSA2_ERR_UNSUPPORTED, "at most %d candidates a token", cp::kMaxCand);
  cp::SelArgs a{};
  a.score = score;
  a.ids = ids;
  a.G = n_ranks;
  a.T = n_tok;
  a.n = n;
  a.S = 1;
  a.k = k;
  a.out = out;
  a.out_n = out_n;
  a.status = status_ptr();
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Launch L_("cp_merge", st);
  cp::k_cp_select<false><<<dim3(n_tok, 1), cp::kThreads, 0, st>>>(a);
  return cuda_check(cudaGetLastError(), "k_cp_select");
}

int csa2_cp_pool_scores(const csa2_query_batch* qb, const uint8_t* q_codes, const uint8_t* q_scales,
                        const float* const* w, int32_t n_sel, int32_t H_I, const csa2_fp4_cache* k_idx,
                        const int32_t* local_pool, const int32_t* pool_n, int32_t P, float* scores, void* stream) {
  clear_last_error();
  if (!w || n_sel < 1 || n_sel > kMaxSel) return fail(CSA2_ERR_UNSUPPORTED, "1..%d selector layers", kMaxSel);
  for (int i = 0; i < n_sel; ++i)
    if (int rc = check_index_args(qb, q_codes, q_scales, w[i], H_I, k_idx, P, 1)) return rc;
  if (!local_pool || !pool_n || !scores) return fail(CSA2_ERR_INVALID_ARG, "NULL buffer");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t qstride_c = (size_t)qb->n_tok * H_I * (k_idx->dim / 2), qstride_s = (size_t)qb->n_tok * H_I * (k_idx->dim / 32);
  for (int i = 0; i < n_sel; ++i)
    if (int rc = launch_rescore(qb, q_codes + i * qstride_c, q_scales + i * qstride_s, w[i], H_I, k_idx, local_pool,
                                pool_n, P, scores + (size_t)i * qb->n_tok * P * kBlock, st))
      return rc;
  return CSA2_OK;
}

int csa2_cp_select_positions(const float* scores, int32_t n_ranks, int32_t n_sel, int32_t n_tok, const int32_t* pool,
                             const int32_t* pool_n, int32_t P, int32_t K, int32_t* idx, int32_t* idx_n, void* stream) {
  clear_last_error();
  if (!scores || !pool || !pool_n || !idx || !idx_n || n_ranks < 1 || n_sel < 1 || n_tok < 1 || n_tok > 65535)
    return fail(CSA2_ERR_INVALID_ARG, "bad arguments");
  if (P < 1 || (int64_t)P * kBlock > cp::kMaxCand) return fail(CSA2_ERR_UNSUPPORTED, "P must be in [1, 2048]");
  if (K < 1 || K > P * kBlock) return fail(CSA2_ERR_UNSUPPORTED, "K must be in [1, 8P]");
  cp::SelArgs a{};
  a.score = scores;
  a.pool = pool;
  a.pool_n = pool_n;
  a.G = n_ranks;
  a.T = n_tok;
  a.S = n_sel;
  a.P = P;
  a.k = K;
  a.out = idx;
  a.out_n = idx_n;
  a.status = status_ptr();
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Launch L_("cp_select_positions", st);
  cp::k_cp_select<true><<<dim3(n_tok, n_sel), cp::kThreads, 0, st>>>(a);
  return cuda_check(cudaGetLastError(), "k_cp_select");
}

int csa2_cp_localize(const int32_t* ids, const int32_t* n_in, int32_t n_tok, int32_t k, int64_t lo, int64_t hi,
                     int32_t compact, int32_t* out, int32_t* out_n, void* stream) {
  clear_last_error();
  if (!ids || !n_in || !out || !out_n || n_tok < 1 || k < 1 || lo < 0 || hi < lo || n_tok > 65535)
    return fail(CSA2_ERR_INVALID_ARG, "bad arguments");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Launch L_("cp_localize", st);
  cp::k_cp_localize<<<n_tok, cp::kThreads, 0, st>>>(ids, n_in, k, lo, hi, compact, out, out_n);
  return cuda_check(cudaGetLastError(), "k_cp_localize");
}

int csa2_cp_attend_merge(const float* o_parts, const float* lse_parts, int32_t n_ranks, int64_t o_rank_stride,
                         int64_t lse_rank_stride, int32_t n_tok, int32_t Hq, int32_t D, void* out, int32_t out_dtype,
                         float* lse, void* stream) {
  clear_last_error();
  if (!o_parts || !lse_parts || !out || n_ranks < 1 || n_tok < 1 || Hq < 1 || D < 1 || n_tok > 65535 || Hq > 65535)
    return fail(CSA2_ERR_INVALID_ARG, "bad arguments");
  if (out_dtype != CSA2_F32 && out_dtype != CSA2_BF16) return fail(CSA2_ERR_INVALID_ARG, "bad dtype");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Launch L_("cp_attend_merge", st);
  cp::k_cp_attend_merge<<<dim3(Hq, n_tok), 128, 0, st>>>(o_parts, lse_parts, n_ranks, o_rank_stride, lse_rank_stride,
                                                          n_tok, Hq, D, out, out_dtype == CSA2_F32, lse);
  return cuda_check(cudaGetLastError(), "k_cp_attend_merge");
}

}  // extern "C"
