/*
 * csa2.h -- C ABI of the CSA2 FP4 sparse decode library (libcsa2.so), sm_100a.
 *
 * The library implements one decode step of CSA2 (DeepSeek-V4.1-Flash pages,
 * dbyun.net article 10794, section "KV Cache 成为这一代架构改造的核心"):
 *   - a Full layer scans every visible position of the FP4 indexer K cache,
 *     keeps the best P blocks of 8 positions as a candidate pool (the pages
 *     give P = 2048, i.e. at most 16384 positions) and its own top-K;
 *   - a Reindex layer rescores only that pool with its own indexer query and
 *     keeps its top-K (the pages give K = 512);
 *   - a Reuse layer reuses the index list and runs attention only, over the
 *     FP4 Main KV; optionally merged with sliding-window attention over an FP8
 *     SWA KV (prism.simon-ai.net article 7901, SWA section: 128 tokens).
 * Workload choices that the pages do not fix: the FP4 format (E2M1 codes,
 * one E4M3 scale per 32 elements), the indexer score
 * s_t = sum_h w_h * max(0, q_h . k_t), block score = max over the block,
 * MQA attention with V = the K latent and scale 1/sqrt(D).
 *
 * Conventions (all entry points):
 *   - Every pointer inside a descriptor or passed as a tensor is a DEVICE
 *     pointer owned by the caller, unless the comment says "host".  The
 *     library never allocates device memory; scratch space is the caller's
 *     `workspace` of at least the size returned by the matching
 *     csa2_*_workspace_size() call, 256-byte aligned.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Every call is asynchronous on that stream and returns a
 *     csa2_status synchronously describing argument validation and launch
 *     errors only.
 *   - Errors found on the device while the kernels run (non-finite quantiser
 *     input, an out-of-range index in the inputs, a wait that timed out) are
 *     recorded in a per-device status word; csa2_get_status() synchronises the
 *     stream, returns and clears it.
 *   - Index outputs are ascending, padded with -1, with a count array.
 *   - Functions are thread-safe as long as concurrent calls use different
 *     output and workspace buffers.  csa2_last_error() is per thread.
 *   - The quantiser, scan and attention kernels are launched with
 *     programmatic stream serialisation: their CTAs may be placed while the
 *     previous kernel on the stream runs, but each waits for that kernel's
 *     completion before touching global memory, so stream order is kept.
 *     The environment variable CSA2_OVERLAP (read once per process: a mask of
 *     1 quantiser, 2 scan, 4 rescoring, 8 selections, 16 attention; 0 = none)
 *     replaces the default set (1 | 2 | 16).
 */
#ifndef CSA2_H
#define CSA2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------- */
enum {
  CSA2_OK = 0,
  CSA2_ERR_INVALID_ARG = -1,  /* null pointer, negative size, inconsistent descriptor */
  CSA2_ERR_UNSUPPORTED = -2,  /* shape outside the supported set (e.g. dim % 32 != 0) */
  CSA2_ERR_WORKSPACE = -3,    /* workspace too small or misaligned */
  CSA2_ERR_CUDA = -4,         /* a CUDA runtime call failed (message in csa2_last_error) */
  CSA2_ERR_TIMEOUT = -5,      /* device: a bounded wait inside a kernel gave up */
  CSA2_ERR_NONFINITE = -6,    /* device: quantiser input held Inf/NaN (that group is zeroed) */
  CSA2_ERR_RANGE = -7         /* device: an index/page entry of the inputs was out of range (skipped),
                               * or a main query value has no fp16 form (|q| >= 65520 or NaN) */
};

enum { CSA2_F32 = 0, CSA2_BF16 = 1 };                         /* element types of q / out */
enum { CSA2_MODE_FULL = 0, CSA2_MODE_REINDEX = 1, CSA2_MODE_REUSE = 2 };

/* ---- descriptors -------------------------------------------------------- */

/* One decode batch.  Sequence b holds seq_len[b] cached positions, the last
 * W_b = tok_start[b+1]-tok_start[b] of which are this step's query tokens;
 * query token i = tok_start[b]+j sits at position tok_pos[i] = seq_len[b]-W_b+j
 * and sees positions 0..tok_pos[i] (causal). */
typedef struct csa2_query_batch {
  int32_t n_seq;             /* B >= 1 */
  int32_t n_tok;             /* T = sum_b W_b >= 1 */
  int32_t max_seq_len;       /* host-known upper bound on seq_len[b] */
  int32_t max_q_per_seq;     /* host-known upper bound on W_b */
  const int32_t* seq_len;    /* [B] */
  const int32_t* tok_start;  /* [B+1], tok_start[0] = 0, tok_start[B] = T */
  const int32_t* tok_seq;    /* [T] sequence of each query token */
  const int32_t* tok_pos;    /* [T] position of each query token */
} csa2_query_batch;

/* An FP4 cache (indexer K or Main KV): row r holds dim E2M1 codes packed two
 * per byte (element 2i in the low nibble) in codes[r][dim/2] and one E4M3
 * scale per 32 elements in scales[r][dim/32].  Position t of sequence b lives
 * in row  page_table[b*max_pages + t/page_size]*page_size + t%page_size  when
 * page_table != NULL (page_size must be a multiple of 64, and a table row
 * must cover the batch: max_pages * page_size >= max_seq_len, else the calls
 * return CSA2_ERR_INVALID_ARG), else in row seq_base[b] + t. */
typedef struct csa2_fp4_cache {
  uint8_t* codes;
  uint8_t* scales;
  int64_t n_rows;            /* rows allocated (bounds for checks and TMA) */
  int32_t dim;               /* multiple of 32 */
  int32_t page_size;         /* 0 when unpaged */
  const int32_t* page_table; /* [B][max_pages] or NULL */
  int32_t max_pages;
  const int64_t* seq_base;   /* [B] when unpaged */
} csa2_fp4_cache;

/* FP8 E4M3 sliding-window KV of one layer: a ring per sequence; position t of
 * sequence b is row b*cap + t%cap, value = e4m3(codes[row][c]) * scale[row].
 * The window of a query at p is positions max(0, p-window+1) .. p;
 * cap >= window + max_q_per_seq - 1 so that the whole window is resident. */
typedef struct csa2_swa_desc {
  const uint8_t* codes;      /* [B*cap][dim] */
  const float* scale;        /* [B*cap] */
  int32_t cap;
  int32_t window;            /* 1 .. 256 */
  int32_t dim;               /* equals the Main KV dim */
} csa2_swa_desc;

/* One layer of a decode stack. */
typedef struct csa2_layer_desc {
  int32_t mode;              /* CSA2_MODE_* ; layer 0 must be FULL */
  const float* iq;           /* FULL/REINDEX: indexer query [T][H_I][d_I] fp32 (quantised to FP4 in the step) */
  const float* iw;           /* FULL/REINDEX: head weights [T][H_I] fp32 */
  const void* q;             /* main query [T][Hq][D], q_dtype */
  const csa2_swa_desc* swa;  /* host pointer to a descriptor, or NULL */
  void* out;                 /* [T][Hq][D], out_dtype */
  float* lse;                /* optional [T][Hq] natural-log sum of exp of the scaled scores */
  int32_t* idx_out;          /* optional FULL/REINDEX: copy of the selected positions [T][K] */
  int32_t* pool_out;         /* optional FULL: copy of the pool [T][P] */
} csa2_layer_desc;

/* One decode step through a layer stack sharing one indexer K cache and one
 * Main KV (cross-layer sharing). */
typedef struct csa2_stack_desc {
  csa2_query_batch qb;
  csa2_fp4_cache k_idx;      /* dim = d_I */
  csa2_fp4_cache kv;         /* dim = D */
  int32_t H_I, P, K, Hq;
  int32_t q_dtype, out_dtype;
  float softmax_scale;       /* <= 0 selects 1/sqrt(D) */
  const float* new_k_idx;    /* optional [T][d_I]: this step's indexer keys, appended first */
  const float* new_kv;       /* optional [T][D]: this step's Main KV rows, appended first */
  const int64_t* new_slot_k_idx; /* [T] destination rows in k_idx */
  const int64_t* new_slot_kv;    /* [T] destination rows in kv */
  int32_t n_layers;
  const csa2_layer_desc* layers; /* host array [n_layers] */
  void* attend_wait_event;   /* optional cudaEvent_t: the attention launches of the step
                              * wait for it (e.g. the Main queries copied on another
                              * stream while the indexer runs); NULL = no wait.  The
                              * event must have been recorded before the call. */
} csa2_stack_desc;

/* ---- entry points -------------------------------------------------------- */

/* FP4 quantise (the pages' FP4 indexer Q/K and Main KV; cache fill and the
 * per-step append).  For every group of 32 consecutive elements of a row:
 * s = E4M3_rne_satfinite(amax / 6.0f); element codes are round-to-nearest-even
 * of |x|/s on the E2M1 grid (exact comparison, saturating at 6) with the sign
 * of x; s = 0 gives zero magnitudes.  x: [n_rows][dim] fp32.  Row r is written
 * to codes/scales row slot[r] (slot == NULL: row r).  dim % 32 == 0,
 * 32 <= dim <= 8192.  A group with Inf/NaN input is written as zeros and
 * CSA2_ERR_NONFINITE is recorded. */
int csa2_quantize_fp4(const float* x, int64_t n_rows, int32_t dim, const int64_t* slot, uint8_t* codes,
                      uint8_t* scales, void* stream);

/* Full mode (hierarchical indexer, first stage).  For every query token i and
 * visible position t <= p_i: s_t = sum_h w[i][h] * max(0, q~_{i,h} . k~_t) with
 * q~, k~ the dequantised FP4 values; block score B_j = max over the visible
 * positions of block j (8 positions); keeps the best P blocks (ties to the
 * lower block id; all blocks when there are at most P) -> pool[i][0..pool_n),
 * ascending; then the best K positions of the pool by s_t (ties to the lower
 * position; all when the pool has fewer) -> idx[i][0..idx_n), ascending.
 * q_codes [T][H_I][d_I/2], q_scales [T][H_I][d_I/32], w [T][H_I];
 * pool [T][P], pool_n [T], idx [T][K], idx_n [T]; blockscore: optional
 * [T][ceil(max_seq_len/8)] fp32 copy of B_j (entries past a token's last
 * visible block are unspecified).  d_I = k_idx->dim in {64, 128}; the
 * indexer cache's scale array is read in rows of 16 bytes: n_rows * d_I / 32
 * must be a multiple of 16 (else CSA2_ERR_UNSUPPORTED) and a row that holds a
 * position must start a 16-byte row of it (row * d_I / 32 a multiple of 16;
 * a misplaced row reads as zeros and CSA2_ERR_RANGE is recorded);
 * 1 <= H_I <= 64; 1 <= P <= 4096; 1 <= K <= 2048; K <= 8*P.  Any number of
 * query tokens per sequence: the scan reads the keys once for every 8 of a
 * sequence's tokens (a decode or verify step with W_b <= 8 reads them once). */
int csa2_index_full(const csa2_query_batch* qb, const uint8_t* q_codes, const uint8_t* q_scales, const float* w,
                    int32_t H_I, const csa2_fp4_cache* k_idx, int32_t P, int32_t K, int32_t* pool, int32_t* pool_n,
                    int32_t* idx, int32_t* idx_n, float* blockscore, void* workspace, size_t workspace_bytes,
                    void* stream);

/* Reindex mode: rescore only the pool positions (pool from csa2_index_full of
 * the same batch) with this layer's (q, w) and keep the best K (ties to the
 * lower position), ascending in idx[T][K] / idx_n[T]. */
int csa2_index_reindex(const csa2_query_batch* qb, const uint8_t* q_codes, const uint8_t* q_scales, const float* w,
                       int32_t H_I, const csa2_fp4_cache* k_idx, const int32_t* pool, const int32_t* pool_n,
                       int32_t P, int32_t K, int32_t* idx, int32_t* idx_n, void* workspace, size_t workspace_bytes,
                       void* stream);

/* Reuse mode: attention only.  For query token i and head h:
 * z_t = scale * q[i][h] . k~_t over t in S_i = idx[i][0..idx_n[i]) (rows of the
 * FP4 Main KV, V = the same latent), concatenated when swa != NULL with the
 * window rows max(0,p_i-window+1)..p_i of the FP8 SWA KV; one softmax over the
 * concatenation; out[i][h] = sum softmax(z)_t * v_t, rounded once to out_dtype.
 * q: [T][Hq][D] q_dtype (CSA2_F32 or CSA2_BF16); the tensor-core products
 * take q in fp16 (an fp32 q as an fp16 value plus its fp16 residual), so
 * |q| must stay below 65520 (else CSA2_ERR_RANGE is recorded);
 * out: [T][Hq][D] out_dtype; lse optional [T][Hq].  D = kv->dim in {128, 512};
 * Hq in {16, 32, 64}; CSA2_F32 queries need D * Hq <= 16384 (else
 * CSA2_ERR_UNSUPPORTED); 1 <= K <= 2048. */
int csa2_attend_reuse(const csa2_query_batch* qb, const void* q, int32_t q_dtype, int32_t Hq, const csa2_fp4_cache* kv,
                      const int32_t* idx, const int32_t* idx_n, int32_t K, const csa2_swa_desc* swa,
                      float softmax_scale, void* out, int32_t out_dtype, float* lse, void* workspace,
                      size_t workspace_bytes, void* stream);

/* One decode step: appends new_k_idx/new_kv (if given) with
 * csa2_quantize_fp4, quantises each selector layer's indexer query, then runs
 * the layers in order: FULL -> csa2_index_full; REINDEX -> csa2_index_reindex
 * over the Full layer's pool; REUSE -> the index list of the nearest preceding
 * FULL/REINDEX layer; every layer then attends as csa2_attend_reuse. */
int csa2_decode_stack(const csa2_stack_desc* desc, void* workspace, size_t workspace_bytes, void* stream);

/* Workspace sizes (bytes) of the calls above for the given shapes. */
int csa2_index_workspace_size(const csa2_query_batch* qb, int32_t H_I, int32_t d_I, int32_t P, int32_t K,
                              size_t* bytes);
int csa2_attend_workspace_size(const csa2_query_batch* qb, int32_t Hq, int32_t D, int32_t K, int32_t has_swa,
                               size_t* bytes);
int csa2_stack_workspace_size(const csa2_stack_desc* desc, size_t* bytes);

/* Synchronises `stream`, returns the first device-side error recorded since
 * the last call (CSA2_OK if none) and clears it. */
int csa2_get_status(void* stream);

/* Message of the last error returned on the calling thread ("" if none). */
const char* csa2_last_error(void);

/* Library version, major*10000 + minor*100 + patch. */
int csa2_version(void);

/* csa2_index_reindex without a workspace, for callers that cannot allocate
 * device memory or pass one (for example a serving engine that reserves all
 * device memory for its KV pool at start-up and forbids later allocations,
 * or a plug-in interface with no workspace argument).  The method described
 * on the pages has no counterpart to this call; it computes exactly what
 * csa2_index_reindex computes, with the same kernels, except that its
 * selection runs one CTA per query token (csa2_index_reindex splits a
 * token's candidates over several CTAs when there are few tokens), so for
 * small n_tok it can be slower.
 * Scratch: a fixed file-scope device array of 2^20 fp32 candidate scores
 * (4 MiB) that every GPU loading the library holds until the process exits;
 * requires n_tok * P * 8 <= 2^20, else returns CSA2_ERR_WORKSPACE and
 * launches nothing.  The call allocates nothing (no cudaMalloc, cudaFree or
 * allocating library routine).  Every call looks up the array's device
 * address for the current device (cudaGetSymbolAddress), so the address
 * stays right after a device reset; the first call on a device also loads
 * the library's kernels there, so make it before any stream capture.  Every
 * call shares the one array and leaves its contents behind; each call
 * overwrites every slot it reads, so nothing needs clearing, but calls that
 * overlap on the GPU (other streams, other threads) race on the array and
 * must be serialised. */
int csa2_index_reindex_noalloc(const csa2_query_batch* qb, const uint8_t* q_codes, const uint8_t* q_scales,
                               const float* w, int32_t H_I, const csa2_fp4_cache* k_idx, const int32_t* pool,
                               const int32_t* pool_n, int32_t P, int32_t K, int32_t* idx, int32_t* idx_n,
                               void* stream);

/* Kernel timing (the tracing hook).  While enabled, every kernel the library
 * launches is bracketed by a pair of CUDA events on its stream, aggregated per
 * kernel name.  Off by default; costs two event records per launch when on. */
typedef struct csa2_kernel_stat {
  char name[40];
  int64_t launches;
  double total_ms;
} csa2_kernel_stat;

int csa2_profiler_enable(int on);
/* Synchronises the recorded events, writes up to `cap` per-kernel totals since
 * the last read (or enable) into `out`, sets *n_out, and clears them. */
int csa2_profiler_read(csa2_kernel_stat* out, int32_t cap, int32_t* n_out);

/* ---- context parallelism: one sequence's positions over G GPUs ------------
 * Rank r holds positions [lo_r, hi_r) of each sequence (ascending ranges, lo
 * a multiple of 8) in its own caches and runs the calls above on its slice,
 * with query positions given relative to lo_r (a query sees its whole slice
 * when the slice ends before it, -1: nothing).  These calls combine the
 * ranks' results after the caller's all-gathers (every rank passes the same
 * gathered buffers, rank-major).  Exact: the global top-k of a set split into
 * parts lies in the union of the parts' top-k (hierarchical indexer, dbyun.net
 * article 10794, section "KV Cache 成为这一代架构改造的核心"), and one softmax
 * over a split key set is the log-sum-exp merge of the parts.  All pointers
 * are device pointers; every call is asynchronous on `stream`. */

/* A rank's selected local ids ids[T][n] (-1: none) -> (score, global id):
 * by_id != 0, score = scores[t][ld-strided row][id] (block scores), else
 * scores[t][i]; global id = id + offset; out_score/out_id [T][n] (-inf / -1
 * for none). */
int csa2_cp_candidates(const float* scores, int64_t ld, const int32_t* ids, int32_t n_tok, int32_t n, int32_t by_id,
                       int32_t offset, float* out_score, int32_t* out_id, void* stream);

/* Gathered candidate lists score/ids [n_ranks][T][n] -> per token the k
 * best by score (ties to the lower id), ascending, in out[T][k] (-1 padded),
 * counts out_n[T].  n_ranks * n <= 16384. */
int csa2_cp_merge(const float* score, const int32_t* ids, int32_t n_ranks, int32_t n_tok, int32_t n, int32_t k,
                  int32_t* out, int32_t* out_n, void* stream);

/* Global id lists ids[T][k] (ascending, n_in[t] valid) -> this rank's ids
 * (id - lo for lo <= id < hi): compact != 0, its entries in order, -1 padded,
 * counts out_n; compact == 0, entry i stays at i (-1 where not its own) and
 * out_n = n_in. */
int csa2_cp_localize(const int32_t* ids, const int32_t* n_in, int32_t n_tok, int32_t k, int64_t lo, int64_t hi,
                     int32_t compact, int32_t* out, int32_t* out_n, void* stream);

/* Pool-position scores of n_sel selector layers (queries [n_sel][T][H_I][..]
 * FP4, weights w[i] [T][H_I], host array of n_sel device pointers) over
 * `local_pool` [T][P] (the global pool made local and aligned with
 * csa2_cp_localize(compact = 0): -1 where another rank owns the block):
 * scores [n_sel][T][8P], -inf where not this rank's. */
int csa2_cp_pool_scores(const csa2_query_batch* qb, const uint8_t* q_codes, const uint8_t* q_scales,
                        const float* const* w, int32_t n_sel, int32_t H_I, const csa2_fp4_cache* k_idx,
                        const int32_t* local_pool, const int32_t* pool_n, int32_t P, float* scores, void* stream);

/* Gathered pool-position scores [n_ranks][n_sel][T][8P] -> per selector and
 * token the best K positions of the global pool[T][P] (ties to the lower
 * position), ascending, in idx[n_sel][T][K] (-1 padded), idx_n[n_sel][T].
 * P <= 2048. */
int csa2_cp_select_positions(const float* scores, int32_t n_ranks, int32_t n_sel, int32_t n_tok, const int32_t* pool,
                             const int32_t* pool_n, int32_t P, int32_t K, int32_t* idx, int32_t* idx_n, void* stream);

/* Gathered attention parts: rank g's part at o_parts + g * o_rank_stride,
 * [T][Hq][D] fp32 (its csa2_attend_reuse output over its own selected rows),
 * and lse_parts + g * lse_rank_stride, [T][Hq] (natural log, -inf for an
 * empty part) -> out [T][Hq][D] in out_dtype and, optionally, lse [T][Hq]
 * of the union (strides in elements). */
int csa2_cp_attend_merge(const float* o_parts, const float* lse_parts, int32_t n_ranks, int64_t o_rank_stride,
                         int64_t lse_rank_stride, int32_t n_tok, int32_t Hq, int32_t D, void* out, int32_t out_dtype,
                         float* lse, void* stream);

/* Tensor-core peak probe (a measurement hook, not part of the decode step):
 * every SM issues back-to-back dense M = 128, N = 256 MMAs from fixed
 * shared-memory operands, kind 0: kind::f16 (the attention products, fp16 in,
 * fp32 accumulate, K = 16), kind 1: kind::mxf4nvf4 with UE4M3 scales per 16
 * elements (the indexer products, K = 64); `iters` MMAs per issuing thread
 * (16 .. 2^20), two issuing threads per SM.  Writes the best of two timed runs
 * (after a warm-up run) in TFLOP/s (2 M N K per MMA) to *tflops.
 * Synchronises `stream`. */
int csa2_tensor_peak(int32_t kind, int32_t iters, double* tflops, void* stream);

/* Number of kernels this process has launched through the library. */
int64_t csa2_launch_count(void);

/* Test hook for the bounded-wait machinery: launches one CTA whose thread
 * waits on an mbarrier that nothing completes, giving up after `limit_ns`
 * nanoseconds (1e3 .. 1e10) and recording CSA2_ERR_TIMEOUT.  No fault, no
 * trap; the context stays usable. */
int csa2_selftest_wait_timeout(int64_t limit_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* CSA2_H */
