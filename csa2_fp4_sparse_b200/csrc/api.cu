// api.cu -- the C ABI of libcsa2.so: argument validation, workspace carving
// and kernel launches on the caller's stream.  No device allocation here.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <cstdlib>
#include <algorithm>
#include <atomic>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "internal.h"
#include "kernels_simt.cuh"
#include "select.cuh"

namespace csa2 {

__device__ int g_status;  // per-device status word (first device-side error)

static thread_local char t_err[512];

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_err, sizeof(t_err), fmt, ap);
  va_end(ap);
  return code;
}

int cuda_check(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return CSA2_OK;
  return fail(CSA2_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool overlap_launches(int kind) {
  static const int mask = [] {
    const char* e = std::getenv("CSA2_OVERLAP");
    return e ? std::atoi(e) : kOverlapQuantize | kOverlapScan | kOverlapAttend;
  }();
  return (mask & kind) != 0;
}

int* status_ptr() {
  static int* cache[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (!cache[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return nullptr;
    cache[dev] = static_cast<int*>(p);
  }
  return cache[dev];
}

// ---------------------------------------------------------------- profiler
namespace {
std::atomic<int64_t> g_launches{0};
std::atomic<bool> g_prof_on{false};
std::mutex g_prof_mu;
struct ProfRec {
  const char* name;
  cudaEvent_t a, b;
};
std::vector<ProfRec> g_prof_recs;
std::vector<cudaEvent_t> g_event_pool;

cudaEvent_t pool_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}
}  // namespace

Launch::Launch(const char* n, cudaStream_t s) : name(n), st(s), slot(-1) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (!g_prof_on.load(std::memory_order_relaxed)) return;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  ProfRec r{n, pool_event(), pool_event()};
  cudaEventRecord(r.a, s);
  g_prof_recs.push_back(r);
  slot = (int)g_prof_recs.size() - 1;
}

Launch::~Launch() {
  if (slot < 0) return;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (slot < (int)g_prof_recs.size()) cudaEventRecord(g_prof_recs[slot].b, st);
}

// ---------------------------------------------------------------- validation
static int check_batch(const csa2_query_batch* qb) {
  if (!qb) return fail(CSA2_ERR_INVALID_ARG, "query batch is NULL");
  if (qb->n_seq < 1 || qb->n_tok < 1) return fail(CSA2_ERR_INVALID_ARG, "n_seq and n_tok must be >= 1");
  if (qb->max_seq_len < 1 || qb->max_q_per_seq < 1 || qb->max_q_per_seq > qb->max_seq_len)
    return fail(CSA2_ERR_INVALID_ARG, "bad max_seq_len/max_q_per_seq");
  if (!qb->seq_len || !qb->tok_start || !qb->tok_seq || !qb->tok_pos)
    return fail(CSA2_ERR_INVALID_ARG, "query batch arrays must be non-NULL");
  return CSA2_OK;
}

// the cache descriptor, and that a paged cache's table covers every position
// the batch can address (the kernels index page_table[b][t / page_size]
// without a bound: a sequence longer than its table row would read the next
// sequence's pages)
static int check_cache(const csa2_fp4_cache* c, const char* name, const csa2_query_batch* qb) {
  if (!c) return fail(CSA2_ERR_INVALID_ARG, "%s cache is NULL", name);
  if (!c->codes || !c->scales || c->n_rows < 1) return fail(CSA2_ERR_INVALID_ARG, "%s cache buffers missing", name);
  if (c->dim < 32 || c->dim % 32) return fail(CSA2_ERR_UNSUPPORTED, "%s dim %d not a multiple of 32", name, c->dim);
  if (c->page_table) {
    if (c->page_size < 64 || c->page_size % 64 || c->max_pages < 1)
      return fail(CSA2_ERR_UNSUPPORTED, "%s page_size must be a positive multiple of 64", name);
    if ((int64_t)qb->max_seq_len > (int64_t)c->max_pages * c->page_size)
      return fail(CSA2_ERR_INVALID_ARG, "%s: max_seq_len %d exceeds max_pages * page_size = %lld", name,
                  qb->max_seq_len, (long long)c->max_pages * c->page_size);
  } else if (!c->seq_base) {
    return fail(CSA2_ERR_INVALID_ARG, "%s: unpaged cache needs seq_base", name);
  }
  return CSA2_OK;
}

struct Carve {
  uint8_t* base;
  size_t cap, used = 0;
  void* take(size_t bytes) {
    size_t off = (used + 255) & ~size_t(255);
    used = off + bytes;
    return base ? base + off : nullptr;
  }
  bool ok() const { return used <= cap; }
};

static int n_blocks_max(const csa2_query_batch* qb) { return (qb->max_seq_len + kBlock - 1) / kBlock; }

// Key counts that seed the selections: kHistBins counts per group, filled by
// the scoring kernels, zeroed by one memset per call and left zeroed by every
// selection; the block selection's T groups, then the position selection's
// n_sel * T groups.
struct SelPlan {
  uint32_t* blk = nullptr;
  uint32_t* pos = nullptr;
  size_t bytes = 0;
};
static SelPlan take_select_scratch(Carve& c, const csa2_query_batch* qb, int, int n_sel) {
  SelPlan s;
  const int64_t gb = qb->n_tok, gp = (int64_t)qb->n_tok * n_sel;
  s.bytes = (size_t)(gb + gp) * kHistBins * 4;
  auto* z = static_cast<uint32_t*>(c.take(s.bytes));
  if (z) {
    s.blk = z;
    s.pos = z + gb * kHistBins;
  }
  return s;
}
static size_t select_ws(const csa2_query_batch* qb, int P, int n_sel) {
  Carve c{nullptr, 0};
  take_select_scratch(c, qb, P, n_sel);
  return c.used + 256;
}
static int clear_select_counts(const SelPlan& s, cudaStream_t st) {
  return cuda_check(cudaMemsetAsync(s.blk, 0, s.bytes, st), "clear selection counts");
}

// block scores, pool position scores, selection scratch
static size_t index_ws(const csa2_query_batch* qb, int P) {
  Carve c{nullptr, 0};
  c.take((size_t)qb->n_tok * n_blocks_max(qb) * 4);  // block scores
  c.take((size_t)qb->n_tok * P * kBlock * 4);        // pool position scores
  c.take(select_ws(qb, P, 1));                       // selection scratch
  return c.used + 256;
}

// attention: split partials exist only while a launch has fewer than 148
// (token, layer) pairs, and a pair is split over at most 148 / pairs CTAs, so
// at most 148 partial slots are ever used (296 kept for headroom)
constexpr int64_t kMaxPartialSlots = 296;

static size_t attend_ws(const csa2_query_batch* qb, int Hq, int D) {
  Carve c{nullptr, 0};
  c.take((size_t)kMaxPartialSlots * Hq * D * 4);
  c.take((size_t)kMaxPartialSlots * Hq * 2 * 4);
  c.take((size_t)qb->n_tok * kMaxAttLayers * 4);  // split arrival counters
  return c.used + 256;
}

// ---------------------------------------------------------------- launches
// every job of `J` (jobs with no rows dropped) in one launch
static int launch_quantize_jobs(QuantJobs& J, cudaStream_t st) {
  const int64_t total = J.begin[J.n];
  if (total == 0) return CSA2_OK;
  int64_t grid = (total + 255) / 256;
  if (grid > 148 * 32) grid = 148 * 32;
  Launch L_("quantize_fp4", st);
  return cuda_check(
      launch_overlapped(kOverlapQuantize, k_quantize_fp4, dim3((unsigned)grid), dim3(256), 0, st, J, status_ptr()),
      "k_quantize_fp4");
}

// appends a job of `rows` rows to J (returns false when J is full)
static bool add_quant_job(QuantJobs& J, const float* x, int64_t rows, int dim, const int64_t* slot, uint8_t* codes,
                          uint8_t* scales) {
  if (rows <= 0) return true;
  if (J.n >= kQuantJobs) return false;
  J.job[J.n] = QuantJob{x, slot, codes, scales, dim};
  J.begin[J.n + 1] = J.begin[J.n] + rows * (dim / 8);
  ++J.n;
  return true;
}

int launch_quantize(const float* x, int64_t n_rows, int dim, const int64_t* slot, uint8_t* codes, uint8_t* scales,
                    cudaStream_t st) {
  QuantJobs J{};
  add_quant_job(J, x, n_rows, dim, slot, codes, scales);
  return launch_quantize_jobs(J, st);
}

static int launch_scan(const csa2_query_batch* qb, const uint8_t* qc, const uint8_t* qs, const float* w, int H,
                       const csa2_fp4_cache* kc, float* bs, int64_t ld, uint32_t* hist, cudaStream_t st) {
  return launch_scan_tc(qb, qc, qs, w, H, kc, bs, ld, hist, st);
}

// n_sel selector layers (queries [n_sel][T][H][...], weights w[i], scores
// [n_sel][T][8P]), up to kMaxSel in one launch; hist: the groups' key counts
// for the selection that follows (NULL: none)
static int launch_rescore_multi(const csa2_query_batch* qb, const uint8_t* qc, const uint8_t* qs,
                                const float* const* w, int n_sel, int H, const csa2_fp4_cache* kc,
                                const int32_t* pool, const int32_t* pool_n, int P, float* scores, uint32_t* hist,
                                cudaStream_t st) {
  return launch_rescore_tc(qb, qc, qs, w, n_sel, H, kc, pool, pool_n, P, scores, hist, st);
}

int launch_rescore(const csa2_query_batch* qb, const uint8_t* qc, const uint8_t* qs, const float* w, int H,
                   const csa2_fp4_cache* kc, const int32_t* pool, const int32_t* pool_n, int P, float* scores,
                   cudaStream_t st) {
  return launch_rescore_multi(qb, qc, qs, &w, 1, H, kc, pool, pool_n, P, scores, nullptr, st);
}

// SMs of the current device
static int num_sms_dev() {
  static int n[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!n[dev]) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    n[dev] = v > 0 ? v : 148;
  }
  return n[dev];
}

static int launch_select_multi(const csa2_query_batch* qb, const float* score, int64_t ld, int mode,
                               const int32_t* pool, const int32_t* pool_n, int P, int k_out, int32_t* out,
                               int32_t* out_n, int n_sel, cudaStream_t st);

// n_sel score matrices [n_sel][T][ld] -> lists [n_sel][T][k_out], counts
// [n_sel][T], seeded by the scoring kernel's key counts `hist`
// (k_select_cluster: the group's candidates split over a cluster of S CTAs
// while there are fewer groups than SMs)
static int launch_select_cluster(const csa2_query_batch* qb, const float* score, int64_t ld, int mode,
                                 const int32_t* pool, const int32_t* pool_n, int P, int k_out, int32_t* out,
                                 int32_t* out_n, int n_sel, uint32_t* hist, cudaStream_t st) {
  if (qb->n_tok > 65535 || n_sel > 65535) return fail(CSA2_ERR_UNSUPPORTED, "more than 65535 query tokens");
  const int64_t groups = (int64_t)qb->n_tok * n_sel;
  const int n_max = std::max(1, mode == 0 ? n_blocks_max(qb) : P * kBlock);
  SelCParams sp{};
  sp.qb = *qb;
  sp.score = score;
  sp.ld = ld;
  sp.mode = mode;
  sp.pool = pool;
  sp.pool_n = pool_n;
  sp.P = P;
  sp.k_out = k_out;
  sp.out = out;
  sp.out_n = out_n;
  sp.hist = hist;
  sp.words = (n_max + 31) / 32;
  sp.cap = std::min(kSelCandCap, n_max);
  sp.status = status_ptr();
  const SelCLayout lay(sp.words, sp.cap, mode == 1 ? P : 0);
  // the group's bitmaps, candidates and pool row in one CTA's shared memory;
  // longer candidate lists (contexts beyond about 4.7M positions) take the
  // selection without key counts
  constexpr int kDynMax = 200 * 1024;
  if (lay.bytes > (uint32_t)kDynMax)
    return launch_select_multi(qb, score, ld, mode, pool, pool_n, P, k_out, out, out_n, n_sel, st);
  static bool attr_done[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    if (int rc = cuda_check(cudaFuncSetAttribute(k_select_cluster, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 kDynMax),
                            "select smem attribute"))
      return rc;
    if (int rc = cuda_check(
            cudaFuncSetAttribute(k_select_cluster, cudaFuncAttributeNonPortableClusterSizeAllowed, 1),
            "select cluster attribute"))
      return rc;
    attr_done[dev] = true;
  }
  // CTAs per group: about 4096 candidates each (measured: 8192 and 2048
  // slower where the groups are few), a power of two <= 16, the whole grid
  // within the SMs, and a cluster shape the GPU can place
  int S = 1;
  const int sms = std::min(num_sms_dev(), kSelMaxGroups);
  if (groups < sms) {
    int want = (int)std::min<int64_t>({(int64_t)(n_max + 4095) / 4096, 16, sms / groups});
    while (S * 2 <= want) S *= 2;
  }
  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute at[2];
  cfg.blockDim = dim3(kSelThreads);
  cfg.dynamicSmemBytes = lay.bytes;
  cfg.stream = st;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  for (;; S /= 2) {
    cfg.gridDim = dim3(S, qb->n_tok, n_sel);
    at[0].val.clusterDim.x = S;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    int nc = 0;
    if (S == 1 || (cudaOccupancyMaxActiveClusters(&nc, k_select_cluster, &cfg) == cudaSuccess && nc >= 1)) break;
    cudaGetLastError();  // a refused shape is not an error of the call
  }
  cfg.numAttrs = overlap_launches(kOverlapSelect) ? 2 : 1;
  Launch L_(mode == 0 ? "select_blocks" : "select_positions", st);
  return cuda_check(cudaLaunchKernelEx(&cfg, k_select_cluster, sp), "k_select_cluster");
}

// the same without key counts (one CTA per group, k_select's own rounds)
static int launch_select_multi(const csa2_query_batch* qb, const float* score, int64_t ld, int mode,
                               const int32_t* pool, const int32_t* pool_n, int P, int k_out, int32_t* out,
                               int32_t* out_n, int n_sel, cudaStream_t st) {
  if (qb->n_tok > 65535 || n_sel > 65535) return fail(CSA2_ERR_UNSUPPORTED, "more than 65535 query tokens");
  SelParams sp{};
  sp.qb = *qb;
  sp.score = score;
  sp.ld = ld;
  sp.mode = mode;
  sp.pool = pool;
  sp.pool_n = pool_n;
  sp.P = P;
  sp.k_out = k_out;
  sp.out = out;
  sp.out_n = out_n;
  sp.status = status_ptr();
  const dim3 grid(1, qb->n_tok, n_sel);
  Launch L_(mode == 0 ? "select_blocks" : "select_positions", st);
  return cuda_check(launch_overlapped(kOverlapSelect, k_select, grid, dim3(kSelThreads), 0, st, sp), "k_select");
}

int launch_select(const csa2_query_batch* qb, const float* score, int64_t ld, int mode, const int32_t* pool,
                  const int32_t* pool_n, int P, int k_out, int32_t* out, int32_t* out_n, cudaStream_t st) {
  return launch_select_multi(qb, score, ld, mode, pool, pool_n, P, k_out, out, out_n, 1, st);
}

// Attention of n_layers (<= kMaxAttLayers) layers, each with its own index
// list, in one launch.  ws: attend_ws() bytes.
int launch_attend_layers(const csa2_query_batch* qb, int q_dtype, int Hq, const csa2_fp4_cache* kv, int K,
                         const AttendLayer* layers, int n_layers, float scale, int out_dtype, void* ws,
                         cudaStream_t st) {
  const int D = kv->dim;
  const csa2_swa_desc* swa = layers[0].swa;
  if (!attend_tc_supported(D, Hq, q_dtype)) return fail(CSA2_ERR_UNSUPPORTED, "attention shape D=%d Hq=%d", D, Hq);
  Carve c{static_cast<uint8_t*>(ws), ~size_t(0)};
  float* part_o = static_cast<float*>(c.take((size_t)kMaxPartialSlots * Hq * D * 4));
  float* part_ml = static_cast<float*>(c.take((size_t)kMaxPartialSlots * Hq * 2 * 4));
  int* done = static_cast<int*>(c.take((size_t)qb->n_tok * kMaxAttLayers * 4));
  // 64-row chunks; with fewer than 148 (token, layer) pairs one token's
  // chunks are spread over up to 4 CTAs (one wave of one CTA per SM), whose
  // partials the last one merges
  const int chunks = (K + 63) / 64 + (swa ? (swa->window + 63) / 64 : 0);
  const int64_t pairs = (int64_t)qb->n_tok * n_layers;
  int nsplit = 1;
  if (pairs < 148) nsplit = (int)std::max<int64_t>(1, std::min<int64_t>(std::min(chunks, 4), 148 / pairs));
  if (nsplit > 1) {
    if (int rc = cuda_check(cudaMemsetAsync(done, 0, (size_t)pairs * 4, st), "clear split counters")) return rc;
  }
  return launch_attend_tc(qb, q_dtype, Hq, kv, K, layers, n_layers, scale, out_dtype, part_o, part_ml, done, nsplit,
                          st);
}

int launch_attend(const csa2_query_batch* qb, const void* q, int q_dtype, int Hq, const csa2_fp4_cache* kv,
                  const int32_t* idx, const int32_t* idx_n, int K, const csa2_swa_desc* swa, float scale, void* out,
                  int out_dtype, float* lse, void* ws, cudaStream_t st) {
  AttendLayer one{idx, idx_n, q, out, lse, swa};
  return launch_attend_layers(qb, q_dtype, Hq, kv, K, &one, 1, scale, out_dtype, ws, st);
}

}  // namespace csa2

using namespace csa2;

// ============================================================================
// C ABI
// ============================================================================
extern "C" {

const char* csa2_last_error(void) { return t_err; }

int csa2_version(void) { return 100; }

int csa2_get_status(void* stream) {
  int rc = cuda_check(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)), "cudaStreamSynchronize");
  if (rc) return rc;
  int v = 0, zero = 0;
  rc = cuda_check(cudaMemcpyFromSymbol(&v, g_status, sizeof(int)), "read status");
  if (rc) return rc;
  rc = cuda_check(cudaMemcpyToSymbol(g_status, &zero, sizeof(int)), "clear status");
  if (rc) return rc;
  return v;
}

int csa2_quantize_fp4(const float* x, int64_t n_rows, int32_t dim, const int64_t* slot, uint8_t* codes,
                      uint8_t* scales, void* stream) {
  t_err[0] = 0;
  if (n_rows < 0) return fail(CSA2_ERR_INVALID_ARG, "n_rows < 0");
  if (dim < 32 || dim > 8192 || dim % 32) return fail(CSA2_ERR_UNSUPPORTED, "dim %d unsupported", dim);
  if (n_rows > 0 && (!x || !codes || !scales)) return fail(CSA2_ERR_INVALID_ARG, "NULL buffer");
  if (reinterpret_cast<uintptr_t>(x) % 16 || reinterpret_cast<uintptr_t>(codes) % 4)
    return fail(CSA2_ERR_INVALID_ARG, "x must be 16-byte aligned and codes 4-byte aligned");
  return launch_quantize(x, n_rows, dim, slot, codes, scales, static_cast<cudaStream_t>(stream));
}

int csa2_index_workspace_size(const csa2_query_batch* qb, int32_t H_I, int32_t d_I, int32_t P, int32_t K,
                              size_t* bytes) {
  t_err[0] = 0;
  if (int rc = check_batch(qb)) return rc;
  if (!bytes || P < 1 || K < 1 || H_I < 1) return fail(CSA2_ERR_INVALID_ARG, "bad arguments");
  (void)d_I;
  *bytes = index_ws(qb, P);
  return CSA2_OK;
}

int csa2_attend_workspace_size(const csa2_query_batch* qb, int32_t Hq, int32_t D, int32_t K, int32_t has_swa,
                               size_t* bytes) {
  t_err[0] = 0;
  if (int rc = check_batch(qb)) return rc;
  if (!bytes || Hq < 1 || D < 32 || K < 1) return fail(CSA2_ERR_INVALID_ARG, "bad arguments");
  (void)has_swa;
  *bytes = attend_ws(qb, Hq, D);
  return CSA2_OK;
}

static int check_index_common(const csa2_query_batch* qb, const uint8_t* qc, const uint8_t* qs, const float* w,
                              int H_I, const csa2_fp4_cache* kc, int P, int K) {
  if (int rc = check_batch(qb)) return rc;
  if (int rc = check_cache(kc, "k_idx", qb)) return rc;
  if (!qc || !qs || !w) return fail(CSA2_ERR_INVALID_ARG, "indexer query buffers must be non-NULL");
  if (kc->dim != 64 && kc->dim != 128) return fail(CSA2_ERR_UNSUPPORTED, "d_I must be 64 or 128");
  if ((kc->n_rows * (kc->dim / 32)) % 16)
    return fail(CSA2_ERR_UNSUPPORTED, "indexer cache: n_rows * d_I / 32 must be a multiple of 16");
  if (H_I < 1 || H_I > 64) return fail(CSA2_ERR_UNSUPPORTED, "H_I must be in [1, 64]");
  if (P < 1 || P > 4096) return fail(CSA2_ERR_UNSUPPORTED, "P must be in [1, 4096]");
  if (K < 1 || K > 2048 || K > P * kBlock) return fail(CSA2_ERR_UNSUPPORTED, "K must be in [1, min(2048, 8P)]");
  return CSA2_OK;
}

}  // extern "C"

namespace csa2 {
int check_index_args(const csa2_query_batch* qb, const uint8_t* qc, const uint8_t* qs, const float* w, int H_I,
                     const csa2_fp4_cache* kc, int P, int K) {
  return check_index_common(qb, qc, qs, w, H_I, kc, P, K);
}
void clear_last_error() { t_err[0] = 0; }
}  // namespace csa2

extern "C" {

int csa2_index_full(const csa2_query_batch* qb, const uint8_t* q_codes, const uint8_t* q_scales, const float* w,
                    int32_t H_I, const csa2_fp4_cache* k_idx, int32_t P, int32_t K, int32_t* pool, int32_t* pool_n,
                    int32_t* idx, int32_t* idx_n, float* blockscore, void* workspace, size_t workspace_bytes,
                    void* stream) {
  t_err[0] = 0;
  if (int rc = check_index_common(qb, q_codes, q_scales, w, H_I, k_idx, P, K)) return rc;
  if (!pool || !pool_n || !idx || !idx_n) return fail(CSA2_ERR_INVALID_ARG, "output buffers must be non-NULL");
  if (!workspace || reinterpret_cast<uintptr_t>(workspace) % 256 || workspace_bytes < index_ws(qb, P))
    return fail(CSA2_ERR_WORKSPACE, "workspace too small or misaligned (need %zu)", index_ws(qb, P));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Carve c{static_cast<uint8_t*>(workspace), workspace_bytes};
  const int64_t ld = n_blocks_max(qb);
  float* bs = static_cast<float*>(c.take((size_t)qb->n_tok * ld * 4));
  float* sc = static_cast<float*>(c.take((size_t)qb->n_tok * P * kBlock * 4));
  const SelPlan sp = take_select_scratch(c, qb, P, 1);
  if (blockscore) bs = blockscore;
  if (int rc = clear_select_counts(sp, st)) return rc;
  if (int rc = launch_scan(qb, q_codes, q_scales, w, H_I, k_idx, bs, ld, sp.blk, st)) return rc;
  if (int rc = launch_select_cluster(qb, bs, ld, 0, nullptr, nullptr, P, P, pool, pool_n, 1, sp.blk, st)) return rc;
  if (int rc = launch_rescore_multi(qb, q_codes, q_scales, &w, 1, H_I, k_idx, pool, pool_n, P, sc, sp.pos, st))
    return rc;
  return launch_select_cluster(qb, sc, (int64_t)P * kBlock, 1, pool, pool_n, P, K, idx, idx_n, 1, sp.pos, st);
}

int csa2_index_reindex(const csa2_query_batch* qb, const uint8_t* q_codes, const uint8_t* q_scales, const float* w,
                       int32_t H_I, const csa2_fp4_cache* k_idx, const int32_t* pool, const int32_t* pool_n,
                       int32_t P, int32_t K, int32_t* idx, int32_t* idx_n, void* workspace, size_t workspace_bytes,
                       void* stream) {
  t_err[0] = 0;
  if (int rc = check_index_common(qb, q_codes, q_scales, w, H_I, k_idx, P, K)) return rc;
  if (!pool || !pool_n || !idx || !idx_n) return fail(CSA2_ERR_INVALID_ARG, "pool/idx buffers must be non-NULL");
  if (!workspace || reinterpret_cast<uintptr_t>(workspace) % 256 || workspace_bytes < index_ws(qb, P))
    return fail(CSA2_ERR_WORKSPACE, "workspace too small or misaligned (need %zu)", index_ws(qb, P));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Carve c{static_cast<uint8_t*>(workspace), workspace_bytes};
  c.take((size_t)qb->n_tok * n_blocks_max(qb) * 4);
  float* sc = static_cast<float*>(c.take((size_t)qb->n_tok * P * kBlock * 4));
  const SelPlan sp = take_select_scratch(c, qb, P, 1);
  if (int rc = clear_select_counts(sp, st)) return rc;
  if (int rc = launch_rescore_multi(qb, q_codes, q_scales, &w, 1, H_I, k_idx, pool, pool_n, P, sc, sp.pos, st))
    return rc;
  return launch_select_cluster(qb, sc, (int64_t)P * kBlock, 1, pool, pool_n, P, K, idx, idx_n, 1, sp.pos, st);
}

static int check_attend(const csa2_query_batch* qb, const void* q, int q_dtype, int Hq, const csa2_fp4_cache* kv,
                        bool have_idx, int K, const csa2_swa_desc* swa, void* out, int out_dtype) {
  if (int rc = check_batch(qb)) return rc;
  if (int rc = check_cache(kv, "kv", qb)) return rc;
  if (kv->dim != 128 && kv->dim != 512) return fail(CSA2_ERR_UNSUPPORTED, "D must be 128 or 512");
  if (Hq != 16 && Hq != 32 && Hq != 64) return fail(CSA2_ERR_UNSUPPORTED, "Hq must be 16, 32 or 64");
  if (K < 1 || K > 2048) return fail(CSA2_ERR_UNSUPPORTED, "K must be in [1, 2048]");
  if (!q || !have_idx || !out) return fail(CSA2_ERR_INVALID_ARG, "NULL buffer");
  if ((q_dtype != CSA2_F32 && q_dtype != CSA2_BF16) || (out_dtype != CSA2_F32 && out_dtype != CSA2_BF16))
    return fail(CSA2_ERR_INVALID_ARG, "bad dtype");
  if (q_dtype == CSA2_F32 && kv->dim * Hq > 16384)
    return fail(CSA2_ERR_UNSUPPORTED, "fp32 queries need D * Hq <= 16384 (use bf16 queries)");
  if (swa) {
    if (!swa->codes || !swa->scale) return fail(CSA2_ERR_INVALID_ARG, "swa buffers missing");
    if (swa->dim != kv->dim) return fail(CSA2_ERR_INVALID_ARG, "swa dim must equal the Main KV dim");
    if (swa->window < 1 || swa->window > 256) return fail(CSA2_ERR_UNSUPPORTED, "swa window must be in [1,256]");
    if (swa->cap < swa->window + qb->max_q_per_seq - 1)
      return fail(CSA2_ERR_INVALID_ARG, "swa cap must be >= window + max_q_per_seq - 1");
  }
  return CSA2_OK;
}

int csa2_attend_reuse(const csa2_query_batch* qb, const void* q, int32_t q_dtype, int32_t Hq, const csa2_fp4_cache* kv,
                      const int32_t* idx, const int32_t* idx_n, int32_t K, const csa2_swa_desc* swa,
                      float softmax_scale, void* out, int32_t out_dtype, float* lse, void* workspace,
                      size_t workspace_bytes, void* stream) {
  t_err[0] = 0;
  if (int rc = check_attend(qb, q, q_dtype, Hq, kv, idx && idx_n, K, swa, out, out_dtype)) return rc;
  size_t need = attend_ws(qb, Hq, kv->dim);
  if (!workspace || reinterpret_cast<uintptr_t>(workspace) % 256 || workspace_bytes < need)
    return fail(CSA2_ERR_WORKSPACE, "workspace too small or misaligned (need %zu)", need);
  float scale = softmax_scale > 0.0f ? softmax_scale : 1.0f / std::sqrt((float)kv->dim);
  return launch_attend(qb, q, q_dtype, Hq, kv, idx, idx_n, K, swa, scale, out, out_dtype, lse, workspace,
                       static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------- stack
// Selector layers (FULL, REINDEX) each produce one index list; a REUSE layer
// attends over the list of the nearest selector before it.
static int count_selectors(const csa2_stack_desc* d) {
  int n = 0;
  for (int l = 0; l < d->n_layers; ++l) n += d->layers[l].mode != CSA2_MODE_REUSE;
  return n;
}

static size_t stack_ws(const csa2_stack_desc* d, size_t* sub_off) {
  const csa2_query_batch* qb = &d->qb;
  const int dI = d->k_idx.dim, T = qb->n_tok;
  const int ns = count_selectors(d);
  Carve c{nullptr, 0};
  c.take((size_t)ns * T * d->H_I * (dI / 2));   // quantised indexer queries, every selector
  c.take((size_t)ns * T * d->H_I * (dI / 32));  // and their scales
  c.take((size_t)T * d->P * 4);                 // pool
  c.take((size_t)T * 4);                        // pool_n
  c.take((size_t)ns * T * d->K * 4);            // index lists, every selector
  c.take((size_t)ns * T * 4);                   // list lengths
  Carve ix{nullptr, 0};
  ix.take((size_t)T * n_blocks_max(qb) * 4);                             // block scores
  ix.take((size_t)std::min(ns, kMaxSel) * T * d->P * kBlock * 4);        // pool position scores
  ix.take(select_ws(qb, d->P, std::min(ns, kMaxSel)));                  // selection scratch
  size_t sub = ix.used + 256;
  sub = std::max(sub, attend_ws(qb, d->Hq, d->kv.dim));
  c.take(0);
  *sub_off = c.used;
  c.take(sub);
  return c.used + 256;
}

int csa2_stack_workspace_size(const csa2_stack_desc* d, size_t* bytes) {
  t_err[0] = 0;
  if (!d || !bytes) return fail(CSA2_ERR_INVALID_ARG, "NULL argument");
  if (int rc = check_batch(&d->qb)) return rc;
  if (d->n_layers < 1 || !d->layers) return fail(CSA2_ERR_INVALID_ARG, "no layers");
  size_t off;
  *bytes = stack_ws(d, &off);
  return CSA2_OK;
}

static int copy_i32(const int32_t* src, int32_t* dst, int64_t n, cudaStream_t st) {
  Launch L_("copy", st);
  k_copy_i32<<<64, 256, 0, st>>>(src, dst, n);
  return cuda_check(cudaGetLastError(), "copy");
}

int csa2_decode_stack(const csa2_stack_desc* d, void* workspace, size_t workspace_bytes, void* stream) {
  t_err[0] = 0;
  if (!d) return fail(CSA2_ERR_INVALID_ARG, "desc is NULL");
  const csa2_query_batch* qb = &d->qb;
  if (int rc = check_batch(qb)) return rc;
  if (d->n_layers < 1 || !d->layers) return fail(CSA2_ERR_INVALID_ARG, "no layers");
  if (d->layers[0].mode != CSA2_MODE_FULL) return fail(CSA2_ERR_INVALID_ARG, "layer 0 must be FULL");
  for (int l = 0; l < d->n_layers; ++l) {
    const csa2_layer_desc& L = d->layers[l];
    if (L.mode < CSA2_MODE_FULL || L.mode > CSA2_MODE_REUSE) return fail(CSA2_ERR_INVALID_ARG, "layer %d: bad mode", l);
    if (L.mode != CSA2_MODE_REUSE && (!L.iq || !L.iw))
      return fail(CSA2_ERR_INVALID_ARG, "layer %d: selector layer needs iq and iw", l);
    if (int rc = check_attend(qb, L.q, d->q_dtype, d->Hq, &d->kv, true, d->K, L.swa, L.out, d->out_dtype))
      return rc;
  }
  if (int rc = check_cache(&d->k_idx, "k_idx", qb)) return rc;
  if (d->k_idx.dim != 64 && d->k_idx.dim != 128) return fail(CSA2_ERR_UNSUPPORTED, "d_I must be 64 or 128");
  if ((d->k_idx.n_rows * (d->k_idx.dim / 32)) % 16)
    return fail(CSA2_ERR_UNSUPPORTED, "indexer cache: n_rows * d_I / 32 must be a multiple of 16");
  if (d->H_I < 1 || d->H_I > 64 || d->P < 1 || d->P > 4096 || d->K < 1 || d->K > 2048 || d->K > d->P * kBlock)
    return fail(CSA2_ERR_UNSUPPORTED, "H_I/P/K out of the supported range");
  size_t sub_off;
  size_t need = stack_ws(d, &sub_off);
  if (!workspace || reinterpret_cast<uintptr_t>(workspace) % 256 || workspace_bytes < need)
    return fail(CSA2_ERR_WORKSPACE, "workspace too small or misaligned (need %zu)", need);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int T = qb->n_tok, dI = d->k_idx.dim, NL = d->n_layers;
  const int n_sel = count_selectors(d);
  const size_t q_codes_sz = (size_t)T * d->H_I * (dI / 2), q_scales_sz = (size_t)T * d->H_I * (dI / 32);
  Carve c{static_cast<uint8_t*>(workspace), workspace_bytes};
  uint8_t* qc = static_cast<uint8_t*>(c.take(n_sel * q_codes_sz));
  uint8_t* qsc = static_cast<uint8_t*>(c.take(n_sel * q_scales_sz));
  int32_t* pool = static_cast<int32_t*>(c.take((size_t)T * d->P * 4));
  int32_t* pool_n = static_cast<int32_t*>(c.take((size_t)T * 4));
  int32_t* idx = static_cast<int32_t*>(c.take((size_t)n_sel * T * d->K * 4));
  int32_t* idx_n = static_cast<int32_t*>(c.take((size_t)n_sel * T * 4));
  uint8_t* sub = static_cast<uint8_t*>(workspace) + sub_off;
  size_t sub_bytes = workspace_bytes - sub_off;
  const float scale = d->softmax_scale > 0.0f ? d->softmax_scale : 1.0f / std::sqrt((float)d->kv.dim);

  // selector layers in order, and each layer's selector
  std::vector<int> sel_layer;
  std::vector<int> layer_sel(NL);
  for (int l = 0; l < NL; ++l) {
    if (d->layers[l].mode != CSA2_MODE_REUSE) sel_layer.push_back(l);
    layer_sel[l] = (int)sel_layer.size() - 1;
  }
  if (d->new_k_idx && !d->new_slot_k_idx) return fail(CSA2_ERR_INVALID_ARG, "new_k_idx needs new_slot_k_idx");
  if (d->new_kv && !d->new_slot_kv) return fail(CSA2_ERR_INVALID_ARG, "new_kv needs new_slot_kv");
  Carve sc_c{sub, sub_bytes};
  const int64_t ld = n_blocks_max(qb);
  float* bs = static_cast<float*>(sc_c.take((size_t)T * ld * 4));
  float* sc = static_cast<float*>(sc_c.take((size_t)std::min(n_sel, kMaxSel) * T * d->P * kBlock * 4));
  const SelPlan sel = take_select_scratch(sc_c, qb, d->P, std::min(n_sel, kMaxSel));
  // cleared first, so that the step's kernels follow one another directly
  if (int rc = clear_select_counts(sel, st)) return rc;
  // this step's appended keys and Main KV rows and every selector's indexer
  // queries: one quantisation launch (more when there are many selectors)
  {
    QuantJobs J{};
    if (d->new_k_idx) add_quant_job(J, d->new_k_idx, T, dI, d->new_slot_k_idx, d->k_idx.codes, d->k_idx.scales);
    if (d->new_kv) add_quant_job(J, d->new_kv, T, d->kv.dim, d->new_slot_kv, d->kv.codes, d->kv.scales);
    for (int si = 0; si < n_sel; ++si) {
      const float* x = d->layers[sel_layer[si]].iq;
      if (!add_quant_job(J, x, (int64_t)T * d->H_I, dI, nullptr, qc + si * q_codes_sz, qsc + si * q_scales_sz)) {
        if (int rc = launch_quantize_jobs(J, st)) return rc;
        J = QuantJobs{};
        add_quant_job(J, x, (int64_t)T * d->H_I, dI, nullptr, qc + si * q_codes_sz, qsc + si * q_scales_sz);
      }
    }
    if (int rc = launch_quantize_jobs(J, st)) return rc;
  }
  // each FULL layer builds the pool that it and the REINDEX layers after it
  // rescore; the rescoring and position selection of consecutive selectors
  // run up to kMaxSel at a time
  int s = 0;
  while (s < n_sel) {
    const csa2_layer_desc& F = d->layers[sel_layer[s]];
    if (F.mode == CSA2_MODE_FULL) {
      if (int rc = launch_scan(qb, qc + s * q_codes_sz, qsc + s * q_scales_sz, F.iw, d->H_I, &d->k_idx, bs, ld,
                               sel.blk, st))
        return rc;
      if (int rc = launch_select_cluster(qb, bs, ld, 0, nullptr, nullptr, d->P, d->P, pool, pool_n, 1, sel.blk, st))
        return rc;
      if (F.pool_out)
        if (int rc = copy_i32(pool, F.pool_out, (int64_t)T * d->P, st)) return rc;
    }
    int n = 1;
    while (s + n < n_sel && n < kMaxSel && d->layers[sel_layer[s + n]].mode != CSA2_MODE_FULL) ++n;
    const float* ws[kMaxSel];
    for (int i = 0; i < n; ++i) ws[i] = d->layers[sel_layer[s + i]].iw;
    if (int rc = launch_rescore_multi(qb, qc + s * q_codes_sz, qsc + s * q_scales_sz, ws, n, d->H_I, &d->k_idx, pool,
                                      pool_n, d->P, sc, sel.pos, st))
      return rc;
    if (int rc = launch_select_cluster(qb, sc, (int64_t)d->P * kBlock, 1, pool, pool_n, d->P, d->K,
                                    idx + (size_t)s * T * d->K, idx_n + (size_t)s * T, n, sel.pos, st))
      return rc;
    for (int i = 0; i < n; ++i)
      if (int32_t* o = d->layers[sel_layer[s + i]].idx_out)
        if (int rc = copy_i32(idx + (size_t)(s + i) * T * d->K, o, (int64_t)T * d->K, st)) return rc;
    s += n;
  }
  // attention of every layer: consecutive layers alike in having a sliding
  // window or not, up to kMaxAttLayers per launch (after the caller's event,
  // when one is given: only attention reads the Main queries)
  if (d->attend_wait_event) {
    const cudaError_t e = cudaStreamWaitEvent(st, static_cast<cudaEvent_t>(d->attend_wait_event), 0);
    if (e != cudaSuccess) return fail(CSA2_ERR_CUDA, "cudaStreamWaitEvent: %s", cudaGetErrorString(e));
  }
  int l = 0;
  while (l < NL) {
    AttendLayer group[kMaxAttLayers];
    int ng = 0;
    const bool has_swa = d->layers[l].swa != nullptr;
    while (l < NL && ng < kMaxAttLayers && (d->layers[l].swa != nullptr) == has_swa) {
      const csa2_layer_desc& G = d->layers[l];
      const int si = layer_sel[l];
      group[ng++] = AttendLayer{idx + (size_t)si * T * d->K, idx_n + (size_t)si * T, G.q, G.out, G.lse, G.swa};
      ++l;
    }
    if (int rc = launch_attend_layers(qb, d->q_dtype, d->Hq, &d->kv, d->K, group, ng, scale, d->out_dtype, sub, st))
      return rc;
  }
  return CSA2_OK;
}

int csa2_profiler_enable(int on) {
  t_err[0] = 0;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof_on.store(on != 0);
  return CSA2_OK;
}

int csa2_profiler_read(csa2_kernel_stat* out, int32_t cap, int32_t* n_out) {
  t_err[0] = 0;
  if (!n_out || (cap > 0 && !out)) return fail(CSA2_ERR_INVALID_ARG, "NULL output");
  std::lock_guard<std::mutex> lk(g_prof_mu);
  std::map<std::string, std::pair<int64_t, double>> agg;
  int rc = CSA2_OK;
  for (auto& r : g_prof_recs) {
    float ms = 0.0f;
    cudaError_t e = cudaEventSynchronize(r.b);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, r.a, r.b);
    if (e != cudaSuccess && rc == CSA2_OK) rc = cuda_check(e, "profiler event");
    auto& a = agg[r.name];
    a.first += 1;
    a.second += ms;
    g_event_pool.push_back(r.a);
    g_event_pool.push_back(r.b);
  }
  g_prof_recs.clear();
  int n = 0;
  for (auto& kv : agg) {
    if (n < cap) {
      snprintf(out[n].name, sizeof(out[n].name), "%s", kv.first.c_str());
      out[n].launches = kv.second.first;
      out[n].total_ms = kv.second.second;
    }
    ++n;
  }
  *n_out = n < cap ? n : cap;
  return rc;
}

int64_t csa2_launch_count(void) { return g_launches.load(); }

int csa2_selftest_wait_timeout(int64_t limit_ns, void* stream) {
  t_err[0] = 0;
  if (limit_ns < 1000 || limit_ns > 10000000000LL) return fail(CSA2_ERR_INVALID_ARG, "limit_ns out of range");
  Launch L_("selftest_wait", static_cast<cudaStream_t>(stream));
  k_selftest_wait<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns, status_ptr());
  return cuda_check(cudaGetLastError(), "k_selftest_wait");
}

}  // extern "C"
