// scan_tc.cu -- the indexer scoring on the 5th-generation tensor cores
// (sm_100a): the Full layer's scan of the whole visible context (block scores)
// and the pool rescoring of the Full layer's own top-K and of every Reindex
// layer (position scores), one templated kernel.
//
// For every query token i of sequence b and visible position t <= p_i:
//   s_t = sum_h w[i][h] * max(0, q~_{i,h} . k~_t),   B_j = max_{t in block j} s_t
// (hierarchical indexer of the DeepSeek-V4.1-Flash pages, dbyun.net article
// 10794, section "KV Cache 成为这一代架构改造的核心": the first Full layer scans
// the whole visible context and keeps blocks of 8 positions; later layers
// rescore only the pool).
//
// Work: one persistent CTA per SM walks a contiguous range of (group, stage)
// items (its first item found by all threads with a block scan over the
// groups' stage counts).  A stage is 256 positions of the FP4 indexer K cache
// (two 128-row MMA tiles) when every sequence has one query token, else 128
// positions; a group is up to four "query columns" that share its stages: the
// scan's group is query tokens of one sequence (one pass over the sequence's
// keys per group), the rescoring's group is one query token and up to four
// selector layers (the token's pool is gathered once for all of them).
//
// Warp roles (20 warps):
//   0, 1    producers, alternate stages: scan, TMA boxes of up to 256 rows of
//           codes (in the 64B/32B swizzle the MMA reads) and of the rows'
//           per-32 E4M3 scales, loaded with an L2 evict-first policy (the key
//           stream is read once); rescoring, 16 pool blocks of 8 rows
//           gathered with per-lane 16-byte cp.async;
//   2, 3    MMA issuers, alternate stages: per tile and query column two
//           tcgen05.mma.kind::mxf4nvf4.block_scale.block16 (M = 128 positions,
//           N = heads, K = 64 each) into the column's part of a TMEM
//           accumulator slot, then one commit per stage, which frees the
//           stage for the producer and hands the slot to the epilogue;
//   4 .. 7  scale-factor warps, one per TMEM lane quarter: each writes the
//           stage's scales in the block-scale layout with tcgen05.st (each
//           per-32 scale twice: the MMA takes one UE4M3 scale per 16
//           elements) and arrives on the stage's scale barrier;
//   8 .. 19 epilogue, three warpgroups: a stage's units (tiles x columns) go
//           half to one warpgroup and half to the next, the warpgroups taking
//           stages in turn; TMEM -> registers (one position per thread),
//           ReLU, weighted head sum, block max over 8 lanes (scan) and the
//           score stores; the slot is released as soon as the last load of a
//           unit has landed.  Every score's key is counted by its top 12 bits
//           in shared memory; the counts go to the group's global histogram
//           (one atomic per non-empty bin) when the CTA leaves the group.
// A tcgen05 instruction costs its issuing thread 60-170 cycles and a TMA
// instruction several hundred, while different warps issue concurrently; the
// roles above keep every issuing thread's per-stage instruction count small.
// All waits are bounded; on timeout the kernel records CSA2_ERR_TIMEOUT,
// drains its own copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "internal.h"
#include "tc_common.cuh"

namespace csa2 {
namespace scan_tc {

constexpr int kTile = 128;      // positions per MMA tile = MMA M
constexpr int kMaxWc = 4;       // query columns per group at most
constexpr int kEpiWG = 3;       // epilogue warpgroups
constexpr int kThreads = 32 * (8 + 4 * kEpiWG);
constexpr int kProd0 = 0;       // producer warps 0, 1
constexpr int kMma0 = 2;        // MMA warps 2, 3
constexpr int kSf0 = 4;         // scale-factor warps 4..7 (lane quarters 0..3)
constexpr int kEpi0 = 8;        // epilogue warpgroups 8..11, 12..15, 16..19
constexpr uint32_t kTmemCols = 512;

// Shared-memory and TMEM maps for stages of kSub MMA tiles (kSub * 128
// positions; two tiles a stage halve every per-stage cost per position).
// The stage ring is even (producer and MMA warps take stages in turn).
template <int kSub>
struct Layout {
  static constexpr int kStages = kSub == 2 ? 6 : 12;
  static constexpr uint32_t kCodeStage = 8192u * kSub;               // kSub x 128 rows x <= 64 B
  static constexpr uint32_t kRawStage = kSub == 2 ? 1024u : 2048u;    // raw scales (rescoring: 16 boxes at 128 B)
  static constexpr uint32_t kColSfa = 0;                             // [kStages][kSub][8]
  static constexpr uint32_t kColSfb = kColSfa + kStages * 8 * kSub;  // [kMaxWc][8]
  static constexpr uint32_t kColAcc = kColSfb + kMaxWc * 8;          // accumulator slots
  static constexpr uint32_t kAccCols = kTmemCols - kColAcc;
  static constexpr uint32_t kOffA = 0;                               // [kStages][kCodeStage]
  static constexpr uint32_t kOffRaw = kOffA + kStages * kCodeStage;
  static constexpr uint32_t kOffB = kOffRaw + kStages * kRawStage;   // [kMaxWc][64 rows][64 B]
  static constexpr uint32_t kOffSfb = kOffB + kMaxWc * 4096;         // [kMaxWc][2][512]
  static constexpr uint32_t kOffW = kOffSfb + kMaxWc * 1024;         // [kEpiWG][kMaxWc][64] f32
  static constexpr uint32_t kOffPos = kOffW + kEpiWG * kMaxWc * 64 * 4;  // [kEpiWG][kMaxWc] i64 query positions
  // key counts of the current group, [query column][kHistBins] (a two-tile
  // stage serves one query column)
  static constexpr int kHistCols = kSub == 2 ? 1 : kMaxWc;
  static constexpr uint32_t kOffHist = kOffPos + kEpiWG * kMaxWc * 8;
  static constexpr uint32_t kOffBar = kOffHist + kHistCols * kHistBins * 4;
  static constexpr uint32_t kNumBars = 3 * kStages + 12 + 3;  // full, done, sf; acc_empty[6][2]; drain[2], sfb
  static constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;      // tmem base, abort flag
  static constexpr uint32_t kSmemBytes = kOffMisc + 16 + 1024;      // + alignment slack
  static_assert(kOffB % 1024 == 0, "B tiles must be 1024-aligned");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

struct Params {
  csa2_query_batch qb;
  const uint8_t* q_codes;   // [n_sel][T][H][d_I/2]
  const uint8_t* q_scales;  // [n_sel][T][H][d_I/32]
  const float* w[kMaxSel];  // per selector [T][H]
  int n_sel;                // rescore: selector layers (scan: 1)
  int cpg;                  // groups per sequence (scan) or per token (rescore)
  int wc;                   // query columns per group (<= kMaxWc)
  int H, Nh, DI;            // heads, heads padded to 16 (MMA N per column), key dim
  int slot_cols, n_slots;   // accumulator slots of (query columns x Nh) columns
  int box_rows;             // scan: rows per TMA box (256, 128, or 64 for 64-row pages)
  int rows;                 // positions per stage (kSub * 128)
  const uint8_t* codes;     // the indexer cache (rescoring gathers it directly)
  const uint8_t* scales;
  int64_t n_rows;
  int page_size, max_pages;
  const int32_t* page_table;
  const int64_t* seq_base;
  float* out;        // scan: block scores [T][ld]; rescore: pool-position scores [n_sel*T][ld]
  int64_t ld;
  const int32_t* pool;   // rescore: [T][pool_cap] block ids
  const int32_t* pool_n; // rescore: [T]
  int pool_cap;
  uint32_t* hist;        // key counts by the top 12 bits, [group][kHistBins] (group = selector * T + token), or NULL
  int* status;
  uint64_t wait_ns;
};

// Groups: scan group g = (sequence b, chunk c), c < cpg, holds the sequence's
// query tokens c*wc ..; rescore group g = (token t, chunk c), c < cpg, holds
// selectors c*wc ..
template <bool kRescore>
__device__ __forceinline__ int n_groups(const Params& P) {
  return (kRescore ? P.qb.n_tok : P.qb.n_seq) * P.cpg;
}

// group g: first query token, query columns (0: empty chunk), sequence, first selector
template <bool kRescore>
__device__ __forceinline__ void group_info(const Params& P, int g, int* tok0, int* W, int* b, int* sel0) {
  if (kRescore) {
    *tok0 = g / P.cpg;
    *sel0 = (g % P.cpg) * P.wc;
    *W = max(0, min(P.wc, P.n_sel - *sel0));
    *b = __ldg(P.qb.tok_seq + *tok0);
  } else {
    *b = g / P.cpg;
    *sel0 = 0;
    const int t_end = __ldg(P.qb.tok_start + *b + 1);
    *tok0 = __ldg(P.qb.tok_start + *b) + (g % P.cpg) * P.wc;
    *W = max(0, min(P.wc, t_end - *tok0));
  }
}

// stages of group g: scan, the 128-position tiles holding a position visible
// to one of its tokens; rescore, the token's pool in 16-block tiles
template <bool kRescore>
__device__ __forceinline__ int group_tiles(const Params& P, int g) {
  int tok0, W, b, sel0;
  group_info<kRescore>(P, g, &tok0, &W, &b, &sel0);
  if (W <= 0) return 0;
  if (kRescore) return (min(__ldg(P.pool_n + tok0), P.pool_cap) + 15) / 16;
  const int64_t vis = min((int64_t)__ldg(P.qb.tok_pos + tok0 + W - 1) + 1, (int64_t)__ldg(P.qb.seq_len + b));
  return (int)((max(vis, (int64_t)0) + P.rows - 1) / P.rows);
}

// This CTA's contiguous range of (group, stage) work in group-major order,
// found by all threads of the CTA together: each sums the stages of a run of
// consecutive groups, a block scan places the runs, and the thread whose run
// holds the CTA's first stage finds its group (a serial walk over every group
// cost up to a dependent load chain per group).  Results in shared memory:
// first group, first stage in it, number of stages (0: no work).
template <bool kRescore>
__device__ void work_start(const Params& P, long long* s_wsum, int* s_g0, int* s_t0, long long* s_n) {
  const int ng = n_groups<kRescore>(P);
  const int per = (ng + kThreads - 1) / kThreads;
  const int g_lo = min(ng, (int)threadIdx.x * per), g_hi = min(ng, g_lo + per);
  long long mine = 0;
  for (int g = g_lo; g < g_hi; ++g) mine += group_tiles<kRescore>(P, g);
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  long long incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) s_wsum[wid] = incl;
  if (threadIdx.x == 0) {
    *s_g0 = 0;
    *s_t0 = 0;
  }
  __syncthreads();
  long long before = 0, total = 0;
  for (int w = 0; w < kThreads / 32; ++w) {
    const long long v = s_wsum[w];
    if (w < wid) before += v;
    total += v;
  }
  const long long excl = before + incl - mine;
  const long long begin = total * blockIdx.x / gridDim.x, end = total * (blockIdx.x + 1) / gridDim.x;
  if (mine > 0 && begin < end && excl <= begin && begin < excl + mine) {  // one thread
    long long acc = excl;
    int g = g_lo;
    for (; g < g_hi - 1; ++g) {
      const int t = group_tiles<kRescore>(P, g);
      if (acc + t > begin) break;
      acc += t;
    }
    *s_g0 = g;
    *s_t0 = (int)(begin - acc);
  }
  if (threadIdx.x == 0) *s_n = end - begin;
  __syncthreads();
}

// iterator over the stages of [begin, end)
template <bool kRescore>
struct TileIter {
  int b, tile, ntile;  // b: group
  int64_t left;
  // start at stage t0 of group g0 (from work_start), n stages in all
  __device__ void init(const Params& P, int g0, int t0, int64_t n) {
    b = g0;
    tile = t0;
    left = n;
    ntile = n > 0 ? group_tiles<kRescore>(P, g0) : 0;
  }
  __device__ bool valid() const { return left > 0; }
  __device__ void next(const Params& P) {
    --left;
    if (++tile >= ntile && left > 0) {
      const int ng = n_groups<kRescore>(P);
      do {
        ++b;
        ntile = group_tiles<kRescore>(P, b);
      } while (ntile == 0 && b < ng - 1);
      tile = 0;
    }
  }
};

__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, const Params& P, volatile int* abort) {
  if (*abort) return false;
  if (mbar_wait_bounded(bar, parity, P.wait_ns)) return true;
  set_status(P.status, CSA2_ERR_TIMEOUT);
  *abort = 1;
  return false;
}

// the same for a whole warp, probed by lane 0 only
__device__ __forceinline__ bool warp_wait_or_abort(uint32_t bar, uint32_t parity, const Params& P,
                                                   volatile int* abort) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = wait_or_abort(bar, parity, P, abort);
  return __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
}

// cache row of position `pos` (0 <= pos < max_seq_len, so 32-bit) of
// sequence b, or -1 when outside the cache
__device__ __forceinline__ int64_t key_row(const Params& P, int b, int64_t pos, int64_t base) {
  int64_t row;
  if (P.page_table) {
    const uint32_t p32 = (uint32_t)pos, ps = (uint32_t)P.page_size;  // unsigned 32-bit divide: the short one
    const uint32_t q = p32 / ps;
    const int32_t pg = __ldg(P.page_table + (int64_t)b * P.max_pages + q);
    row = (int64_t)pg * P.page_size + (p32 - q * ps);
  } else {
    row = base + pos;
  }
  return (row >= 0 && row < P.n_rows) ? row : -1;
}

template <bool kRescore, int kSub>
__global__ void __launch_bounds__(kThreads, 1)
    k_index_tc(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_scales,
               const __grid_constant__ Params P) {
  using Lay = Layout<kSub>;
  constexpr int kStages = Lay::kStages;
  constexpr int kRows = kTile * kSub;  // positions per stage
  constexpr uint32_t kCodeStage = Lay::kCodeStage, kRawStage = Lay::kRawStage, kColSfa = Lay::kColSfa,
                     kColSfb = Lay::kColSfb, kColAcc = Lay::kColAcc, kOffA = Lay::kOffA, kOffRaw = Lay::kOffRaw,
                     kOffB = Lay::kOffB, kOffSfb = Lay::kOffSfb, kOffW = Lay::kOffW, kOffPos = Lay::kOffPos,
                     kOffBar = Lay::kOffBar, kOffMisc = Lay::kOffMisc, kOffHist = Lay::kOffHist;
  constexpr int kHistCols = Lay::kHistCols;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar_full = sbase + kOffBar;          // [kStages] TMA landed
  const uint32_t bar_done = bar_full + kStages * 8;   // [kStages] MMAs of the stage complete (commit)
  const uint32_t bar_sf = bar_done + kStages * 8;     // [kStages] scale factors in TMEM (4 warps)
  // [6 slots][2 MMA warps] accumulator slot read (4 warps): the epilogue
  // releases a slot on the barrier of the MMA warp that uses it next, so that
  // every barrier has one waiter and one releaser, both in stage order (a
  // barrier waited by two warps that take turns could be waited two phases
  // ahead, where its parity reads as complete)
  const uint32_t bar_acce = bar_sf + kStages * 8;
  const uint32_t bar_drain = bar_acce + 12 * 8;       // [2] MMA warps' drains
  const uint32_t bar_sfb = bar_drain + 2 * 8;         // query scale-factor copies
  volatile uint32_t* tmem_holder = reinterpret_cast<volatile uint32_t*>(smem + kOffMisc);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row_bytes = P.DI / 2, spr = P.DI / 32, ksteps = P.DI / 64;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      // scan: one arrival with the TMA byte count; rescoring: the 32 lanes of
      // the producer warp, each when its copies have landed
      mbar_init(bar_full + 8 * i, kRescore ? 32 : 1);
      mbar_init(bar_done + 8 * i, 1);
      mbar_init(bar_sf + 8 * i, 4);
    }
    // every epilogue unit of a stage (one MMA tile x query column) arrives
    // from its four warps; a stage with fewer units than the launch's widest
    // group weights its last unit's arrivals
    for (int i = 0; i < 12; ++i) mbar_init(bar_acce + 8 * i, 4 * kSub * P.wc);
    mbar_init(bar_drain, 1);
    mbar_init(bar_drain + 8, 1);
    mbar_init(bar_sfb, 1);
    *abort = 0;
    tc::fence_barrier_init();
    tc::tma_prefetch_desc(&tm_codes);
    tc::tma_prefetch_desc(&tm_scales);
  }
  if (warp == kMma0) {
    tc::tmem_alloc(sbase + kOffMisc, kTmemCols);
    tc::tmem_relinquish();
    tc::fence_before_sync();
  }
  uint32_t* hist_s = reinterpret_cast<uint32_t*>(smem + kOffHist);
  for (int i = threadIdx.x; i < kHistCols * kHistBins; i += kThreads) hist_s[i] = 0u;
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_holder;
  grid_dep_wait();  // the previous kernel's queries, pools and cleared counts

  __shared__ long long s_wsum[kThreads / 32], s_nwork;
  __shared__ int s_g0, s_t0;
  work_start<kRescore>(P, s_wsum, &s_g0, &s_t0, &s_nwork);
  const int w_g0 = s_g0, w_t0 = s_t0;
  const int64_t w_n = s_nwork;

  if (warp < kMma0) {
    // ------------------------------------------------------------ producers
    // lane k issues box k of the stage: scan 1 or 2 boxes of 128 / 64 rows,
    // rescore 16 pool blocks of 8 rows (codes and scales each)
    const int pw = warp - kProd0;
    const int box_rows = kRescore ? kBlock : P.box_rows;
    const int nbox = kRescore ? 16 : kRows / box_rows;
    const uint32_t tx = (uint32_t)kRows * row_bytes + (uint32_t)kRows * spr;
    TileIter<kRescore> ti;
    ti.init(P, w_g0, w_t0, w_n);
    int it = 0, s = 0;  // this CTA's stage count, ring stage
    uint32_t n = 0;     // use of the ring stage
    auto adv = [&]() {
      ++it;
      if (++s == kStages) {
        s = 0;
        ++n;
      }
    };
    int cur_g = -1, tok0 = 0, b = 0, np_g = 0;
    int64_t base = 0, len = 0;
    // rescore: lane e < 16 holds the pool id of block e of stage (pf_g,
    // pf_tile), loaded one stage of this warp ahead of its use
    int pf_g = -1, pf_tile = -1;
    int32_t pf_blk = -1;
    const uint64_t l2_ef = tc::l2_policy_evict_first();
    for (; ti.valid(); ti.next(P), adv()) {
      if ((it & 1) != pw || *abort) continue;
      if (lane == 0) {
        // the stage is free once the MMAs of its previous use completed
        if ((n == 0 || wait_or_abort(bar_done + 8 * s, (n - 1) & 1, P, abort)) && !kRescore)
          tc::mbar_arrive_expect_tx(bar_full + 8 * s, tx);
      }
      __syncwarp();
      if (*abort) continue;
      if (ti.b != cur_g) {
        cur_g = ti.b;
        int W, sel0;
        group_info<kRescore>(P, cur_g, &tok0, &W, &b, &sel0);
        len = __ldg(P.qb.seq_len + b);
        base = P.page_table ? 0 : __ldg(P.seq_base + b);
        if (kRescore) np_g = min(__ldg(P.pool_n + tok0), P.pool_cap);  // the token's pool size in blocks
      }
      if (kRescore) {
        // gather: 16 pool blocks of 8 rows, 16-byte asynchronous copies from
        // every lane (a TMA instruction per block and array would cost the
        // warp hundreds of cycles each); codes land in the swizzle the MMA
        // reads, each block's scales at its 128-byte slot.  Rows outside the
        // cache are zero-filled.
        int32_t blk = -1;
        if (lane < 16) {
          const int e = ti.tile * 16 + lane;
          blk = (pf_g == ti.b && pf_tile == ti.tile) ? pf_blk
                                                     : (e < np_g ? __ldg(P.pool + (int64_t)tok0 * P.pool_cap + e) : -1);
        }
        // this warp's next stage (two on), when in the same group: its pool
        // ids load while this stage's copies are issued
        if (ti.left > 2 && ti.tile + 2 < ti.ntile) {
          pf_g = ti.b;
          pf_tile = ti.tile + 2;
          const int e2 = pf_tile * 16 + lane;
          pf_blk = (lane < 16 && e2 < np_g) ? __ldg(P.pool + (int64_t)tok0 * P.pool_cap + e2) : -1;
        }
        int64_t my_row0 = -1;  // lane e < 16: first cache row of block e
        // (a block past the sequence holds no key: zero-filled, scored -inf)
        if (blk >= 0 && (int64_t)blk * kBlock < len) {
          const int64_t row0 = key_row(P, b, (int64_t)blk * kBlock, base);
          if (row0 >= 0 && ((row0 * spr) & 15) == 0) my_row0 = row0;
          else set_status(P.status, CSA2_ERR_RANGE);
        }
        // 16-byte chunks a code row: 1 << cshift (d_I is 64 or 128); shifts,
        // not divisions by a runtime value, keep this loop short
        const int cshift = P.DI == 128 ? 2 : 1;
        const uint32_t a_base = sbase + kOffA + s * kCodeStage;
        for (int c = lane; c < (kTile << cshift); c += 32) {
          const int r = c >> cshift, ch = c & ((1 << cshift) - 1);
          const int64_t row0 = __shfl_sync(0xffffffffu, my_row0, r / kBlock);
          const int64_t gr = row0 + r % kBlock;
          const bool in = row0 >= 0 && gr < P.n_rows;
          const int sch = (P.DI == 128) ? (ch ^ ((r >> 1) & 3)) : (ch ^ ((r >> 2) & 1));
          tc::cp_async_16(a_base + r * row_bytes + sch * 16, in ? P.codes + gr * row_bytes + ch * 16 : P.codes,
                          in ? 16u : 0u);
        }
        {
          const int per_blk = kBlock * spr / 16;  // scale chunks a block (2 or 1)
          const int e = lane / per_blk, h = lane % per_blk;
          const int64_t row0 = __shfl_sync(0xffffffffu, my_row0, min(e, 31));
          // bytes of this chunk inside the scale array (a block cut by the
          // cache's end keeps its first rows; the rest is zero-filled)
          const int64_t first = row0 + h * (16 / spr);
          const uint32_t nb = row0 >= 0 ? (uint32_t)max((int64_t)0, min((int64_t)16, (P.n_rows - first) * spr)) : 0u;
          if (e < 16)
            tc::cp_async_16(sbase + kOffRaw + s * kRawStage + e * 128 + h * 16,
                            nb ? P.scales + first * spr : P.scales, nb);
        }
        tc::cp_async_arrive_noinc(bar_full + 8 * s);  // the stage completes when all 32 lanes' copies landed
      } else if (lane < nbox) {
        int64_t pos0 = -1;
        pos0 = (int64_t)ti.tile * kRows + lane * box_rows;
        if (pos0 >= len) pos0 = -1;
        const int64_t row0 = pos0 >= 0 ? key_row(P, b, pos0, base) : -1;
        // out of the cache, or not 16-byte aligned in the scale array: the
        // box is read out of range (zeros) and the row reported
        int32_t ry = (int32_t)P.n_rows, sy = (int32_t)(P.n_rows * spr / 16);
        if (row0 >= 0 && ((row0 * spr) & 15) == 0) {
          ry = (int32_t)row0;
          sy = (int32_t)(row0 * spr / 16);
        } else if (pos0 >= 0) {
          set_status(P.status, CSA2_ERR_RANGE);
        }
        tc::tma_load_2d_hint(sbase + kOffA + s * kCodeStage + lane * box_rows * row_bytes, &tm_codes, bar_full + 8 * s,
                             0, ry, l2_ef);
        const uint32_t slot = (uint32_t)(box_rows * spr);
        tc::tma_load_2d_hint(sbase + kOffRaw + s * kRawStage + lane * slot, &tm_scales, bar_full + 8 * s, 0, sy, l2_ef);
      }
      __syncwarp();
    }
    // this thread's copies land before it leaves (the scale-factor warps also
    // wait for every stage's landing before the CTA ends)
    if (kRescore) tc::cp_async_wait_all();
  } else if (warp < kSf0) {
    // ------------------------------------------------------------ MMA issuers
    // Both walk every stage (both see every change of group) and issue the
    // MMAs of the stages of their parity.
    const int mw = warp - kMma0;
    const uint32_t my_drain = bar_drain + 8 * mw;
    const uint32_t idesc = tc::idesc_mxf4nvf4(128, P.Nh);
    const tc::SmemLayout sw = (P.DI == 128) ? tc::kSwizzle64B : tc::kSwizzle32B;
    const uint32_t sbo = 8u * row_bytes;  // 8 rows per swizzle atom
    TileIter<kRescore> ti;
    ti.init(P, w_g0, w_t0, w_n);
    int it = 0, s = 0, slot = 0;  // stage count, ring stage, accumulator slot
    uint32_t n = 0, u = 0;        // uses of the ring stage and of the slot
    auto adv = [&]() {
      ++it;
      if (++s == kStages) {
        s = 0;
        ++n;
      }
      if (++slot == P.n_slots) {
        slot = 0;
        ++u;
      }
    };
    uint32_t drain_n = 0, sfb_n = 0;
    int cur_g = -1, W = 0;
    // No early exit from this loop: both issuers meet at the same named
    // barriers; after a failed wait a warp keeps walking without issuing.
    for (; ti.valid(); ti.next(P), adv()) {
      if (ti.b != cur_g) {
        if (cur_g >= 0) {  // every MMA reading the old queries must finish first
          if (lane == 0) tc::commit(my_drain);
          __syncwarp();
          warp_wait_or_abort(my_drain, drain_n & 1, P, abort);
          ++drain_n;
        }
        tc::named_sync(5, 64);  // both issuers drained
        cur_g = ti.b;
        int tok0, b, sel0;
        group_info<kRescore>(P, cur_g, &tok0, &W, &b, &sel0);
        if (mw == 0 && !*abort) {
          // query rows of this group's columns: scan, its tokens; rescore,
          // selector (sel0 + j) of its token
          auto qrow = [&](int j) -> int64_t {
            return kRescore ? (int64_t)(sel0 + j) * P.qb.n_tok + tok0 : (int64_t)(tok0 + j);
          };
          // B operand: query codes, swizzled like the TMA-written A tiles,
          // in 16-byte asynchronous copies that are all in flight together
          // (heads past H zero-filled); a code row is 1 << cshift chunks
          // (shifts, not divisions by a runtime value: this loop is one
          // warp's serial work on the way to the first MMA)
          const int cshift = P.DI == 128 ? 2 : 1;
          for (int j = 0; j < W; ++j) {
            const uint8_t* src = P.q_codes + qrow(j) * P.H * row_bytes;
            const uint32_t dst = sbase + kOffB + j * 4096;
            for (int e = lane; e < (64 << cshift); e += 32) {
              const int n = e >> cshift, ch = e & ((1 << cshift) - 1);
              const int sch = (P.DI == 128) ? (ch ^ ((n >> 1) & 3)) : (ch ^ ((n >> 2) & 1));
              const bool in = n < P.H;
              tc::cp_async_16(dst + n * row_bytes + sch * 16, in ? src + n * row_bytes + ch * 16 : P.q_codes,
                              in ? 16u : 0u);
            }
          }
          // B scale factors, [m0 (32)][m1 (4)][k (4)] per 64-element K step:
          // lane m0 first loads the scale words of its heads m1*32 + m0 of
          // every column (all loads in flight together), then duplicates each
          // per-32 scale into the per-16 layout
          uint32_t hw[kMaxWc][4];
#pragma unroll
          for (int j = 0; j < kMaxWc; ++j)
#pragma unroll
            for (int m1 = 0; m1 < 4; ++m1) {
              const int n = m1 * 32 + lane;
              hw[j][m1] = 0u;
              if (j < W && n < P.H) {
                const uint8_t* sp = P.q_scales + (qrow(j) * P.H + n) * spr;
                hw[j][m1] = spr == 4 ? __ldg(reinterpret_cast<const uint32_t*>(sp))
                                     : (uint32_t)__ldg(reinterpret_cast<const uint16_t*>(sp));
              }
            }
#pragma unroll
          for (int j = 0; j < kMaxWc; ++j)
            for (int ks = 0; ks < ksteps; ++ks)
              if (j < W) {
                const uint32_t sel = ks == 0 ? 0x1100u : 0x3322u;
                *reinterpret_cast<uint4*>(smem + kOffSfb + (j * 2 + ks) * 512 + lane * 16) =
                    make_uint4(__byte_perm(hw[j][0], 0, sel), __byte_perm(hw[j][1], 0, sel),
                               __byte_perm(hw[j][2], 0, sel), __byte_perm(hw[j][3], 0, sel));
              }
          tc::cp_async_wait_all();
          tc::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tc::fence_after_sync();
            for (int j = 0; j < W; ++j)
              for (int ks = 0; ks < ksteps; ++ks)
                tc::cp_32x128b_warpx4(tmem + kColSfb + j * 8 + ks * 4,
                                      tc::smem_desc(sbase + kOffSfb + (j * 2 + ks) * 512, 16, 128, tc::kSwizzleNone));
            tc::commit(bar_sfb);
            wait_or_abort(bar_sfb, sfb_n & 1, P, abort);  // the copies landed before anyone issues
          }
          ++sfb_n;
        }
        tc::named_sync(6, 64);  // new queries in place
        tc::fence_after_sync();
      }
      if ((it & 1) != mw || *abort) continue;  // the other issuer's stage (or nothing left to do)
      // this warp's earlier waits on its barrier of the slot: every use
      // (even slot count: the slot's stages all have this warp's parity) or
      // every other use (odd count: the parity of the slot's stages alternates)
      const uint32_t ph = (P.n_slots & 1) ? (u - 1) >> 1 : u - 1;
      if (lane == 0) {
        // the three conditions probed together first (their latencies
        // overlap); a bounded wait on each only when one is not yet met
        const uint32_t b_acce = bar_acce + 8 * (slot * 2 + mw);
        const bool r0 = mbar_try_wait(bar_full + 8 * s, n & 1);
        const bool r1 = mbar_try_wait(bar_sf + 8 * s, n & 1);
        const bool r2 = u == 0 || mbar_try_wait(b_acce, ph & 1);
        bool ok = r0 && r1 && r2 && !*abort;
        if (!ok) {
          ok = wait_or_abort(bar_full + 8 * s, n & 1, P, abort);                    // codes landed
          if (ok) ok = wait_or_abort(bar_sf + 8 * s, n & 1, P, abort);              // scale factors in TMEM
          if (ok && u > 0) ok = wait_or_abort(b_acce, ph & 1, P, abort);            // slot read
        }
        if (ok) {
          tc::fence_after_sync();
          if (kRescore) tc::fence_proxy_async_smem();  // codes written by cp.async (generic proxy)
          const uint32_t sfa = tmem + kColSfa + (uint32_t)s * 8 * kSub;
          const uint32_t acc = tmem + kColAcc + (uint32_t)(slot * P.slot_cols);
          // tile m of the stage (rows m*128 ..) and query column j into the
          // slot's part (m * W + j) * Nh
#pragma unroll
          for (int m = 0; m < kSub; ++m)
            for (int j = 0; j < W; ++j)
              for (int ks = 0; ks < ksteps; ++ks) {
                const uint64_t ad =
                    tc::smem_desc(sbase + kOffA + s * kCodeStage + m * kTile * row_bytes + ks * 32, 16, sbo, sw);
                const uint64_t bd = tc::smem_desc(sbase + kOffB + j * 4096 + ks * 32, 16, sbo, sw);
                tc::mma_mxf4nvf4(acc + (m * W + j) * P.Nh, ad, bd, idesc, sfa + m * 8 + ks * 4,
                                 tmem + kColSfb + j * 8 + ks * 4, ks > 0 ? 1u : 0u);
              }
          // one commit: the stage's shared memory and scale factors are free
          // and the slot holds the scores once these MMAs complete
          tc::commit(bar_done + 8 * s);
        }
      }
      __syncwarp();
    }
    // drain: no MMA or copy of ours in flight at teardown
    if (lane == 0) {
      tc::commit(my_drain);
      if (!mbar_wait_bounded(my_drain, drain_n & 1, P.wait_ns)) set_status(P.status, CSA2_ERR_TIMEOUT);
    }
    __syncwarp();
  } else if (warp < kEpi0) {
    // ------------------------------------------------------------ scale factors
    // raw per-32 scales of the stage's rows -> the block-scale layout the
    // MMA reads (K step ks: per-16 scales (s_2ks, s_2ks, s_2ks+1, s_2ks+1);
    // lane m0 of every lane quarter holds rows m1*32 + m0 in column m1),
    // written by this warp into its own lane quarter
    const int q = warp & 3;
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    TileIter<kRescore> ti;
    ti.init(P, w_g0, w_t0, w_n);
    int s = 0;
    uint32_t n = 0;
    const int box_rows = kRescore ? kBlock : P.box_rows;
    const int bshift = __ffs(box_rows) - 1;  // box_rows is a power of two (256, 128, 64 or 8)
    const int slot_bytes = kRescore ? 128 : box_rows * spr;
    const bool one_box4 = !kRescore && box_rows >= kRows && spr == 4;
    for (; ti.valid(); ti.next(P), (++s == kStages ? (s = 0, ++n) : 0u)) {
      if (!warp_wait_or_abort(bar_full + 8 * s, n & 1, P, abort)) break;
      const uint8_t* raw = smem + kOffRaw + s * kRawStage;
      // tile m of the stage: rows m*128 + m1*32 + lane, columns m*8 ..
      uint32_t r[kSub][8];
      if (one_box4) {  // the stage's scales are one [rows][4] array: word rw is row rw's
        const uint32_t* raw32 = reinterpret_cast<const uint32_t*>(raw) + lane;
#pragma unroll
        for (int m = 0; m < kSub; ++m)
#pragma unroll
          for (int m1 = 0; m1 < 4; ++m1) {
            const uint32_t wv = raw32[m * kTile + m1 * 32];
            r[m][m1] = __byte_perm(wv, 0, 0x1100u);      // K step 0: scales 0, 1
            r[m][4 + m1] = __byte_perm(wv, 0, 0x3322u);  // K step 1: scales 2, 3
          }
      } else {
#pragma unroll
        for (int m = 0; m < kSub; ++m)
#pragma unroll
          for (int m1 = 0; m1 < 4; ++m1) {
            const int rw = m * kTile + m1 * 32 + lane;
            const uint8_t* src = raw + (rw >> bshift) * slot_bytes + (rw & (box_rows - 1)) * spr;
            const uint32_t wv = (spr == 4) ? *reinterpret_cast<const uint32_t*>(src)
                                           : (uint32_t)*reinterpret_cast<const uint16_t*>(src);
            r[m][m1] = __byte_perm(wv, 0, 0x1100u);      // K step 0: scales 0, 1
            r[m][4 + m1] = __byte_perm(wv, 0, 0x3322u);  // K step 1: scales 2, 3
          }
      }
      const uint32_t ta = tmem + lane_base + kColSfa + (uint32_t)s * 8 * kSub;
      if (ksteps == 2) {
        if (kSub == 2) {
          const uint32_t r16[16] = {r[0][0], r[0][1], r[0][2], r[0][3], r[0][4], r[0][5], r[0][6], r[0][7],
                                    r[kSub - 1][0], r[kSub - 1][1], r[kSub - 1][2], r[kSub - 1][3],
                                    r[kSub - 1][4], r[kSub - 1][5], r[kSub - 1][6], r[kSub - 1][7]};
          tc::st_32x32b_x16(ta, r16);
        } else {
          tc::st_32x32b_x8(ta, r[0]);
        }
      } else {
#pragma unroll
        for (int m = 0; m < kSub; ++m) {
          const uint32_t r4[4] = {r[m][0], r[m][1], r[m][2], r[m][3]};
          tc::st_32x32b_x4(ta + m * 8, r4);
        }
      }
      tc::st_wait();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar_sf + 8 * s);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int wg = (warp - kEpi0) / 4;   // warpgroup: the stages it with it % kEpiWG == wg
    const int quarter = warp & 3;        // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;
    const int ept = threadIdx.x - kEpi0 * 32 - wg * 128;  // 0..127 within the warpgroup
    float* w_g = reinterpret_cast<float*>(smem + kOffW) + wg * kMaxWc * 64;
    int64_t* pos_g = reinterpret_cast<int64_t*>(smem + kOffPos) + wg * kMaxWc;
    TileIter<kRescore> ti;
    ti.init(P, w_g0, w_t0, w_n);
    // stage count, ring stage, slot, first warpgroup of the stage.  A stage's
    // units (its MMA tiles x query columns) are split between its warpgroup
    // wgc (the first half) and the next one (the rest), so that they are
    // reduced in parallel.  Every warpgroup takes
    // part in every third stage, so before it waits for a stage's commit it
    // has seen the commit of a stage of the same MMA warp at most six stages
    // back: the barrier cannot be a phase behind the one waited for.
    int it = 0, s = 0, slot = 0, wgc = 0;
    uint32_t n = 0;
    auto adv = [&]() {
      ++it;
      if (++s == kStages) {
        s = 0;
        ++n;
      }
      if (++slot == P.n_slots) slot = 0;
      if (++wgc == kEpiWG) wgc = 0;
    };
    int cur_g = -1, W = 0, tok0 = 0, sel0 = 0, np_e = 0;
    bool dead = false;  // a wait of this warp (two-tile stages) or warpgroup gave up
    const int ng = P.Nh / 16;
    // The group's key counts gather in shared memory (per CTA) and go to the
    // global counts, one atomic per non-empty bin, when the CTA leaves the
    // group: every SM adding each score to one group's global bins directly
    // contended on the few bins that hold most scores
    constexpr int kEpiThreads = 128 * kEpiWG;
    const int et = threadIdx.x - kEpi0 * 32;  // 0 .. kEpiThreads-1
    auto flush_counts = [&]() {
      for (int i = et; i < W * kHistBins; i += kEpiThreads) {
        const uint32_t v = hist_s[i];
        if (v) {
          const int j = i / kHistBins;
          const int64_t grow = kRescore ? (int64_t)(sel0 + j) * P.qb.n_tok + tok0 : (int64_t)(tok0 + j);
          atomicAdd(P.hist + grow * kHistBins + (i % kHistBins), v);
          hist_s[i] = 0u;
        }
      }
    };
    // no early exit: the warps of the epilogue meet at named barriers
    for (; ti.valid(); ti.next(P), adv()) {
      if (ti.b != cur_g) {
        tc::named_sync(7, kEpiThreads);  // every epilogue warp is done with the old group
        if (P.hist && cur_g >= 0) {
          flush_counts();
          tc::named_sync(7, kEpiThreads);
        }
        cur_g = ti.b;
        int bseq;
        group_info<kRescore>(P, cur_g, &tok0, &W, &bseq, &sel0);
        for (int e = ept; e < W * 64; e += 128) {
          const int j = e / 64, h = e % 64;
          // half weights: the epilogue's ReLU is s + |s| = 2 max(s, 0)
          const float* wsrc = P.w[kRescore ? sel0 + j : 0] + (int64_t)(kRescore ? tok0 : tok0 + j) * P.H;
          w_g[e] = h < P.H ? 0.5f * __ldg(wsrc + h) : 0.0f;
        }
        if (ept < W) pos_g[ept] = __ldg(P.qb.tok_pos + (kRescore ? tok0 : tok0 + ept));
        if (kRescore) np_e = min(__ldg(P.pool_n + tok0), P.pool_cap);
        tc::named_sync(1 + wg, 128);
      }
      // units of this stage, the first half to warpgroup wgc, the rest to the
      // next (with one accumulator slot, as in rescoring four selectors at a
      // time, the slot is free once both halves are read: half the wait)
      const int nu = kSub * W, half = (nu + 1) / 2;
      int mj0 = 0, mj1 = 0;  // this warpgroup's units
      if (wgc == wg) {
        mj1 = half;
      } else if (wgc + 1 == wg || wgc + 1 == wg + kEpiWG) {
        mj0 = half;
        mj1 = nu;
      }
      if (mj0 >= mj1 || dead) continue;  // no unit of this stage (or nothing left to do)
      int32_t blk = -1;  // rescore: this thread's pool block, loaded while the stage's MMAs run
      if (kRescore) {
        const int i = ti.tile * kTile + row;
        blk = (i / kBlock) < np_e ? __ldg(P.pool + (int64_t)tok0 * P.pool_cap + i / kBlock) : -1;
      }
      // two-tile stages: every warp probes for itself (measured faster);
      // otherwise one prober per warpgroup, the other warps parked on the
      // named barrier
      const uint32_t b_done = bar_done + 8 * s;
      const bool got = kSub == 2 ? (*abort == 0 && mbar_wait_warp(b_done, n & 1, P.wait_ns))
                                 : mbar_wait_group(b_done, n & 1, P.wait_ns, ept == 0, *abort != 0, 1 + wg, 128);
      if (!got) {
        if ((kSub == 2 ? lane : ept) == 0 && !*abort) {
          set_status(P.status, CSA2_ERR_TIMEOUT);
          *abort = 1;
        }
        dead = true;
        continue;
      }
      tc::fence_after_sync();
      const int64_t t0 = (int64_t)ti.tile * kRows;
      const uint32_t taddr0 = tmem + ((uint32_t)(quarter * 32) << 16) + kColAcc + (uint32_t)(slot * P.slot_cols);
      for (int mj = mj0; mj < mj1; ++mj) {  // unit: tile m = mj / W of the stage, query column j = mj % W
        // two-tile stages only serve one query token per sequence (W = 1)
        const int m = kSub == 1 ? 0 : mj, j = kSub == 1 ? mj : 0;
        const float* wj = w_g + j * 64;
        const uint32_t taddr = taddr0 + mj * P.Nh;
        // the column's scores in two halves of 32 heads (register budget):
        // weighted sum in packed pairs (four float2 chains).  ReLU as
        // s + |s| (an add on the FMA pipe, which the epilogue leaves idle,
        // instead of a max on the busier ALU pipe) against half weights:
        // (w/2)(2s) is w*s exactly, so every product is w*max(s, 0)
        float2 a2[4] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f),
                        make_float2(0.0f, 0.0f)};
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          if (hf * 2 >= ng) break;
          uint32_t r[2][16];
#pragma unroll
          for (int g = 0; g < 2; ++g)
            if (hf * 2 + g < ng) tc::ld_32x32b_x16(taddr + (hf * 2 + g) * 16, r[g]);
          tc::ld_wait();
          if (hf == 1 || ng <= 2) {  // this unit's part of the slot is read once its last load landed:
            tc::fence_before_sync();  // for the warp issuing the slot's next use
            __syncwarp();
            if (lane == 0)
              tc::mbar_arrive_cnt(bar_acce + 8 * (slot * 2 + ((it + P.n_slots) & 1)),
                                  mj == nu - 1 ? (uint32_t)(1 + kSub * P.wc - nu) : 1u);
          }
#pragma unroll
          for (int g = 0; g < 2; ++g)
            if (hf * 2 + g < ng) {
#pragma unroll
              for (int k4 = 0; k4 < 4; ++k4) {
                const float4 w4 = *reinterpret_cast<const float4*>(wj + (hf * 2 + g) * 16 + k4 * 4);
                const float s0 = __uint_as_float(r[g][k4 * 4 + 0]), s1 = __uint_as_float(r[g][k4 * 4 + 1]);
                const float s2 = __uint_as_float(r[g][k4 * 4 + 2]), s3 = __uint_as_float(r[g][k4 * 4 + 3]);
                const float2 x0 = make_float2(s0 + fabsf(s0), s1 + fabsf(s1));
                const float2 x1 = make_float2(s2 + fabsf(s2), s3 + fabsf(s3));
                a2[2 * g] = __ffma2_rn(make_float2(w4.x, w4.y), x0, a2[2 * g]);
                a2[2 * g + 1] = __ffma2_rn(make_float2(w4.z, w4.w), x1, a2[2 * g + 1]);
              }
            }
        }
        const float acc = ((a2[0].x + a2[1].x) + (a2[0].y + a2[1].y)) + ((a2[2].x + a2[3].x) + (a2[2].y + a2[3].y));
        const int64_t p = pos_g[kRescore ? 0 : j];
        if (kRescore) {
          // pool entry i = tile*128 + row: position pool[i/8]*8 + i%8
          const int i = ti.tile * kTile + row;
          const int64_t pos = (int64_t)blk * kBlock + (i % kBlock);
          const int64_t orow = (int64_t)(sel0 + j) * P.qb.n_tok + tok0;  // selector * T + token
          const bool valid = blk >= 0 && pos <= p && i < P.pool_cap * kBlock;
          if (i < P.pool_cap * kBlock) P.out[orow * P.ld + i] = valid ? acc : -INFINITY;
          if (P.hist && valid) {
            const uint32_t key = score_key(acc);
            if (key) atomicAdd(hist_s + j * kHistBins + (key >> kHistShift), 1u);
          }
        } else {
          const int64_t t = t0 + m * kTile + row;
          float sc = (t <= p) ? acc : -INFINITY;
          sc = fmaxf(sc, __shfl_xor_sync(0xffffffffu, sc, 1));
          sc = fmaxf(sc, __shfl_xor_sync(0xffffffffu, sc, 2));
          sc = fmaxf(sc, __shfl_xor_sync(0xffffffffu, sc, 4));
          if ((lane & 7) == 0 && t <= p) {
            P.out[(int64_t)(tok0 + j) * P.ld + t / kBlock] = sc;
            const uint32_t key = score_key(sc);
            if (P.hist && key) atomicAdd(hist_s + j * kHistBins + (key >> kHistShift), 1u);
          }
        }
      }
    }
    tc::named_sync(7, kEpiThreads);  // the last group's counts are complete
    if (P.hist && cur_g >= 0) flush_counts();
  }
  grid_dep_launch();
  // after a failed wait some tile loads may still be in flight: give them
  // time to land before the CTA's shared memory is released (bounded)
  if (threadIdx.x == 0 && *abort) {
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 200000ull) __nanosleep(1000);
  }
  __syncthreads();
  if (warp == kMma0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace scan_tc

// ---------------------------------------------------------------- host side
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// codes: [n_rows][row_bytes] u8, box {row_bytes, box_rows}, swizzle = row_bytes
int make_codes_map(CUtensorMap* m, const uint8_t* codes, int64_t n_rows, int row_bytes, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return fail(CSA2_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)n_rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  cuuint32_t box[2] = {(cuuint32_t)row_bytes, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  CUtensorMapSwizzle sw = row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(CSA2_ERR_CUDA, "cuTensorMapEncodeTiled(codes) failed: %d", (int)r);
  return CSA2_OK;
}

// scales: the [n_rows][spr] byte array seen as rows of 16 bytes (n_rows * spr
// a multiple of 16), box of box_rows * spr / 16 such rows (the scales of
// box_rows cache rows)
int make_scales_map(CUtensorMap* m, const uint8_t* scales, int64_t n_rows, int spr, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return fail(CSA2_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  if ((n_rows * spr) % 16) return fail(CSA2_ERR_UNSUPPORTED, "indexer cache rows * d_I/32 must be a multiple of 16");
  cuuint64_t dims[2] = {16, (cuuint64_t)(n_rows * spr / 16)};
  cuuint64_t strides[1] = {16};
  cuuint32_t box[2] = {16, (cuuint32_t)(box_rows * spr / 16)};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(scales), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(CSA2_ERR_CUDA, "cuTensorMapEncodeTiled(scales) failed: %d", (int)r);
  return CSA2_OK;
}

static int num_sms() {
  static int n[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 148;
  if (!n[dev]) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    n[dev] = v > 0 ? v : 148;
  }
  return n[dev];
}

template <bool kRescore, int kSub>
static int launch_index_tc(const csa2_query_batch* qb, const uint8_t* qc, const uint8_t* qs, const float* const* w,
                           int n_sel, int H, const csa2_fp4_cache* kc, const int32_t* pool, const int32_t* pool_n,
                           int pool_cap, float* out, int64_t ld, uint32_t* hist, cudaStream_t st) {
  using namespace scan_tc;
  using Lay = Layout<kSub>;
  constexpr int kRows = kTile * kSub;
  if (kc->n_rows >= (int64_t(1) << 31)) return fail(CSA2_ERR_UNSUPPORTED, "cache too large for TMA");
  if (n_sel < 1 || n_sel > kMaxSel) return fail(CSA2_ERR_UNSUPPORTED, "1..%d selector layers per launch", kMaxSel);
  // scan boxes: a stage's rows, or the largest power of two (>= 64) that
  // does not cross a page
  int box_rows = kRows;
  if (!kRescore && kc->page_table)
    while (box_rows > 64 && kc->page_size % box_rows != 0) box_rows /= 2;
  if (kRescore) box_rows = kBlock;
  CUtensorMap tmc, tms;
  if (int rc = make_codes_map(&tmc, kc->codes, kc->n_rows, kc->dim / 2, box_rows)) return rc;
  if (int rc = make_scales_map(&tms, kc->scales, kc->n_rows, kc->dim / 32, box_rows)) return rc;
  Params p{};
  p.qb = *qb;
  p.q_codes = qc;
  p.q_scales = qs;
  for (int i = 0; i < n_sel; ++i) p.w[i] = w[i];
  p.n_sel = n_sel;
  // query columns per group and groups per sequence (scan) or token (rescore)
  const int cols = kRescore ? n_sel : std::max(1, qb->max_q_per_seq);
  p.H = H;
  p.Nh = (H + 15) / 16 * 16;
  p.DI = kc->dim;
  // accumulator slots for wc query columns per group: as many as fit, a
  // divisor of the stage count (so that a stage's commit barrier cannot run
  // two phases ahead of a slot's reader)
  auto slots_for = [&](int wc) {
    int ns = std::min<int>(6, (int)(Lay::kAccCols / (uint32_t)(kSub * wc * p.Nh)));
    while (ns > 1 && Lay::kStages % ns) --ns;
    return ns;
  };
  // the widest group that still leaves two accumulator slots (MMAs of one
  // stage overlap the epilogue of the previous one); one slot only when even
  // a single column leaves no second
  int wc = std::min(cols, kMaxWc);
  // rescoring with plenty of stages per CTA: the widest group (every pool
  // block gathered once for up to four selectors) even with one slot; the
  // gathers, not the epilogue, bound it there
  const bool wide = kRescore && (int64_t)qb->n_tok * ((int64_t)pool_cap * kBlock / kRows) >= 4ll * num_sms();
  if (!wide)
    while (wc > 1 && slots_for(wc) < 2) --wc;
  p.wc = wc;
  p.cpg = (cols + wc - 1) / wc;
  p.slot_cols = kSub * wc * p.Nh;
  const int ns = slots_for(wc);
  if (ns < 1) return fail(CSA2_ERR_UNSUPPORTED, "index accumulators do not fit in TMEM");
  p.n_slots = ns;
  p.box_rows = box_rows;
  p.rows = kRows;
  p.codes = kc->codes;
  p.scales = kc->scales;
  p.n_rows = kc->n_rows;
  p.page_size = kc->page_size;
  p.max_pages = kc->max_pages;
  p.page_table = kc->page_table;
  p.seq_base = kc->seq_base;
  p.out = out;
  p.ld = ld;
  p.pool = pool;
  p.pool_n = pool_n;
  p.pool_cap = pool_cap;
  p.hist = hist;
  p.status = status_ptr();
  p.wait_ns = 1000000000ull;  // 1 s
  static bool attr_done[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    if (int rc = cuda_check(cudaFuncSetAttribute(k_index_tc<kRescore, kSub>,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::kSmemBytes),
                            "index smem attribute"))
      return rc;
    int fit = 0;  // one CTA of kThreads threads at this register count must fit on an SM
    if (int rc = cuda_check(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&fit, k_index_tc<kRescore, kSub>, kThreads,
                                                                          Lay::kSmemBytes),
                            "index occupancy"))
      return rc;
    if (fit < 1) return fail(CSA2_ERR_UNSUPPORTED, "index kernel does not fit on an SM");
    attr_done[dev] = true;
  }
  Launch L_(kRescore ? "rescore_tc" : "scan_tc", st);
  return cuda_check(launch_overlapped(kRescore ? kOverlapRescore : kOverlapScan, k_index_tc<kRescore, kSub>,
                                      dim3(num_sms()), dim3(kThreads), Lay::kSmemBytes, st, tmc, tms, p),
                    "k_index_tc");
}

int launch_scan_tc(const csa2_query_batch* qb, const uint8_t* qc, const uint8_t* qs, const float* w, int H,
                   const csa2_fp4_cache* kc, float* bs, int64_t ld, uint32_t* hist, cudaStream_t st) {
  // one query token per sequence: stages of two MMA tiles (256 positions)
  if (qb->max_q_per_seq <= 1)
    return launch_index_tc<false, 2>(qb, qc, qs, &w, 1, H, kc, nullptr, nullptr, 0, bs, ld, hist, st);
  return launch_index_tc<false, 1>(qb, qc, qs, &w, 1, H, kc, nullptr, nullptr, 0, bs, ld, hist, st);
}

// n_sel selector layers at once: queries [n_sel][T][H][...], weights w[sel],
// scores [n_sel][T][8P]; a token's pool is gathered once for up to four of them
int launch_rescore_tc(const csa2_query_batch* qb, const uint8_t* qc, const uint8_t* qs, const float* const* w,
                      int n_sel, int H, const csa2_fp4_cache* kc, const int32_t* pool, const int32_t* pool_n, int P,
                      float* scores, uint32_t* hist, cudaStream_t st) {
  return launch_index_tc<true, 1>(qb, qc, qs, w, n_sel, H, kc, pool, pool_n, P, scores, (int64_t)P * kBlock, hist,
                                  st);
}

}  // namespace csa2
