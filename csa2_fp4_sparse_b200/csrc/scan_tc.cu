// scan_tc.cu -- the indexer scoring on the 5th-generation tensor cores
// (sm_100a): the Full layer's scan of the whole visible context (block scores)
// and the pool rescoring of the Full layer's own top-K and of every Reindex
// layer (position scores), one templated kernel.
//
// For every query token i of sequence b and visible position t <= p_i:
//   s_t = sum_h w[i][h] * max(0, q~_{i,h} . k~_t),   B_j = max_{t in block j} s_t
// (hierarchical indexer of the DeepSeek-V4.1-Flash pages, dbyun.net article
// 10794, section "KV Cache 成为这一代架构改造的核心": the first Full layer scans
// the whole visible context and keeps blocks of 8 positions).
//
// Design (one persistent CTA per SM, warp-specialised):
//   warp 0      TMA producer (rescoring: warps 0, 21, 22 on alternate groups
//               of tiles, as a TMA instruction costs its warp ~110 cycles and
//               a rescoring tile gathers 32 boxes): tiles of 128 positions of
//               the FP4 indexer K cache
//               (codes with the 64B/32B swizzle the MMA expects, plus the raw
//               E4M3 scales) into a shared-memory ring of 17 stages (15 when
//               rescoring);
//   warps 19,20 scale-factor warps (alternate passes of two tiles):
//               rearrange each landed tile's scales into the tensor-core
//               scale-factor layout (each per-32 E4M3 scale written twice, as
//               the block-scaled MMA takes one UE4M3 scale per 16 elements)
//               and copy it to TMEM (tcgen05.cp); a commit hands the stage to
//               the MMA warp;
//   warps 1, 18 MMA issuers (alternate tiles, two epilogue warpgroups each):
//               issue tcgen05.mma kind::mxf4nvf4 (M = 128 positions, N =
//               heads, K = 64 per instruction) per query token into a ring of
//               TMEM accumulators (2 units per issuer); one commit per job hands
//               the accumulator to the epilogue, one per tile returns the
//               stage to the producer.  A tcgen05 instruction costs its
//               issuing thread 100-200 cycles, so the copies are issued by the
//               scale-factor warps, not here;
//   warps 2..17 epilogue, four warpgroups: warpgroup e takes the accumulator
//               jobs of MMA warp (e & 1) whose job count has parity e >> 1:
//               TMEM -> registers (one position per thread), ReLU, weighted
//               head sum, block max over 8 lanes, block-score store.
// The key cache is streamed from HBM exactly once per sequence for all of its
// query tokens.  In rescoring mode the producer instead gathers the 16 pool
// blocks of a tile (8 rows each, one swizzle atom per block) for one query
// token, and the epilogue writes one score per pool position.  All waits are
// bounded; on timeout the kernel records CSA2_ERR_TIMEOUT, drains its own
// copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "internal.h"
#include "tc_common.cuh"

namespace csa2 {
namespace scan_tc {

constexpr int kTile = 128;      // positions per tile = MMA M
constexpr int kChunk = 64;      // rows per TMA box
constexpr int kAccUnits = 4;    // TMEM accumulator ring, 64 columns each (2 per MMA issuer)
constexpr int kMaxW = 8;        // query tokens of one sequence per tile
constexpr int kEpiWG = 4;       // epilogue warpgroups (warps 2..17)
constexpr int kThreads = 736;   // 23 warps: 3 producers, 2 MMA issuers, 4 epilogue warpgroups, 2 scale-factor warps
constexpr int kProducers = 3;   // TMA producer warps 0, 21, 22 when rescoring (a TMA instruction costs its
                                // warp ~110 cycles and a rescoring tile gathers 32 boxes); the scan uses warp 0
constexpr int kMmaWarpB = 18;   // second MMA issuer (the first is warp 1); they take alternate tiles
constexpr int kSfWarp = 19;     // scale-factor warps 19 and 20 take alternate passes of two tiles
constexpr int kUnitsPer = kAccUnits / 2;  // accumulator units of each MMA issuer
constexpr uint32_t kColAcc = 0;
constexpr uint32_t kTmemCols = 512;

// Shared-memory and TMEM map.  A tile's stage stays occupied from its load
// to the completion of its MMAs (~8-9 K cycles: load latency under full HBM
// load, scale-factor pass, MMA), so the ring is as deep as shared memory
// allows: 17 stages for the scan, 15 for the rescoring (whose raw-scale slot
// holds 16 gathered boxes).
template <bool kRescore>
struct Ly {
  static constexpr int kStages = kRescore ? 15 : 17;
  // raw scales: every TMA box gets its own 128-byte-aligned slot (TMA writes
  // shared memory at 128-byte-aligned addresses): scan 2 boxes at 256-byte
  // slots, rescoring 16 boxes at 128-byte slots
  static constexpr uint32_t kRawStage = kRescore ? 2048 : 512;
  static constexpr uint32_t kColSfa = kAccUnits * 64;            // key scale factors, 8 columns per stage
  static constexpr uint32_t kColSfb = kColSfa + kStages * 8;     // query scale factors, 8 columns per token
  static_assert(kColSfb + kMaxW * 8 <= kTmemCols, "TMEM budget");
  static constexpr uint32_t kOffA = 0;                                   // [kStages][8192]
  static constexpr uint32_t kOffRaw = kOffA + kStages * 8192;            // [kStages][kRawStage]
  static constexpr uint32_t kOffSfa = kOffRaw + kStages * kRawStage;     // [kStages][2][512]
  static constexpr uint32_t kOffB = (kOffSfa + kStages * 1024 + 1023) / 1024 * 1024;  // [kMaxW][64 rows][64 B]
  static constexpr uint32_t kOffSfb = kOffB + kMaxW * 4096;              // [kMaxW][2][512]
  static constexpr uint32_t kOffW = kOffSfb + kMaxW * 1024;              // [kEpiWG][kMaxW][64] f32
  static constexpr uint32_t kOffPos = kOffW + kEpiWG * kMaxW * 64 * 4;   // [1 + kEpiWG][kMaxW] i64 query positions
  static constexpr uint32_t kOffBar = kOffPos + (1 + kEpiWG) * kMaxW * 8;  // mbarriers
  static constexpr uint32_t kNumBars = 3 * kStages + 2 * kAccUnits + 5;
  static constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;           // tmem base, abort flag
  static constexpr uint32_t kSmemBytes = kOffMisc + 16 + 1024;           // + alignment slack
  static_assert(kOffB % 1024 == 0, "B tiles must be 1024-aligned");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

struct Params {
  csa2_query_batch qb;
  const uint8_t* q_codes;   // [n_sel][T][H][d_I/2]
  const uint8_t* q_scales;  // [n_sel][T][H][d_I/32]
  const float* w[kMaxSel];  // per selector [T][H]
  int n_sel;                // rescore: selector layers (scan: 1)
  int qchunks;              // scan: groups per sequence, each of up to kMaxW of its query tokens
  int H, N, DI;
  int64_t n_rows;
  int page_size, max_pages;
  const int32_t* page_table;
  const int64_t* seq_base;
  float* out;        // scan: block scores [T][ld]; rescore: pool-position scores [T][ld]
  int64_t ld;
  const int32_t* pool;   // rescore: [T][pool_cap] block ids
  const int32_t* pool_n; // rescore: [T]
  int pool_cap;
  int* status;
  uint64_t wait_ns;
};

// Work groups: a chunk of up to kMaxW query tokens of one sequence (scan:
// the chunk's tokens share every tile; sequence b's chunk c is group
// b * qchunks + c and holds its tokens c*kMaxW ..; a decode step with at most
// kMaxW tokens per sequence has one chunk per sequence, and longer token runs
// (verify, chunked prefill) read the keys once per chunk) or a query token
// (rescore: its own pool).  Tiles are 128 positions.
template <bool kRescore>
__device__ __forceinline__ int n_groups(const Params& P) {
  return kRescore ? P.n_sel * P.qb.n_tok : P.qb.n_seq * P.qchunks;
}

// first query token, number of query tokens (0: empty chunk), sequence of group g
template <bool kRescore>
__device__ __forceinline__ void group_info(const Params& P, int g, int* tok0, int* W, int* b) {
  if (kRescore) {
    *tok0 = g % P.qb.n_tok;  // group = (selector, token)
    *W = 1;
    *b = __ldg(P.qb.tok_seq + *tok0);
  } else {
    *b = g / P.qchunks;
    const int t_end = __ldg(P.qb.tok_start + *b + 1);
    *tok0 = __ldg(P.qb.tok_start + *b) + (g % P.qchunks) * kMaxW;
    *W = max(0, min(kMaxW, t_end - *tok0));
  }
}

// tiles of group g: those holding a position visible to one of its tokens
template <bool kRescore>
__device__ __forceinline__ int group_tiles(const Params& P, int g) {
  if (kRescore) return (min(__ldg(P.pool_n + g % P.qb.n_tok), P.pool_cap) + 15) / 16;
  int tok0, W, b;
  group_info<false>(P, g, &tok0, &W, &b);
  if (W <= 0) return 0;
  const int64_t vis = min((int64_t)__ldg(P.qb.tok_pos + tok0 + W - 1) + 1, (int64_t)__ldg(P.qb.seq_len + b));
  return (int)((max(vis, (int64_t)0) + kTile - 1) / kTile);
}

// this CTA's contiguous range of (group, tile) work in group-major order
template <bool kRescore>
__device__ __forceinline__ void work_range(const Params& P, int64_t* begin, int64_t* end) {
  int64_t total = 0;
  for (int g = 0; g < n_groups<kRescore>(P); ++g) total += group_tiles<kRescore>(P, g);
  *begin = total * blockIdx.x / gridDim.x;
  *end = total * (blockIdx.x + 1) / gridDim.x;
}

// iterator over the tiles of [begin, end)
template <bool kRescore>
struct TileIter {
  int b, tile, ntile;  // b: group
  int64_t left;
  __device__ void init(const Params& P, int64_t begin, int64_t end) {
    b = 0;
    int64_t acc = 0;
    const int ng = n_groups<kRescore>(P);
    ntile = group_tiles<kRescore>(P, 0);
    while (b < ng - 1 && acc + ntile <= begin) {
      acc += ntile;
      ++b;
      ntile = group_tiles<kRescore>(P, b);
    }
    tile = (int)(begin - acc);
    left = end - begin;
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

template <bool kRescore>
__global__ void __launch_bounds__(kThreads, 1)
    k_index_tc(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_scales,
               const __grid_constant__ Params P) {
  using L = Ly<kRescore>;
  constexpr int kStages = L::kStages;
  constexpr uint32_t kRawStage = L::kRawStage;
  constexpr uint32_t kOffA = L::kOffA, kOffRaw = L::kOffRaw, kOffSfa = L::kOffSfa, kOffB = L::kOffB,
                     kOffSfb = L::kOffSfb, kOffW = L::kOffW, kOffPos = L::kOffPos, kOffBar = L::kOffBar,
                     kOffMisc = L::kOffMisc, kColSfa = L::kColSfa, kColSfb = L::kColSfb;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar_full = sbase + kOffBar;
  const uint32_t bar_empty = bar_full + kStages * 8;
  const uint32_t bar_accf = bar_empty + kStages * 8;
  const uint32_t bar_acce = bar_accf + kAccUnits * 8;
  const uint32_t bar_drain = bar_acce + kAccUnits * 8;
  const uint32_t bar_sfr = bar_drain + 8;
  const uint32_t bar_drain2 = bar_sfr + 8 * kStages;
  const uint32_t bar_drain_b = bar_drain2 + 8;
  const uint32_t bar_sfb = bar_drain_b + 8;
  const uint32_t bar_drain_c = bar_sfb + 8;
  volatile uint32_t* tmem_holder = reinterpret_cast<volatile uint32_t*>(smem + kOffMisc);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
  float* w_s = reinterpret_cast<float*>(smem + kOffW);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row_bytes = P.DI / 2, spr = P.DI / 32, ksteps = P.DI / 64;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(bar_full + 8 * i, 1);
      mbar_init(bar_empty + 8 * i, 1);
    }
    for (int i = 0; i < kAccUnits; ++i) {
      mbar_init(bar_accf + 8 * i, 1);
      mbar_init(bar_acce + 8 * i, 4);
    }
    mbar_init(bar_drain, 1);
    for (int i = 0; i < kStages; ++i) mbar_init(bar_sfr + 8 * i, 1);
    mbar_init(bar_drain2, 1);
    mbar_init(bar_drain_b, 1);
    mbar_init(bar_sfb, 1);
    mbar_init(bar_drain_c, 1);
    *abort = 0;
    tc::fence_barrier_init();
    tc::tma_prefetch_desc(&tm_codes);
    tc::tma_prefetch_desc(&tm_scales);
  }
  if (warp == 1) {
    tc::tmem_alloc(sbase + kOffMisc, kTmemCols);
    tc::tmem_relinquish();
    tc::fence_before_sync();
  }
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_holder;

  int64_t wb, we;
  work_range<kRescore>(P, &wb, &we);

  if (warp == 0 || warp >= kSfWarp + 2) {
    // ------------------------------------------------------------ producers
    // G tiles per iteration, `boxes` lanes per tile (scan: 2 boxes of 64 rows,
    // rescore: 16 blocks of 8 rows): the lanes of different tiles wait for
    // their stages and issue their copies concurrently; the producer warps
    // take alternate groups of G tiles.
    const int pi = warp == 0 ? 0 : warp - (kSfWarp + 1);
    constexpr int nprod = kRescore ? kProducers : 1;  // the scan's 4 boxes a tile need one warp
    const uint32_t tx = (uint32_t)kTile * row_bytes + (uint32_t)kTile * spr;
    const int32_t oob_row = (int32_t)P.n_rows;
    const int32_t oob_x = (int32_t)(((P.n_rows * spr) + 15) / 16 * 16);
    constexpr int boxes = kRescore ? 16 : 2;
    constexpr int rows_per_box = kTile / boxes;
    // tiles per group: a group is issued once all its stages are free, so a
    // small group keeps most of the ring in flight
    constexpr int G = (32 / boxes) < 4 ? (32 / boxes) : 4;
    const int lt = lane / boxes, bx = lane % boxes;
    const bool has_slot = lane < G * boxes;
    TileIter<kRescore> ti;
    ti.init(P, wb, we);
    for (int k = 0; k < pi * G + lt; ++k) ti.next(P);
    int64_t it = pi * G + lt;  // this lane's tile
    const int64_t total = pi < nprod ? we - wb : 0;
    int cur_g = -1, tok0 = 0, b = 0;
    int64_t base = 0, len = 0;
    for (int64_t g0 = pi * G; g0 < total; g0 += nprod * G) {
      const bool act = has_slot && ti.valid();
      const int s = (int)(it % kStages);
      const uint32_t n = (uint32_t)(it / kStages);
      // the first lane of each tile waits for its stage and arms it (one warp
      // instruction probes the stages of all the group's tiles at once)
      if (act && bx == 0) {
        if (wait_or_abort(bar_empty + 8 * s, (n & 1) ^ 1, P, abort)) tc::mbar_arrive_expect_tx(bar_full + 8 * s, tx);
      }
      __syncwarp();  // every stage of this group armed before any copy lands
      if (act && !*abort) {
        if (ti.b != cur_g) {
          cur_g = ti.b;
          int W;
          group_info<kRescore>(P, cur_g, &tok0, &W, &b);
          len = __ldg(P.qb.seq_len + b);
          base = P.page_table ? 0 : __ldg(P.seq_base + b);
        }
        int64_t pos0 = -1;
        if (kRescore) {
          const int e = ti.tile * 16 + bx;
          const int np = min(__ldg(P.pool_n + tok0), P.pool_cap);
          const int32_t blk = e < np ? __ldg(P.pool + (int64_t)tok0 * P.pool_cap + e) : -1;
          if (blk >= 0) pos0 = (int64_t)blk * kBlock;
        } else {
          pos0 = (int64_t)ti.tile * kTile + bx * kChunk;
          if (pos0 >= len) pos0 = -1;
        }
        int64_t row0 = -1;
        if (pos0 >= 0) {
          if (P.page_table) {
            const int32_t pg = __ldg(P.page_table + (int64_t)b * P.max_pages + pos0 / P.page_size);
            row0 = (int64_t)pg * P.page_size + pos0 % P.page_size;
          } else {
            row0 = base + pos0;
          }
        }
        int32_t ry = oob_row, sx = oob_x;
        if (row0 >= 0 && row0 < P.n_rows && ((row0 * spr) & 15) == 0) {
          ry = (int32_t)row0;
          sx = (int32_t)(row0 * spr);
        } else if (row0 >= 0) {
          set_status(P.status, CSA2_ERR_RANGE);  // misplaced row: read as zeros
        }
        tc::tma_load_2d(sbase + kOffA + s * 8192 + bx * rows_per_box * row_bytes, &tm_codes, bar_full + 8 * s, 0,
                        ry);
        tc::tma_load_1d(sbase + kOffRaw + s * kRawStage + bx * (kRawStage / boxes), &tm_scales, bar_full + 8 * s,
                        sx);
      }
      __syncwarp();
      if (*abort) break;
      for (int k = 0; k < nprod * G; ++k) ti.next(P);
      it += nprod * G;
    }
    // copies in flight: the scale-factor warps wait for every tile's landing
    // before the CTA ends (after a failed wait, see the end of the kernel)
  } else if (warp == 1 || warp == kMmaWarpB) {
    // ------------------------------------------------------------ MMA issuers
    // Both issuers walk every tile (so both see every change of group) and
    // issue the MMAs of the tiles of their parity; a single issuing thread is
    // limited by the latency of its barrier tests and MMA issues, two overlap.
    const int mw = warp == 1 ? 0 : 1;
    const uint32_t my_drain = mw == 0 ? bar_drain : bar_drain_b;
    const uint32_t idesc = tc::idesc_mxf4nvf4(128, P.N);
    const tc::SmemLayout sw = (P.DI == 128) ? tc::kSwizzle64B : tc::kSwizzle32B;
    const uint32_t sbo = 8u * row_bytes;  // 8 rows per swizzle atom
    TileIter<kRescore> ti;
    ti.init(P, wb, we);
    int64_t it = 0;
    int cnt = 0;   // jobs issued by this warp
    uint32_t drain_n = 0, sfb_n = 0;
    int cur_b = -1, W = 0, tok0 = 0;
    // No early exit from this loop: both issuers must meet at the same named
    // barriers, so after a failed wait a warp keeps walking the tiles without
    // issuing anything (every later wait returns at once once *abort is set).
    for (; ti.valid(); ti.next(P), ++it) {
      if (ti.b != cur_b) {
        if (cur_b >= 0) {  // every MMA reading the old queries must finish first
          if (lane == 0) tc::commit(my_drain);
          __syncwarp();
          warp_wait_or_abort(my_drain, drain_n & 1, P, abort);
          ++drain_n;
        }
        tc::named_sync(5, 64);  // both issuers drained
        cur_b = ti.b;
        int bseq;
        group_info<kRescore>(P, cur_b, &tok0, &W, &bseq);
        if (W > kMaxW) {
          if (lane == 0 && mw == 0) set_status(P.status, CSA2_ERR_RANGE);
          W = kMaxW;
        }
        if (mw == 0 && !*abort) {
          // query rows of this group: selector * T + token (scan: the sequence's tokens)
          const int64_t qrow0 = kRescore ? (int64_t)(cur_b / P.qb.n_tok) * P.qb.n_tok + tok0 : tok0;
          int64_t* pos_s = reinterpret_cast<int64_t*>(smem + kOffPos);
          if (lane < W) pos_s[lane] = __ldg(P.qb.tok_pos + tok0 + lane);
          // B operand: query codes, swizzled like the TMA-written A tiles
          const int chunks_per_row = row_bytes / 16;
          for (int e = lane; e < W * 64 * chunks_per_row; e += 32) {
            const int j = e / (64 * chunks_per_row);
            const int n = (e / chunks_per_row) % 64;
            const int ch = e % chunks_per_row;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (n < P.H)
              v = __ldg(reinterpret_cast<const uint4*>(P.q_codes + ((int64_t)(qrow0 + j) * P.H + n) * row_bytes) + ch);
            const int sch = (P.DI == 128) ? (ch ^ ((n >> 1) & 3)) : (ch ^ ((n >> 2) & 1));
            *reinterpret_cast<uint4*>(smem + kOffB + j * 4096 + n * row_bytes + sch * 16) = v;
          }
          // B scale factors: [m0 (32)][m1 (4)][k (4)] per 64-element K step
          for (int e = lane; e < W * ksteps * 32; e += 32) {
            const int j = e / (ksteps * 32), ks = (e / 32) % ksteps, m0 = e % 32;
            uint32_t v[4];
#pragma unroll
            for (int m1 = 0; m1 < 4; ++m1) {
              const int n = m1 * 32 + m0;
              uint32_t a = 0, b2 = 0;
              if (n < P.H) {
                const uint8_t* sp = P.q_scales + ((int64_t)(qrow0 + j) * P.H + n) * spr + 2 * ks;
                a = __ldg(sp);
                b2 = __ldg(sp + 1);
              }
              v[m1] = a | (a << 8) | (b2 << 16) | (b2 << 24);
            }
            *reinterpret_cast<uint4*>(smem + kOffSfb + (j * 2 + ks) * 512 + m0 * 16) =
                make_uint4(v[0], v[1], v[2], v[3]);
          }
          tc::fence_proxy_async_smem();
          __syncwarp();
          bool ok = true;
          if (lane == 0) {
            tc::fence_after_sync();
            for (int j = 0; j < W; ++j)
              for (int ks = 0; ks < ksteps; ++ks)
                tc::cp_32x128b_warpx4(tmem + kColSfb + j * 8 + ks * 4,
                                      tc::smem_desc(sbase + kOffSfb + (j * 2 + ks) * 512, 16, 128, tc::kSwizzleNone));
            tc::commit(bar_sfb);
            ok = wait_or_abort(bar_sfb, sfb_n & 1, P, abort);  // the copies landed before anyone issues
          }
          ++sfb_n;
          (void)ok;
        }
        tc::named_sync(6, 64);  // new queries and positions in place
        tc::fence_after_sync();
      }
      if ((int)(it & 1) != mw || *abort) continue;  // the other issuer's tile (or nothing left to do)
      const int s = (int)(it % kStages);
      const uint32_t n = (uint32_t)(it / kStages);
      bool okw = true;
      if (lane == 0) {
        okw = wait_or_abort(bar_sfr + 8 * s, n & 1, P, abort);  // tile landed, scale factors in TMEM
        tc::fence_after_sync();
        const uint32_t sfa = tmem + kColSfa + (uint32_t)s * 8;
        const int64_t* pos_s = reinterpret_cast<const int64_t*>(smem + kOffPos);
        const int64_t t0 = (int64_t)ti.tile * kTile;
        for (int j = 0; j < W && okw; ++j) {
          if (!kRescore && t0 > pos_s[j]) continue;
          const int u = mw * kUnitsPer + cnt % kUnitsPer;
          const uint32_t m = (uint32_t)(cnt / kUnitsPer);
          if (!wait_or_abort(bar_acce + 8 * u, (m & 1) ^ 1, P, abort)) {
            okw = false;
            break;
          }
          tc::fence_after_sync();
          for (int ks = 0; ks < ksteps; ++ks) {
            const uint64_t ad = tc::smem_desc(sbase + kOffA + s * 8192 + ks * 32, 16, sbo, sw);
            const uint64_t bd = tc::smem_desc(sbase + kOffB + j * 4096 + ks * 32, 16, sbo, sw);
            tc::mma_mxf4nvf4(tmem + kColAcc + u * 64, ad, bd, idesc, sfa + ks * 4, tmem + kColSfb + j * 8 + ks * 4,
                             ks > 0 ? 1u : 0u);
          }
          tc::commit(bar_accf + 8 * u);
          ++cnt;
        }
        // the stage goes back to the producer as soon as the MMAs that read
        // it complete
        if (okw) tc::commit(bar_empty + 8 * s);
      }
      cnt = __shfl_sync(0xffffffffu, cnt, 0);
      (void)okw;
    }
    // drain: no MMA or copy of ours in flight at teardown
    if (lane == 0) {
      tc::commit(my_drain);
      if (!mbar_wait_bounded(my_drain, drain_n & 1, P.wait_ns)) set_status(P.status, CSA2_ERR_TIMEOUT);
    }
    __syncwarp();
  } else if (warp == kSfWarp || warp == kSfWarp + 1) {
    // ------------------------------------------------------------ scale factors
    // raw [row][spr] -> [m0 (32)][m1 (4)][k (4)] per 64-element K step, each
    // per-32 scale written twice (the MMA takes one scale per 16 elements);
    // two tiles per pass, so the fixed costs of a pass (proxy fence, copy
    // issue) are shared
    TileIter<kRescore> ti;
    ti.init(P, wb, we);
    int64_t it = 0;
    constexpr int kBoxRows = kRescore ? kBlock : kChunk;
    constexpr uint32_t kSlot = kRescore ? kRawStage / 16 : kRawStage / 2;
    const int sfw = warp - kSfWarp;
    int64_t pass = 0;
    while (ti.valid()) {
      const int nt = ti.left >= 2 ? 2 : 1;
      if ((int)(pass++ & 1) != sfw) {  // the other scale-factor warp's pass
        for (int k = 0; k < nt; ++k) ti.next(P);
        it += nt;
        continue;
      }
      uint32_t wv[2][4];
      bool ok = true;
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        if (k >= nt) break;
        const int s = (int)((it + k) % kStages);
        const uint32_t n = (uint32_t)((it + k) / kStages);
        if (!warp_wait_or_abort(bar_full + 8 * s, n & 1, P, abort)) {
          ok = false;
          break;
        }
        const uint8_t* raw = smem + kOffRaw + s * kRawStage;
#pragma unroll
        for (int m1 = 0; m1 < 4; ++m1) {
          const int r = m1 * 32 + lane;
          const uint8_t* src = raw + (r / kBoxRows) * kSlot + (r % kBoxRows) * spr;
          wv[k][m1] =
              (spr == 4) ? *reinterpret_cast<const uint32_t*>(src) : (uint32_t)*reinterpret_cast<const uint16_t*>(src);
        }
      }
      if (!ok) break;
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        if (k >= nt) break;
        const int s = (int)((it + k) % kStages);
        for (int ks = 0; ks < ksteps; ++ks) {
          const uint32_t sel = ks == 0 ? 0x1100u : 0x3322u;
          *reinterpret_cast<uint4*>(smem + kOffSfa + (s * 2 + ks) * 512 + lane * 16) =
              make_uint4(__byte_perm(wv[k][0], 0, sel), __byte_perm(wv[k][1], 0, sel),
                         __byte_perm(wv[k][2], 0, sel), __byte_perm(wv[k][3], 0, sel));
        }
      }
      tc::fence_proxy_async_smem();
      __syncwarp();
      // copy to TMEM from this warp (tcgen05 instructions cost their issuing
      // thread 100-200 cycles each, so they are spread over the warps that
      // have time); the commit hands the stage over once the copy landed
      if (lane == 0) {
        tc::fence_after_sync();
        for (int k = 0; k < nt; ++k) {
          const int s = (int)((it + k) % kStages);
          for (int ks = 0; ks < ksteps; ++ks)
            tc::cp_32x128b_warpx4(tmem + kColSfa + s * 8 + ks * 4,
                                  tc::smem_desc(sbase + kOffSfa + (s * 2 + ks) * 512, 16, 128, tc::kSwizzleNone));
          tc::commit(bar_sfr + 8 * s);
        }
      }
      __syncwarp();
      for (int k = 0; k < nt; ++k) ti.next(P);
      it += nt;
    }
    // drain: our copies must have landed before teardown
    if (lane == 0) {
      const uint32_t dr = sfw == 0 ? bar_drain2 : bar_drain_c;
      tc::commit(dr);
      if (!mbar_wait_bounded(dr, 0, P.wait_ns)) set_status(P.status, CSA2_ERR_TIMEOUT);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int wg = (warp - 2) / 4;        // warpgroup: warps 2+4wg .. 5+4wg
    const int mw = wg & 1, sub = wg >> 1; // its MMA issuer and job parity
    const int quarter = warp & 3;         // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;
    const int ept = threadIdx.x - 64 - wg * 128;  // 0..127 within the warpgroup
    float* w_g = w_s + wg * kMaxW * 64;
    int64_t* pos_g = reinterpret_cast<int64_t*>(smem + kOffPos) + (1 + wg) * kMaxW;
    TileIter<kRescore> ti;
    ti.init(P, wb, we);
    int64_t it = 0;
    int cnt = 0;  // jobs of this warpgroup's issuer (all parities)
    int cur_b = -1, W = 0, tok0 = 0;
    bool dead = false;  // warpgroup-uniform: a wait of this warpgroup gave up
    // no early exit: the four warps of the warpgroup meet at named barriers
    for (; ti.valid(); ti.next(P), ++it) {
      if (ti.b != cur_b) {
        tc::named_sync(1 + wg, 128);
        cur_b = ti.b;
        int bseq;
        group_info<kRescore>(P, cur_b, &tok0, &W, &bseq);
        W = min(W, kMaxW);
        for (int e = ept; e < W * 64; e += 128) {
          const int j = e / 64, h = e % 64;
          w_g[e] = h < P.H ? __ldg(P.w[kRescore ? cur_b / P.qb.n_tok : 0] + (int64_t)(tok0 + j) * P.H + h) : 0.0f;
        }
        if (ept < W) pos_g[ept] = __ldg(P.qb.tok_pos + tok0 + ept);
        tc::named_sync(1 + wg, 128);
      }
      if ((int)(it & 1) != mw || dead) continue;  // the other issuer's tile (or nothing left to do)
      const int64_t t0 = (int64_t)ti.tile * kTile;
      for (int j = 0; j < W; ++j) {
        const int tok = tok0 + j;
        const int64_t p = pos_g[j];
        if (!kRescore && t0 > p) continue;
        const int job = cnt++;
        if ((job & 1) != sub) continue;  // the other warpgroup of this issuer
        const int u = mw * kUnitsPer + job % kUnitsPer;
        const uint32_t m = (uint32_t)(job / kUnitsPer);
        // one prober per warpgroup; the other warps park on the named barrier
        if (!mbar_wait_group(bar_accf + 8 * u, m & 1, P.wait_ns, ept == 0, *abort != 0, 1 + wg, 128)) {
          if (ept == 0 && !*abort) {
            set_status(P.status, CSA2_ERR_TIMEOUT);
            *abort = 1;
          }
          dead = true;
          break;
        }
        tc::fence_after_sync();
        const float* wj = w_g + j * 64;
        const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + kColAcc + u * 64;
        const int ng = P.N / 16;
        // two halves of 32 columns (register budget); four independent chains,
        // weights read as float4 (broadcast)
        float a4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t r[2][16];
#pragma unroll
          for (int g = 0; g < 2; ++g)
            if (hf * 2 + g < ng) tc::ld_32x32b_x16(taddr + (hf * 2 + g) * 16, r[g]);
          tc::ld_wait();
          if (hf == 1) {  // the accumulator is free once the last load has landed
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(bar_acce + 8 * u);
          }
#pragma unroll
          for (int g = 0; g < 2; ++g)
            if (hf * 2 + g < ng) {
#pragma unroll
              for (int k4 = 0; k4 < 4; ++k4) {
                const float4 w4 = *reinterpret_cast<const float4*>(wj + (hf * 2 + g) * 16 + k4 * 4);
                a4[0] = fmaf(w4.x, fmaxf(__uint_as_float(r[g][k4 * 4 + 0]), 0.0f), a4[0]);
                a4[1] = fmaf(w4.y, fmaxf(__uint_as_float(r[g][k4 * 4 + 1]), 0.0f), a4[1]);
                a4[2] = fmaf(w4.z, fmaxf(__uint_as_float(r[g][k4 * 4 + 2]), 0.0f), a4[2]);
                a4[3] = fmaf(w4.w, fmaxf(__uint_as_float(r[g][k4 * 4 + 3]), 0.0f), a4[3]);
              }
            }
        }
        const float acc = (a4[0] + a4[1]) + (a4[2] + a4[3]);
        if (kRescore) {
          // pool entry i = tile*128 + row: position pool[i/8]*8 + i%8
          const int i = ti.tile * kTile + row;
          const int np = min(__ldg(P.pool_n + tok), P.pool_cap);
          const int32_t blk = (i / kBlock) < np ? __ldg(P.pool + (int64_t)tok * P.pool_cap + i / kBlock) : -1;
          const int64_t pos = (int64_t)blk * kBlock + (i % kBlock);
          const int64_t orow = (int64_t)(cur_b / P.qb.n_tok) * P.qb.n_tok + tok;  // selector * T + token
          if (i < P.pool_cap * kBlock) P.out[orow * P.ld + i] = (blk >= 0 && pos <= p) ? acc : -INFINITY;
        } else {
          const int64_t t = t0 + row;
          float sc = (t <= p) ? acc : -INFINITY;
          sc = fmaxf(sc, __shfl_xor_sync(0xffffffffu, sc, 1));
          sc = fmaxf(sc, __shfl_xor_sync(0xffffffffu, sc, 2));
          sc = fmaxf(sc, __shfl_xor_sync(0xffffffffu, sc, 4));
          if ((lane & 7) == 0 && t <= p) P.out[(int64_t)tok * P.ld + t / kBlock] = sc;
        }
      }
    }
  }
  // after a failed wait some tile loads may still be in flight: give them
  // time to land before the CTA's shared memory is released (bounded)
  if (threadIdx.x == 0 && *abort) {
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 200000ull) __nanosleep(1000);
  }
  __syncthreads();
  if (warp == 1) {
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

// scales: 1-D byte array [n_rows * spr], box of box_rows rows
int make_scales_map(CUtensorMap* m, const uint8_t* scales, int64_t n_rows, int spr, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return fail(CSA2_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[1] = {(cuuint64_t)(n_rows * spr)};
  cuuint64_t strides[1] = {0};
  cuuint32_t box[1] = {(cuuint32_t)(box_rows * spr)};
  cuuint32_t es[1] = {1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, const_cast<uint8_t*>(scales), dims, strides, box, es,
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

template <bool kRescore>
static int launch_index_tc(const csa2_query_batch* qb, const uint8_t* qc, const uint8_t* qs, const float* const* w,
                           int n_sel, int H, const csa2_fp4_cache* kc, const int32_t* pool, const int32_t* pool_n,
                           int pool_cap, float* out, int64_t ld, cudaStream_t st) {
  using namespace scan_tc;
  if (kc->n_rows * (kc->dim / 32) >= (int64_t(1) << 31)) return fail(CSA2_ERR_UNSUPPORTED, "cache too large for TMA");
  const int box_rows = kRescore ? kBlock : kChunk;
  CUtensorMap tmc, tms;
  if (int rc = make_codes_map(&tmc, kc->codes, kc->n_rows, kc->dim / 2, box_rows)) return rc;
  if (int rc = make_scales_map(&tms, kc->scales, kc->n_rows, kc->dim / 32, box_rows)) return rc;
  Params p{};
  p.qb = *qb;
  p.q_codes = qc;
  p.q_scales = qs;
  if (n_sel < 1 || n_sel > kMaxSel) return fail(CSA2_ERR_UNSUPPORTED, "1..%d selector layers per launch", kMaxSel);
  for (int i = 0; i < n_sel; ++i) p.w[i] = w[i];
  p.n_sel = n_sel;
  p.qchunks = kRescore ? 1 : std::max(1, (qb->max_q_per_seq + kMaxW - 1) / kMaxW);
  p.H = H;
  p.N = (H + 15) / 16 * 16;
  p.DI = kc->dim;
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
  p.status = status_ptr();
  p.wait_ns = 1000000000ull;  // 1 s
  static bool attr_done[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    if (int rc = cuda_check(
            cudaFuncSetAttribute(k_index_tc<kRescore>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Ly<kRescore>::kSmemBytes),
            "index smem attribute"))
      return rc;
    int fit = 0;  // one CTA of kThreads threads at this register count must fit on an SM
    if (int rc = cuda_check(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&fit, k_index_tc<kRescore>, kThreads,
                                                                          Ly<kRescore>::kSmemBytes),
                            "index occupancy"))
      return rc;
    if (fit < 1) return fail(CSA2_ERR_UNSUPPORTED, "index kernel does not fit on an SM");
    attr_done[dev] = true;
  }
  Launch L_(kRescore ? "rescore_tc" : "scan_tc", st);
  k_index_tc<kRescore><<<num_sms(), kThreads, Ly<kRescore>::kSmemBytes, st>>>(tmc, tms, p);
  return cuda_check(cudaGetLastError(), "k_index_tc");
}

int launch_scan_tc(const csa2_query_batch* qb, const uint8_t* qc, const uint8_t* qs, const float* w, int H,
                   const csa2_fp4_cache* kc, float* bs, int64_t ld, cudaStream_t st) {
  return launch_index_tc<false>(qb, qc, qs, &w, 1, H, kc, nullptr, nullptr, 0, bs, ld, st);
}

// n_sel selector layers at once: queries [n_sel][T][H][...], weights w[sel],
// scores [n_sel][T][8P]
int launch_rescore_tc(const csa2_query_batch* qb, const uint8_t* qc, const uint8_t* qs, const float* const* w,
                      int n_sel, int H, const csa2_fp4_cache* kc, const int32_t* pool, const int32_t* pool_n, int P,
                      float* scores, cudaStream_t st) {
  return launch_index_tc<true>(qb, qc, qs, w, n_sel, H, kc, pool, pool_n, P, scores, (int64_t)P * kBlock, st);
}

}  // namespace csa2
