// select.cuh -- top-k selection without a global sort: the block top-P pool
// (mode 0) and the pool's top-K positions (mode 1), for one or several
// selector layers at once.  Scores become order-preserving unsigned keys
// (score_key); invalid candidates map to 0 and are never selected.
//
// k_select_cluster (the decode path) starts from the key counts that the
// scoring kernels leave behind (see its own comment below).  k_select takes
// no counts: one CTA per (selector, token) group runs the rounds itself
// (the entry point without a workspace, and candidate lists too long for the
// cluster kernel's shared memory):
//   range     count, smallest and largest valid key of the group;
//   rounds    the key range [base, base + range] is cut into at most 4096 bins
//             of 2^shift keys; the bin where the count from the top reaches
//             the number still wanted holds the k-th largest key, and the next
//             round cuts only that bin.  A 32-bit key needs at most three
//             rounds; a round ends the search early when the whole bin is
//             taken or its width is one key;
//   output    keys above the threshold key, and the lowest-id ties at it,
//             written in ascending id order: every warp owns a contiguous
//             512-id stretch of each tile.
#pragma once

#include "common.cuh"

namespace csa2 {

constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSelPer = 16;                      // keys per thread per tile
constexpr int kSelTile = kSelThreads * kSelPer;  // 8192 ids per tile
constexpr int kSelWarpSpan = 32 * kSelPer;       // 512 ids per warp per tile
constexpr int kSelBins = 4096;
constexpr int kSelRounds = 3;
constexpr int kSelMaxGroups = 148;  // CTAs of a split selection launch at most (the SMs)

struct SelParams {
  csa2_query_batch qb;
  const float* score;  // [n_sel][T][ld]
  int64_t ld;
  int mode;
  const int32_t* pool;    // [T][P] (mode 1), candidate ids [T][P] (mode 2)
  const int32_t* pool_n;  // [T]
  int P;
  int k_out;
  int32_t* out;    // [n_sel][T][k_out]
  int32_t* out_n;  // [n_sel][T]
  int* status;
};

// candidate i -> output id: mode 0 the candidate itself (a block), mode 1 the
// position of pool entry i
__device__ __forceinline__ int32_t sel_id(int mode, int i, const int32_t* pool_row) {
  return mode == 0 ? i : __ldg(pool_row + i / kBlock) * kBlock + (i % kBlock);
}

// one tile of a CTA's segment: lane l of warp w holds ids
// tile + w*512 + j*32 + l (j < 16); keys past the segment end are 0
__device__ __forceinline__ void sel_load_tile(const float* sc, int tile, int hi, uint32_t (&k)[kSelPer]) {
  const int base = tile + (threadIdx.x >> 5) * kSelWarpSpan + (threadIdx.x & 31);
  float v[kSelPer];
#pragma unroll
  for (int j = 0; j < kSelPer; ++j) {
    const int i = base + j * 32;
    v[j] = i < hi ? __ldg(sc + i) : -INFINITY;
  }
#pragma unroll
  for (int j = 0; j < kSelPer; ++j) k[j] = score_key(v[j]);
}

__global__ void __launch_bounds__(kSelThreads) k_select(const __grid_constant__ SelParams P) {
  __shared__ int hist[kSelBins];
  __shared__ int red[3][kSelWarps];
  __shared__ uint32_t redu[2][kSelWarps];
  __shared__ int wgt[kSelWarps], weq[kSelWarps];

  const int tok = blockIdx.y;
  const int T = P.qb.n_tok;
  const int64_t g = (int64_t)blockIdx.z * T + tok;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  grid_dep_wait();  // the scores of the previous kernel
  grid_dep_launch();
  const int64_t p = __ldg(P.qb.tok_pos + tok);
  int n = P.mode == 0 ? (int)max((p + kBlock) / kBlock, (int64_t)0) : min(__ldg(P.pool_n + tok), P.P) * kBlock;
  n = (int)max((int64_t)0, min((int64_t)n, P.ld));  // never past the score row
  const float* sc = P.score + g * P.ld;
  const int32_t* pool_row = P.pool + (int64_t)tok * P.P;

  // the group's ids in tiles of 8192; the first tile stays in registers
  const int lo = 0, hi = n;
  uint32_t k0[kSelPer];
  sel_load_tile(sc, lo, hi, k0);
  auto visit = [&](auto&& f) {
#pragma unroll
    for (int j = 0; j < kSelPer; ++j) f(k0[j]);
    for (int t = lo + kSelTile; t < hi; t += kSelTile) {
      uint32_t k[kSelPer];
      sel_load_tile(sc, t, hi, k);
#pragma unroll
      for (int j = 0; j < kSelPer; ++j) f(k[j]);
    }
  };

  // ---- range and count of the valid keys
  int cnt = 0;
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
  visit([&](uint32_t key) {
    if (key) {
      ++cnt;
      kmin = min(kmin, key);
      kmax = max(kmax, key);
    }
  });
  cnt = __reduce_add_sync(0xffffffffu, cnt);
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  if (lane == 0) {
    red[0][wid] = cnt;
    redu[0][wid] = kmin;
    redu[1][wid] = kmax;
  }
  __syncthreads();
  {
    const int c = lane < kSelWarps ? red[0][lane] : 0;
    const uint32_t mn = lane < kSelWarps ? redu[0][lane] : 0xFFFFFFFFu;
    const uint32_t mx = lane < kSelWarps ? redu[1][lane] : 0u;
    cnt = __reduce_add_sync(0xffffffffu, c);
    kmin = __reduce_min_sync(0xffffffffu, mn);
    kmax = __reduce_max_sync(0xffffffffu, mx);
  }

  // ---- threshold: selected = valid keys > thr, plus the first need_eq ties at thr
  const int k_eff = min(P.k_out, cnt);
  uint32_t thr = 0;
  int need_eq = 0;
  if (k_eff < cnt) {
    uint32_t base = kmin, range = kmax - kmin;
    int remaining = k_eff;
    for (int r = 0; r < kSelRounds; ++r) {
      if (range == 0) {  // every remaining candidate has key == base
        thr = base;
        need_eq = remaining;
        break;
      }
      const int bits = 32 - __clz(range);
      const int shift = bits > 12 ? bits - 12 : 0;
      for (int b = threadIdx.x; b < kSelBins; b += kSelThreads) hist[b] = 0;
      __syncthreads();
      visit([&](uint32_t key) {
        const uint32_t d = key - base;
        if (key && key >= base && d <= range) atomicAdd(&hist[d >> shift], 1);
      });
      __syncthreads();
      // bin where the count from the top reaches `remaining`: 8 bins a thread
      // (thread 0 holds the top bins), then a block scan of the thread sums
      constexpr int kPerT = kSelBins / kSelThreads;
      const int top = kSelBins - 1 - threadIdx.x * kPerT;
      int c[kPerT], tot = 0;
#pragma unroll
      for (int j = 0; j < kPerT; ++j) {
        c[j] = hist[top - j];
        tot += c[j];
      }
      int incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (lane == 31) red[1][wid] = incl;
      if (threadIdx.x == 0) red[2][0] = -1;
      __syncthreads();
      int before = incl - tot;
      for (int w = 0; w < wid; ++w) before += red[1][w];
#pragma unroll
      for (int j = 0; j < kPerT; ++j) {
        if (before < remaining && before + c[j] >= remaining) {  // exactly one thread
          red[2][0] = top - j;
          red[2][1] = before;
          red[2][2] = c[j];
        }
        before += c[j];
      }
      __syncthreads();
      const int bstar = red[2][0], above = red[2][1], in_bin = red[2][2];
      __syncthreads();  // red[] and hist[] are reused
      if (bstar < 0) {  // only with inconsistent counts
        set_status(P.status, CSA2_ERR_RANGE);
        return;
      }
      remaining -= above;
      base += (uint32_t)bstar << shift;
      range = min(range - ((uint32_t)bstar << shift), shift ? (1u << shift) - 1u : 0u);
      if (in_bin == remaining) {  // the whole bin is taken
        thr = base - 1u;
        need_eq = 0;
        break;
      }
      if (shift == 0) {  // one key per bin
        thr = base;
        need_eq = remaining;
        break;
      }
    }
  }

  // ---- output, in ascending id order
  auto is_gt = [&](uint32_t key) { return key != 0u && key > thr; };
  auto is_eq = [&](uint32_t key) { return need_eq > 0 && key != 0u && key == thr; };
  int run_out = 0, run_eq = 0;  // selections and ties in the tiles before this one
  int32_t* o = P.out + g * P.k_out;
  for (int t = lo; t < hi; t += kSelTile) {
    uint32_t k[kSelPer];
    if (t == lo) {
#pragma unroll
      for (int j = 0; j < kSelPer; ++j) k[j] = k0[j];
    } else {
      sel_load_tile(sc, t, hi, k);
    }
    int wg = 0, we = 0;
#pragma unroll
    for (int j = 0; j < kSelPer; ++j) {
      wg += __popc(__ballot_sync(0xffffffffu, is_gt(k[j])));
      we += __popc(__ballot_sync(0xffffffffu, is_eq(k[j])));
    }
    if (lane == 0) {
      wgt[wid] = wg;
      weq[wid] = we;
    }
    __syncthreads();
    // selections and ties of the warps before this one in the tile
    int out_before = run_out, eq_before = run_eq;
    for (int w = 0; w < wid; ++w) {
      out_before += wgt[w] + max(0, min(weq[w], need_eq - eq_before));
      eq_before += weq[w];
    }
    int written = out_before, ties = eq_before;
    const int base = t + wid * kSelWarpSpan + lane;
#pragma unroll
    for (int j = 0; j < kSelPer; ++j) {
      const bool gsel = is_gt(k[j]);
      const bool e = is_eq(k[j]);
      const uint32_t em = __ballot_sync(0xffffffffu, e);
      const int e_rank = ties + __popc(em & ((1u << lane) - 1u));
      const bool take = gsel || (e && e_rank < need_eq);
      const uint32_t sm = __ballot_sync(0xffffffffu, take);
      if (take) o[written + __popc(sm & ((1u << lane) - 1u))] = sel_id(P.mode, base + j * 32, pool_row);
      written += __popc(sm);
      ties += __popc(em);
    }
    for (int w = 0; w < kSelWarps; ++w) {  // the tile's totals
      run_out += wgt[w] + max(0, min(weq[w], need_eq - run_eq));
      run_eq += weq[w];
    }
    __syncthreads();
  }
  for (int j = k_eff + threadIdx.x; j < P.k_out; j += kSelThreads) o[j] = -1;
  if (threadIdx.x == 0) P.out_n[g] = k_eff;
}


// ---------------------------------------------------------------------------
// Histogram-seeded selection on a thread-block cluster (k_select_cluster)
//
// The scoring kernels (scan and pool rescoring) count every valid score of a
// group by the top 12 bits of its key as they store it (kHistBins bins in
// global memory, zeroed before them).  From those counts every CTA knows at
// once the bin b1 that holds the k-th largest key.  The S CTAs of a group
// form one cluster (S = 1 .. 16); all shared state lives in the shared memory
// of CTA 0 of the cluster, which the others reach through distributed shared
// memory:
//   A  every CTA sets, in CTA 0's selection bitmap (one bit per candidate),
//      the bits of its keys above b1 (of b1 too when the whole bin is
//      taken), clears its words of the tie bitmap, and appends the keys of
//      bin b1 (when only part of it is taken) to CTA 0's candidate list;
//   B  after a cluster barrier, CTA 0 finds the exact k-th key among the
//      candidates (two more radix digits of 12 and 8 bits) and sets the bits
//      of the candidates above it, and of those equal to it in the tie bitmap;
//   C  CTA 0 turns the bitmaps into the ascending list of ids: every
//      selected id, and the lowest-id ties while any are still wanted.
// A candidate list longer than its capacity is replaced by rescans of the
// group's scores (correct, slower; only for very flat score distributions).
// CTA 0 leaves the group's counts zeroed for the next scoring launch.

constexpr int kSelCandCap = 8192;  // candidates of bin b1 kept in shared memory

struct SelCParams {
  csa2_query_batch qb;
  const float* score;  // [n_sel][T][ld]
  int64_t ld;
  int mode;               // 0 blocks, 1 pool positions
  const int32_t* pool;    // [T][P] (mode 1)
  const int32_t* pool_n;  // [T]
  int P;
  int k_out;
  int32_t* out;    // [n_sel][T][k_out]
  int32_t* out_n;  // [n_sel][T]
  uint32_t* hist;  // [n_sel * T][kHistBins], filled by the scoring kernel
  int words;       // bitmap words (>= candidates / 32)
  int cap;         // candidate list capacity (<= kSelCandCap)
  int* status;
};

// dynamic shared memory of k_select_cluster (CTA 0's is the group's)
struct SelCLayout {
  uint32_t sel, tie, cand, pool, n_cand, bytes;
  __host__ __device__ SelCLayout(int words, int cap, int P) {
    sel = 0;
    tie = sel + (uint32_t)words * 4;
    cand = (tie + (uint32_t)words * 4 + 15) & ~15u;
    pool = cand + (uint32_t)cap * 8;
    n_cand = (pool + (uint32_t)P * 4 + 15) & ~15u;
    bytes = n_cand + 16;
  }
};

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t map_to_rank0(uint32_t saddr) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, 0;" : "=r"(r) : "r"(saddr));
  return r;
}
__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void st_cluster_v2(uint32_t addr, uint32_t a, uint32_t b) {
  asm volatile("st.shared::cluster.v2.u32 [%0], {%1, %2};" ::"r"(addr), "r"(a), "r"(b) : "memory");
}
__device__ __forceinline__ uint32_t atom_cluster_add(uint32_t addr, uint32_t v) {
  uint32_t old;
  asm volatile("atom.shared::cluster.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(addr), "r"(v) : "memory");
  return old;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// the bin where the count from the top (bins nb-1, nb-2, ...) reaches
// min(want, total): every thread of the block calls it; kPer bins a thread
// (threads past nb / kPer hold none).  *bin = -1 when want <= 0 or total = 0.
template <int kPer, typename Get>
__device__ __forceinline__ void sel_find_bin(Get get, int nb, int want, int* sh, int* bin, int* above, int* in,
                                             int* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int act = nb / kPer;
  const int top = nb - 1 - (int)threadIdx.x * kPer;
  int c[kPer], tot = 0;
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    c[j] = (int)threadIdx.x < act ? get(top - j) : 0;
    tot += c[j];
  }
  int incl = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) sh[wid] = incl;
  if (threadIdx.x == 0) sh[kSelWarps] = -1;
  __syncthreads();
  int before = incl - tot, all = 0;
  for (int w = 0; w < kSelWarps; ++w) {
    const int v = sh[w];
    if (w < wid) before += v;
    all += v;
  }
  want = min(want, all);
  if (want > 0) {
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      if (before < want && before + c[j] >= want) {  // exactly one thread
        sh[kSelWarps] = top - j;
        sh[kSelWarps + 1] = before;
        sh[kSelWarps + 2] = c[j];
      }
      before += c[j];
    }
  }
  __syncthreads();
  *bin = sh[kSelWarps];
  *above = sh[kSelWarps + 1];
  *in = sh[kSelWarps + 2];
  *total = all;
  __syncthreads();  // sh is reused
}

// exclusive block scan of two counts: this thread's prefixes and the totals
__device__ __forceinline__ void sel_scan2(int a, int b, int* sh, int* ea, int* eb, int* ta, int* tb) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int ia = a, ib = b;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int ya = __shfl_up_sync(0xffffffffu, ia, o);
    const int yb = __shfl_up_sync(0xffffffffu, ib, o);
    if (lane >= o) {
      ia += ya;
      ib += yb;
    }
  }
  if (lane == 31) {
    sh[wid] = ia;
    sh[kSelWarps + wid] = ib;
  }
  __syncthreads();
  int pa = 0, pb = 0, sa = 0, sb = 0;
  for (int w = 0; w < kSelWarps; ++w) {
    const int va = sh[w], vb = sh[kSelWarps + w];
    if (w < wid) {
      pa += va;
      pb += vb;
    }
    sa += va;
    sb += vb;
  }
  *ea = pa + ia - a;
  *eb = pb + ib - b;
  *ta = sa;
  *tb = sb;
  __syncthreads();  // sh is reused
}

// grid (S, T, n_sel), clusters of (S, 1, 1); dynamic shared memory SelCLayout
// (at most 64 registers: two CTAs of a launch with more groups than SMs
// share an SM, one's serial phases hiding the other's)
__global__ void __launch_bounds__(kSelThreads, 2) k_select_cluster(const __grid_constant__ SelCParams P) {
  extern __shared__ __align__(16) uint8_t sm[];
  __shared__ int hist_s[kHistBins];
  __shared__ int sh[2 * kSelWarps + 4];

  const int S = gridDim.x, tok = blockIdx.y;
  const int s = (int)cluster_rank();
  const int T = P.qb.n_tok;
  const int64_t g = (int64_t)blockIdx.z * T + tok;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const SelCLayout Lo(P.words, P.cap, P.mode == 1 ? P.P : 0);
  grid_dep_wait();  // the scores and key counts of the previous kernel
  grid_dep_launch();
  uint32_t* bsel = reinterpret_cast<uint32_t*>(sm + Lo.sel);
  uint32_t* btie = reinterpret_cast<uint32_t*>(sm + Lo.tie);
  uint2* cand = reinterpret_cast<uint2*>(sm + Lo.cand);
  int32_t* pool_s = reinterpret_cast<int32_t*>(sm + Lo.pool);
  uint32_t* n_cand = reinterpret_cast<uint32_t*>(sm + Lo.n_cand);
  // CTA 0's shared memory seen from this CTA (distributed shared memory)
  const uint32_t r_sel = map_to_rank0(smem_u32(bsel)), r_tie = map_to_rank0(smem_u32(btie));
  const uint32_t r_cand = map_to_rank0(smem_u32(cand)), r_ncand = map_to_rank0(smem_u32(n_cand));

  const int64_t p = __ldg(P.qb.tok_pos + tok);
  // candidates: never more than a score row or a bitmap holds (a query
  // position past the batch's max_seq_len is not read past the row)
  int n = P.mode == 0 ? (int)max((p + kBlock) / kBlock, (int64_t)0) : min(__ldg(P.pool_n + tok), P.P) * kBlock;
  n = (int)max((int64_t)0, min((int64_t)n, min((int64_t)P.words * 32, P.ld)));
  const float* sc = P.score + g * P.ld;
  const int32_t* pool_row = P.pool + (int64_t)tok * P.P;
  uint32_t* H = P.hist + g * kHistBins;

  if (s == 0 && threadIdx.x == 0) *n_cand = 0u;
  cluster_sync_all();  // every CTA of the cluster runs; CTA 0's counter is set

  // ---- the bin b1 of the k-th largest key, from the scoring kernel's counts
  int b1, above1, in1, cnt;
  sel_find_bin<kHistBins / kSelThreads>([&](int b) { return (int)__ldcg(H + b); }, kHistBins, P.k_out, sh, &b1,
                                        &above1, &in1, &cnt);
  const int k_eff = min(P.k_out, cnt);
  const bool all = k_eff == cnt;              // every valid key is taken
  const int rem1 = all ? 0 : k_eff - above1;  // still wanted from bin b1
  const bool whole = !all && in1 == rem1;     // the whole bin is taken
  const uint32_t ub1 = all ? 0u : (uint32_t)b1;

  // ---- A: this CTA's segment (a multiple of 512 ids, so that a warp's 32
  // consecutive ids fill one bitmap word); the next tile's keys are loaded
  // while this one is processed
  const int seg = ((n + S - 1) / S + kSelWarpSpan - 1) / kSelWarpSpan * kSelWarpSpan;
  const int lo = min(n, s * seg), hi = min(n, lo + seg);
  uint32_t kn[kSelPer];
  if (lo < hi) sel_load_tile(sc, lo, hi, kn);
  for (int t = lo; t < hi; t += kSelTile) {
    uint32_t k[kSelPer];
#pragma unroll
    for (int j = 0; j < kSelPer; ++j) k[j] = kn[j];
    if (t + kSelTile < hi) sel_load_tile(sc, t + kSelTile, hi, kn);
    const int wbase = t + wid * kSelWarpSpan;  // ids wbase + j*32 + lane
    uint32_t myword = 0, cm[kSelPer];
    int nc = 0;
#pragma unroll
    for (int j = 0; j < kSelPer; ++j) {
      const uint32_t bin = k[j] >> kHistShift;
      const bool sel = k[j] != 0u && (all || bin > ub1 || (whole && bin == ub1));
      const bool cd = k[j] != 0u && !all && !whole && bin == ub1;
      const uint32_t w = __ballot_sync(0xffffffffu, sel);
      if (lane == j) myword = w;
      cm[j] = __ballot_sync(0xffffffffu, cd);
      nc += __popc(cm[j]);
    }
    if (lane < kSelPer && wbase + lane * 32 < hi) {
      const uint32_t wi = (uint32_t)((wbase >> 5) + lane) * 4;
      st_cluster_u32(r_sel + wi, myword);
      st_cluster_u32(r_tie + wi, 0u);
    }
    if (nc) {  // warp-uniform
      uint32_t off = 0;
      if (lane == 0) off = atom_cluster_add(r_ncand, (uint32_t)nc);
      off = __shfl_sync(0xffffffffu, off, 0);
#pragma unroll
      for (int j = 0; j < kSelPer; ++j) {
        if ((cm[j] >> lane) & 1u) {
          const uint32_t i = off + __popc(cm[j] & ((1u << lane) - 1u));
          if (i < (uint32_t)P.cap) st_cluster_v2(r_cand + i * 8, k[j], (uint32_t)(wbase + j * 32 + lane));
        }
        off += __popc(cm[j]);
      }
    }
  }
  cluster_sync_all();  // every bitmap word and candidate is in CTA 0
  if (s != 0) return;  // nothing reads the other CTAs' shared memory any more

  // ---- B: the exact k-th key among the candidates of bin b1
  if (P.mode == 1)
    for (int i = threadIdx.x; i < P.P; i += kSelThreads) pool_s[i] = __ldg(pool_row + i);
  uint32_t sel_lo = 0xFFFFFFFFu, tie_key = 0u;  // select key >= sel_lo; ties: key == tie_key
  int need_eq = 0;
  bool range_err = false;
  if (!all && !whole) {
    const int m = (int)*n_cand;
    const bool fits = m <= P.cap;
    // every candidate (key in bin b1): from the list, or by rescanning
    auto visit = [&](auto&& f) {
      if (fits) {
        for (int i = threadIdx.x; i < m; i += kSelThreads) f(cand[i].x, cand[i].y);
      } else {
        // (a rare path: rolled, one key at a time)
        const int wbase = wid * kSelWarpSpan + lane;
#pragma unroll 1
        for (int t = 0; t < n; t += kSelTile)
#pragma unroll 1
          for (int j = 0; j < kSelPer; ++j) {
            const int i = t + wbase + j * 32;
            const uint32_t key = i < n ? score_key(__ldg(sc + i)) : 0u;
            if (key != 0u && (key >> kHistShift) == ub1) f(key, (uint32_t)i);
          }
      }
    };
    // digit 2: key bits 19..8
    for (int b = threadIdx.x; b < kHistBins; b += kSelThreads) hist_s[b] = 0;
    __syncthreads();
    visit([&](uint32_t key, uint32_t) { atomicAdd(&hist_s[(key >> 8) & 0xFFFu], 1); });
    __syncthreads();
    int b2, above2, in2, tot2;
    sel_find_bin<kHistBins / kSelThreads>([&](int b) { return hist_s[b]; }, kHistBins, rem1, sh, &b2, &above2,
                                          &in2, &tot2);
    const int rem2 = rem1 - above2;
    const uint32_t pre2 = (ub1 << 12) | (uint32_t)max(b2, 0);  // the top 24 key bits of the threshold
    if (b2 < 0) {  // counts and scores disagree
      range_err = true;
    } else if (in2 == rem2) {
      sel_lo = pre2 << 8;
    } else {
      // digit 3: key bits 7..0 of the candidates in (b1, b2)
      for (int b = threadIdx.x; b < 256; b += kSelThreads) hist_s[b] = 0;
      __syncthreads();
      visit([&](uint32_t key, uint32_t) {
        if ((key >> 8) == pre2) atomicAdd(&hist_s[key & 0xFFu], 1);
      });
      __syncthreads();
      int b3, above3, in3, tot3;
      sel_find_bin<1>([&](int b) { return hist_s[b]; }, 256, rem2, sh, &b3, &above3, &in3, &tot3);
      const int rem3 = rem2 - above3;
      const uint32_t key3 = (pre2 << 8) | (uint32_t)max(b3, 0);
      if (b3 < 0) {
        range_err = true;
      } else if (in3 == rem3) {
        sel_lo = key3;
      } else {
        sel_lo = key3 + 1u;  // keys are at most 0xFF800000 (+inf): no wrap
        tie_key = key3;
        need_eq = rem3;
      }
    }
    visit([&](uint32_t key, uint32_t id) {
      if (key >= sel_lo) atomicOr(bsel + (id >> 5), 1u << (id & 31));
      else if (need_eq > 0 && key == tie_key) atomicOr(btie + (id >> 5), 1u << (id & 31));
    });
  }
  __syncthreads();

  // ---- C: bitmaps -> ascending ids; position of a selected id = selected
  // ids before it + min(ties before it, need_eq).  A thread takes wpt
  // consecutive words (1..8: every thread busy on short lists)
  int32_t* o = P.out + g * P.k_out;
  const int words_n = (n + 31) / 32;
  const int wpt = min(8, max(1, (words_n + kSelThreads - 1) / kSelThreads));
  int run_sel = 0, run_tie = 0, bad = 0;
  for (int w0 = 0; w0 < words_n; w0 += kSelThreads * wpt) {
    const int wi = w0 + (int)threadIdx.x * wpt;
    uint32_t sw[8], tw[8];
    int cs = 0, ct = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const bool in = j < wpt && wi + j < words_n;
      sw[j] = in ? bsel[wi + j] : 0u;
      tw[j] = (need_eq > 0 && in) ? btie[wi + j] : 0u;
      if (wi + j == words_n - 1 && (n & 31)) {  // ids past n: not candidates
        sw[j] &= (1u << (n & 31)) - 1u;
        tw[j] &= (1u << (n & 31)) - 1u;
      }
      cs += __popc(sw[j]);
      ct += __popc(tw[j]);
    }
    int es, et, ts, tt;
    sel_scan2(cs, ct, sh, &es, &et, &ts, &tt);
    int ns = run_sel + es, nt = run_tie + et;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint32_t mk = sw[j] | tw[j];
      while (mk) {
        const int b = __ffs(mk) - 1;
        mk &= mk - 1u;
        const int id = (wi + j) * 32 + b;
        int pos = -1;
        if ((sw[j] >> b) & 1u) {
          pos = ns + min(nt, need_eq);
          ++ns;
        } else {
          if (nt < need_eq) pos = ns + nt;
          ++nt;
        }
        if (pos >= 0) {
          if (pos < k_eff) o[pos] = P.mode == 0 ? id : pool_s[id / kBlock] * kBlock + (id % kBlock);
          else bad = 1;
        }
      }
    }
    run_sel += ts;
    run_tie += tt;
  }
  if (range_err || bad || run_sel + min(run_tie, need_eq) != k_eff) set_status(P.status, CSA2_ERR_RANGE);
  for (int j = k_eff + threadIdx.x; j < P.k_out; j += kSelThreads) o[j] = -1;
  // leave the counts zeroed for the next scoring launch (every CTA of the
  // cluster read them before the second cluster barrier)
  for (int b = threadIdx.x; b < kHistBins; b += kSelThreads) H[b] = 0u;
  if (threadIdx.x == 0) P.out_n[g] = k_eff;
}

}  // namespace csa2
