// select.cuh -- top-k selection without a global sort: the block top-P pool
// (mode 0) and the pool's top-K positions (mode 1), for one or several
// selector layers at once.
//
// The candidates of one (selector, token) group are split over S CTAs
// (gridDim.x).  Scores become order-preserving unsigned keys (score_key);
// invalid candidates map to 0 and are never selected.
//
//   range     count, smallest and largest valid key of the group;
//   rounds    the key range [base, base + range] is cut into at most 4096 bins
//             of 2^shift keys; the bin where the count from the top reaches
//             the number still wanted holds the k-th largest key, and the next
//             round cuts only that bin.  A 32-bit key needs at most three
//             rounds; a round ends the search early when the whole bin is
//             taken or its width is one key;
//   output    keys above the threshold key, and the lowest-id ties at it,
//             written in ascending id order: every CTA owns a contiguous id
//             segment, every warp a contiguous 512-id stretch of each tile.
//
// With S > 1 the group's CTAs merge their counts and histograms in global
// memory (SelGroup, zeroed before the launch) between group barriers; such
// launches are cooperative, so all CTAs of the grid are resident together and
// every barrier wait ends (each is also bounded in time and reports
// CSA2_ERR_TIMEOUT through the status word).
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
constexpr int kSelMaxSplit = 64;
constexpr int kSelMaxGroups = 148;  // groups of a split launch (fewer than the SMs)

struct SelGroup {
  uint32_t bar;                  // barrier arrivals (S per barrier)
  uint32_t kmin_inv;             // max over CTAs of ~(smallest valid key)
  uint32_t kmax;                 // largest valid key
  int32_t count;                 // valid candidates
  int32_t cta_gt[kSelMaxSplit];  // per CTA: keys above the threshold
  int32_t cta_eq[kSelMaxSplit];  // per CTA: keys equal to it
  int32_t hist[kSelRounds][kSelBins];
};

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
  SelGroup* grp;   // [n_sel][T] when gridDim.x > 1
  int* status;
  uint64_t wait_ns;
};

// candidate i -> output id: mode 0 the candidate itself (a block), mode 1 the
// position of pool entry i, mode 2 the id listed for candidate i (merging
// candidate lists gathered from several ranks)
__device__ __forceinline__ int32_t sel_id(int mode, int i, const int32_t* pool_row) {
  if (mode == 2) return __ldg(pool_row + i);
  return mode == 0 ? i : __ldg(pool_row + i / kBlock) * kBlock + (i % kBlock);
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// barrier of the S CTAs of one group: returns false (and sets the status)
// when the wait ran past its limit
__device__ __forceinline__ bool group_barrier(uint32_t* bar, uint32_t target, uint64_t wait_ns, int* status,
                                              int* flag_s) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(bar, 1u);
    const uint64_t t0 = globaltimer_ns();
    int ok = 1;
    for (uint32_t i = 1; ld_acquire_u32(bar) < target; ++i) {
      if ((i & 15) == 0 && globaltimer_ns() - t0 > wait_ns) {  // the timer is read every 16th probe
        set_status(status, CSA2_ERR_TIMEOUT);
        ok = 0;
        break;
      }
      __nanosleep(64);
    }
    __threadfence();
    *flag_s = ok;
  }
  __syncthreads();
  return *flag_s != 0;
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
  __shared__ int flag_s;

  const int S = gridDim.x, s = blockIdx.x, tok = blockIdx.y;
  const int T = P.qb.n_tok;
  const int64_t g = (int64_t)blockIdx.z * T + tok;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int64_t p = __ldg(P.qb.tok_pos + tok);
  const int n = P.mode == 0   ? (int)((p + kBlock) / kBlock)
                : P.mode == 1 ? min(__ldg(P.pool_n + tok), P.P) * kBlock
                              : P.P;  // mode 2: P candidates a token
  const float* sc = P.score + g * P.ld;
  const int32_t* pool_row = P.pool + (int64_t)tok * P.P;
  SelGroup* G = S > 1 ? P.grp + g : nullptr;
  uint32_t n_bar = 0;

  // this CTA's segment, in tiles of 8192 ids; the first tile stays in registers
  const int seg = (n + S - 1) / S;
  const int lo = min(n, s * seg), hi = min(n, lo + seg);
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
  if (G) {
    if (threadIdx.x == 0) {
      atomicAdd(&G->count, cnt);
      atomicMax(&G->kmin_inv, ~kmin);
      atomicMax(&G->kmax, kmax);
    }
    if (!group_barrier(&G->bar, S * ++n_bar, P.wait_ns, P.status, &flag_s)) return;
    cnt = __ldcg(&G->count);
    kmin = ~__ldcg(&G->kmin_inv);
    kmax = __ldcg(&G->kmax);
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
      if (G) {
        for (int b = threadIdx.x; b < kSelBins; b += kSelThreads)
          if (hist[b]) atomicAdd(&G->hist[r][b], hist[b]);
        if (!group_barrier(&G->bar, S * ++n_bar, P.wait_ns, P.status, &flag_s)) return;
        for (int b = threadIdx.x; b < kSelBins; b += kSelThreads) hist[b] = __ldcg(&G->hist[r][b]);
        __syncthreads();
      }
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
      if (bstar < 0) {  // only with inconsistent counts; every CTA of the group sees the same
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

  // ---- output: this CTA's counts, then its place among the group's CTAs
  auto is_gt = [&](uint32_t key) { return key != 0u && key > thr; };
  auto is_eq = [&](uint32_t key) { return need_eq > 0 && key != 0u && key == thr; };
  int gt = 0, eq = 0;
  visit([&](uint32_t key) {
    gt += is_gt(key);
    eq += is_eq(key);
  });
  gt = __reduce_add_sync(0xffffffffu, gt);
  eq = __reduce_add_sync(0xffffffffu, eq);
  if (lane == 0) {
    red[0][wid] = gt;
    red[1][wid] = eq;
  }
  __syncthreads();
  gt = __reduce_add_sync(0xffffffffu, lane < kSelWarps ? red[0][lane] : 0);
  eq = __reduce_add_sync(0xffffffffu, lane < kSelWarps ? red[1][lane] : 0);
  int run_out = 0, run_eq = 0;  // selections and ties in the group's CTAs before this one
  if (G) {
    if (threadIdx.x == 0) {
      G->cta_gt[s] = gt;
      G->cta_eq[s] = eq;
    }
    if (!group_barrier(&G->bar, S * ++n_bar, P.wait_ns, P.status, &flag_s)) return;
    for (int c = 0; c < s; ++c) {
      const int e = __ldcg(&G->cta_eq[c]);
      run_out += __ldcg(&G->cta_gt[c]) + max(0, min(e, need_eq - run_eq));
      run_eq += e;
    }
  }
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
  if (s == 0) {
    for (int j = k_eff + threadIdx.x; j < P.k_out; j += kSelThreads) o[j] = -1;
    if (threadIdx.x == 0) P.out_n[g] = k_eff;
  }
}

}  // namespace csa2
