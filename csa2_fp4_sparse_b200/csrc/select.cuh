// select.cuh -- top-k selection without a global sort (block top-P pool and
// pool top-K positions).  One CTA of 1024 threads per query token.
//
//   keys      order-preserving unsigned images of the fp32 scores (score_key);
//             invalid candidates map to 0 and are never selected
//   pass A    range [min, max] and count of the valid scores;
//   pass B    4096-bin linear histogram over that range (monotone in the
//             score, so bins are ordered); the bin where the count from the
//             top reaches k holds the k-th largest score;
//   pass C    that bin's keys are gathered into shared memory (few in
//             practice) and its exact k-th key is found by byte-wise radix
//             steps there (or on global memory if they do not fit);
//   output    every warp owns a contiguous id range: it counts its selections,
//             a scan over the 32 warps gives each its output offset, and ties
//             at the k-th key go to the lowest ids (warp ranges are in id
//             order); ids are written ascending.
#pragma once

#include "common.cuh"

namespace csa2 {

constexpr int kSel2Threads = 1024;
constexpr int kSelCand = 6144;  // shared candidate capacity

struct SelShared {
  int hist[256];
  int wsum[32];
  int wsum2[32];
  uint32_t cand_key[kSelCand];
  int cand_n;
  uint32_t prefix;
  int remaining;
  int n_valid;
};

__device__ __forceinline__ void hist_add(int* hist, uint32_t digit, bool active) {
  const uint32_t am = __ballot_sync(0xffffffffu, active);
  if (!active) return;
  const uint32_t peers = __match_any_sync(am, digit);
  if ((__ffs(peers) - 1) == (int)(threadIdx.x & 31)) atomicAdd(&hist[digit], __popc(peers));
}

// after a histogram: pick the byte where the count from the top reaches `remaining`
__device__ __forceinline__ void pick_digit(SelShared& S, int shift) {
  __syncthreads();
  if (threadIdx.x < 32) {
    // warp 0: suffix sums over 256 bins, 8 bins per lane
    const int lane = threadIdx.x;
    int c[8], tot = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      c[i] = S.hist[255 - (lane * 8 + i)];  // descending digit order
      tot += c[i];
    }
    int incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int before = incl - tot;  // keys with a larger digit than this lane's first bin
    const int rem = S.remaining;
    int found = -1, above = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (found < 0 && before + c[i] >= rem) {
        found = 255 - (lane * 8 + i);
        above = before;
      }
      before += c[i];
    }
    const uint32_t mask = __ballot_sync(0xffffffffu, found >= 0);
    const int src = __ffs(mask) - 1;
    found = __shfl_sync(0xffffffffu, found, src);
    above = __shfl_sync(0xffffffffu, above, src);
    if (lane == 0) {
      S.prefix |= (uint32_t)found << shift;
      S.remaining = rem - above;
    }
  }
  __syncthreads();
}

// candidate i -> output id
__device__ __forceinline__ int32_t sel_id(int mode, int i, const int32_t* pool_row) {
  return mode == 0 ? i : __ldg(pool_row + i / kBlock) * kBlock + (i % kBlock);
}

// key of candidate i (0 past the end)
__device__ __forceinline__ uint32_t key_at(const float* sc, int i, int n) { return i < n ? score_key(sc[i]) : 0u; }

// visit every candidate: f(i, key) for i in [0, n), several loads in flight per thread
template <typename F>
__device__ __forceinline__ void for_keys(const float* sc, int n, F&& f) {
  constexpr int kU = 8;
  for (int base = 0; base < n; base += kSel2Threads * kU) {
    uint32_t k[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) k[u] = key_at(sc, base + u * kSel2Threads + threadIdx.x, n);
#pragma unroll
    for (int u = 0; u < kU; ++u) f(base + u * kSel2Threads + threadIdx.x, k[u]);
  }
}

// block-wide float min/max and int sum (all threads get the result)
struct MinMaxCount {
  float mn, mx;
  int cnt;
};

__device__ __forceinline__ MinMaxCount block_minmax_count(MinMaxCount v, float* smf, int* smi) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    v.mn = fminf(v.mn, __shfl_xor_sync(0xffffffffu, v.mn, o));
    v.mx = fmaxf(v.mx, __shfl_xor_sync(0xffffffffu, v.mx, o));
    v.cnt += __shfl_xor_sync(0xffffffffu, v.cnt, o);
  }
  __syncthreads();
  if (lane == 0) {
    smf[wid] = v.mn;
    smf[32 + wid] = v.mx;
    smi[wid] = v.cnt;
  }
  __syncthreads();
  MinMaxCount r{smf[0], smf[32], smi[0]};
  for (int w = 1; w < (int)(blockDim.x >> 5); ++w) {
    r.mn = fminf(r.mn, smf[w]);
    r.mx = fmaxf(r.mx, smf[32 + w]);
    r.cnt += smi[w];
  }
  return r;
}

constexpr int kLinBins = 4096;

struct SelShared2 {
  int hist[kLinBins];
  float redf[64];
  int redi[32];
  int wsum[32];
  int wsum2[32];
  uint32_t cand_key[kSelCand];
  int cand_n;
  int bstar, above;
  uint32_t prefix;
  int remaining;
};

// linear bin of a valid score within [mn, mx] (monotone non-decreasing in s)
__device__ __forceinline__ int lin_bin(float s, float mn, float scale) {
  int b = (int)__fmul_rn(__fsub_rn(s, mn), scale);
  return b < 0 ? 0 : (b >= kLinBins ? kLinBins - 1 : b);
}

// warp 0: the byte where the count from the top of hist[256] reaches *remaining;
// updates *prefix and *remaining (callers synchronise around it)
__device__ __forceinline__ void warp_pick_byte(const int* hist, uint32_t* prefix, int* remaining, int shift) {
  const int lane = threadIdx.x & 31;
  int c[8], tot = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    c[i] = hist[255 - (lane * 8 + i)];
    tot += c[i];
  }
  int incl = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  int before = incl - tot;
  const int rem = *remaining;
  int found = -1, above = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (found < 0 && before + c[i] >= rem) {
      found = 255 - (lane * 8 + i);
      above = before;
    }
    before += c[i];
  }
  const uint32_t mask = __ballot_sync(0xffffffffu, found >= 0);
  const int src = mask ? __ffs(mask) - 1 : 31;
  found = __shfl_sync(0xffffffffu, found, src);
  above = __shfl_sync(0xffffffffu, above, src);
  if (found < 0) found = 0;
  if (lane == 0) {
    *prefix |= (uint32_t)found << shift;
    *remaining = rem - above;
  }
}

// radix step over the shared candidates: fixes the byte at `shift` of the
// remaining-th largest key among candidates matching S.prefix above it
__device__ __forceinline__ void cand_radix_step(SelShared2& S, int nc, int shift) {
  for (int i = threadIdx.x; i < 256; i += kSel2Threads) S.hist[i] = 0;
  __syncthreads();
  const uint32_t hi_mask = shift >= 24 ? 0u : (0xFFFFFFFFu << (shift + 8));
  const uint32_t pre = S.prefix;
  for (int i = threadIdx.x; i < nc; i += kSel2Threads) {
    const uint32_t key = S.cand_key[i];
    if ((key & hi_mask) == (pre & hi_mask)) atomicAdd(&S.hist[(key >> shift) & 255u], 1);
  }
  __syncthreads();
  if (threadIdx.x < 32) warp_pick_byte(S.hist, &S.prefix, &S.remaining, shift);
  __syncthreads();
}

__global__ void __launch_bounds__(kSel2Threads, 1) k_select_topk2(csa2_query_batch qb, const float* __restrict__ score,
                                                               int64_t ld, int mode, const int32_t* __restrict__ pool,
                                                               const int32_t* __restrict__ pool_n, int P, int k_out,
                                                               int32_t* __restrict__ out, int32_t* __restrict__ out_n) {
  __shared__ SelShared2 S;
  const int tok = blockIdx.x;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int64_t p = __ldg(qb.tok_pos + tok);
  const int n = mode == 0 ? (int)((p + kBlock) / kBlock) : min(__ldg(pool_n + tok), P) * kBlock;
  const float* sc = score + (int64_t)tok * ld;
  const int32_t* pool_row = pool + (int64_t)tok * P;

  // pass A: range and count of the valid scores
  MinMaxCount v{INFINITY, -INFINITY, 0};
  for_keys(sc, n, [&](int i, uint32_t key) {
    if (key != 0u) {
      const float f = sc[i];
      v.mn = fminf(v.mn, f);
      v.mx = fmaxf(v.mx, f);
      v.cnt += 1;
    }
  });
  const MinMaxCount r = block_minmax_count(v, S.redf, S.redi);
  const int n_valid = r.cnt;
  const int k_eff = min(k_out, n_valid);
  const bool take_all = k_eff == n_valid;
  uint32_t T = 0;
  int need_eq = 0;
  if (!take_all && r.mx == r.mn) {
    T = score_key(r.mx);  // every valid score ties: the lowest ids win
    need_eq = k_eff;
  } else if (!take_all) {
    // pass B: linear histogram over [mn, mx]
    const float mn = r.mn, scale = (float)kLinBins / (r.mx - r.mn);
    for (int i = threadIdx.x; i < kLinBins; i += kSel2Threads) S.hist[i] = 0;
    __syncthreads();
    for_keys(sc, n, [&](int i, uint32_t key) {
      if (key != 0u) atomicAdd(&S.hist[lin_bin(sc[i], mn, scale)], 1);
    });
    __syncthreads();
    // threshold bin: suffix sums from the top, 4 bins per thread
    {
      constexpr int kPerT = kLinBins / kSel2Threads;
      const int hb = kLinBins - 1 - threadIdx.x * kPerT;  // this thread's highest bin
      int c[kPerT], tot = 0;
#pragma unroll
      for (int j = 0; j < kPerT; ++j) {
        c[j] = S.hist[hb - j];
        tot += c[j];
      }
      int total;
      const int before = block_exclusive_scan(tot, S.wsum, &total);
      int cum = before;
#pragma unroll
      for (int j = 0; j < kPerT; ++j) {
        if (cum < k_eff && cum + c[j] >= k_eff) {
          S.bstar = hb - j;
          S.above = cum;
        }
        cum += c[j];
      }
    }
    __syncthreads();
    const int bstar = S.bstar;
    // pass C: gather the keys of the threshold bin
    if (threadIdx.x == 0) S.cand_n = 0;
    __syncthreads();
    for_keys(sc, n, [&](int i, uint32_t key) {
      if (key != 0u && lin_bin(sc[i], mn, scale) == bstar) {
        const int slot = atomicAdd(&S.cand_n, 1);
        if (slot < kSelCand) S.cand_key[slot] = key;
      }
    });
    __syncthreads();
    const int nc = S.cand_n;
    if (threadIdx.x == 0) {
      S.prefix = 0;
      S.remaining = k_eff - S.above;
    }
    __syncthreads();
    if (nc <= kSelCand) {
      for (int shift = 24; shift >= 0; shift -= 8) cand_radix_step(S, nc, shift);
    } else {
      // more threshold-bin members than fit: resolve the bytes on global memory
      for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = threadIdx.x; i < 256; i += kSel2Threads) S.hist[i] = 0;
        __syncthreads();
        const uint32_t hi_mask = shift >= 24 ? 0u : (0xFFFFFFFFu << (shift + 8));
        const uint32_t pre = S.prefix;
        for_keys(sc, n, [&](int i, uint32_t key) {
          if (key != 0u && lin_bin(sc[i], mn, scale) == bstar && (key & hi_mask) == (pre & hi_mask))
            atomicAdd(&S.hist[(key >> shift) & 255u], 1);
        });
        __syncthreads();
        if (threadIdx.x < 32) warp_pick_byte(S.hist, &S.prefix, &S.remaining, shift);
        __syncthreads();
      }
    }
    T = S.prefix;
    need_eq = S.remaining;
  }
  // output: warp w owns ids [w*span, (w+1)*span)
  const int span = (n + 31) / 32;
  const int lo = min(n, wid * span), hi = min(n, lo + span);
  int gt = 0, eq = 0;
  for (int b0 = lo; b0 < hi; b0 += 32 * 8) {
    uint32_t k8[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) k8[u] = key_at(sc, b0 + u * 32 + lane, hi);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const uint32_t key = k8[u];
      const bool g = key != 0u && (take_all || key > T);
      const bool e = !take_all && key != 0u && key == T;
      gt += __popc(__ballot_sync(0xffffffffu, g));
      eq += __popc(__ballot_sync(0xffffffffu, e));
    }
  }
  if (lane == 0) {
    S.wsum[wid] = gt;
    S.wsum2[wid] = eq;
  }
  __syncthreads();
  // exclusive prefix over the 32 warps (each lane of a warp reads one warp's sum)
  int eq_before = __shfl_sync(0xffffffffu, 0, 0);
  {
    const int v = lane < wid ? S.wsum2[lane] : 0;
    eq_before = __reduce_add_sync(0xffffffffu, v);
  }
  const int take_eq = max(0, min(eq, need_eq - eq_before));
  __syncthreads();
  if (lane == 0) S.wsum2[wid] = take_eq;
  __syncthreads();
  int out_before;
  {
    const int v = lane < wid ? S.wsum[lane] + S.wsum2[lane] : 0;
    out_before = __reduce_add_sync(0xffffffffu, v);
  }
  int32_t* o = out + (int64_t)tok * k_out;
  int written = out_before, eq_taken = 0;
  for (int b0 = lo; b0 < hi; b0 += 32 * 8) {
    uint32_t k8[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) k8[u] = key_at(sc, b0 + u * 32 + lane, hi);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = b0 + u * 32 + lane;
      const uint32_t key = k8[u];
      const bool g = key != 0u && (take_all || key > T);
      const bool e = !take_all && key != 0u && key == T;
      const uint32_t em = __ballot_sync(0xffffffffu, e);
      const int e_rank = __popc(em & ((1u << lane) - 1u));
      const bool sel = g || (e && eq_taken + e_rank < take_eq);
      const uint32_t sm = __ballot_sync(0xffffffffu, sel);
      if (sel) o[written + __popc(sm & ((1u << lane) - 1u))] = sel_id(mode, i, pool_row);
      written += __popc(sm);
      eq_taken = min(take_eq, eq_taken + __popc(em));
    }
  }
  __syncthreads();
  for (int j = k_eff + threadIdx.x; j < k_out; j += kSel2Threads) o[j] = -1;
  if (threadIdx.x == 0) out_n[tok] = k_eff;
}

}  // namespace csa2
