// select.cuh -- top-k selection without a global sort (block top-P pool and
// pool top-K positions).  One CTA of 1024 threads per query token.
//
//   keys      order-preserving unsigned images of the fp32 scores (score_key);
//             invalid candidates map to 0 and are never selected
//   passes 1-2  256-bin histograms of the top two key bytes (shared-memory
//             atomics aggregated per warp with __match_any_sync), each fixing
//             one byte of the k-th largest key;
//   pass 3    candidates that share those 16 bits are gathered into shared
//             memory (few in practice) and the last two bytes are resolved
//             there; if they do not fit, two more global passes resolve them;
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

__global__ void __launch_bounds__(kSel2Threads) k_select_topk2(csa2_query_batch qb, const float* __restrict__ score,
                                                               int64_t ld, int mode, const int32_t* __restrict__ pool,
                                                               const int32_t* __restrict__ pool_n, int P, int k_out,
                                                               int32_t* __restrict__ out, int32_t* __restrict__ out_n) {
  __shared__ SelShared S;
  const int tok = blockIdx.x;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int64_t p = __ldg(qb.tok_pos + tok);
  const int n = mode == 0 ? (int)((p + kBlock) / kBlock) : min(__ldg(pool_n + tok), P) * kBlock;
  const float* sc = score + (int64_t)tok * ld;
  const int32_t* pool_row = pool + (int64_t)tok * P;

  for (int i = threadIdx.x; i < 256; i += kSel2Threads) S.hist[i] = 0;
  if (threadIdx.x == 0) {
    S.prefix = 0;
    S.cand_n = 0;
    S.n_valid = 0;
  }
  __syncthreads();
  // pass 1: top byte, and the number of valid candidates
  int nv = 0;
  for_keys(sc, n, [&](int, uint32_t key) {
    nv += key != 0u;
    hist_add(S.hist, key >> 24, key != 0u);
  });
  nv = __reduce_add_sync(0xffffffffu, nv);
  if (lane == 0) atomicAdd(&S.n_valid, nv);
  __syncthreads();
  const int n_valid = S.n_valid;
  const int k_eff = min(k_out, n_valid);
  const bool take_all = k_eff == n_valid;
  uint32_t T = 0;
  int need_eq = 0;
  if (!take_all) {
    if (threadIdx.x == 0) S.remaining = k_eff;
    pick_digit(S, 24);
    // pass 2: second byte among keys with the chosen top byte
    for (int i = threadIdx.x; i < 256; i += kSel2Threads) S.hist[i] = 0;
    __syncthreads();
    const uint32_t p1 = S.prefix;
    for_keys(sc, n, [&](int, uint32_t key) {
      hist_add(S.hist, (key >> 16) & 255u, key != 0u && (key >> 24) == (p1 >> 24));
    });
    pick_digit(S, 16);
    const uint32_t p2 = S.prefix;
    // pass 3: gather the keys sharing the 16-bit prefix
    for_keys(sc, n, [&](int, uint32_t key) {
      if (key != 0u && (key >> 16) == (p2 >> 16)) {
        const int slot = atomicAdd(&S.cand_n, 1);
        if (slot < kSelCand) S.cand_key[slot] = key;
      }
    });
    __syncthreads();
    const int nc = S.cand_n;
    for (int shift = 8; shift >= 0; shift -= 8) {
      for (int i = threadIdx.x; i < 256; i += kSel2Threads) S.hist[i] = 0;
      __syncthreads();
      const uint32_t pre = S.prefix;
      const uint32_t hi_mask = 0xFFFFFFFFu << (shift + 8);
      if (nc <= kSelCand) {
        for (int base = 0; base < nc; base += kSel2Threads) {
          const int i = base + threadIdx.x;
          const uint32_t key = i < nc ? S.cand_key[i] : 0u;
          hist_add(S.hist, (key >> shift) & 255u, i < nc && (key & hi_mask) == (pre & hi_mask));
        }
      } else {
        for_keys(sc, n, [&](int, uint32_t key) {
          hist_add(S.hist, (key >> shift) & 255u, key != 0u && (key & hi_mask) == (pre & hi_mask));
        });
      }
      pick_digit(S, shift);
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
  int eq_before = 0, out_before = 0;
  for (int w = 0; w < wid; ++w) eq_before += S.wsum2[w];
  const int take_eq = max(0, min(eq, need_eq - eq_before));
  __syncthreads();
  if (lane == 0) S.wsum2[wid] = take_eq;
  __syncthreads();
  for (int w = 0; w < wid; ++w) out_before += S.wsum[w] + S.wsum2[w];
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
