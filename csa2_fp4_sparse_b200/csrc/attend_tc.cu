// attend_tc.cu -- sparse MQA attention (Reuse mode) on the 5th-generation
// tensor cores, with the optional FP8 sliding-window rows in the same softmax.
//
// For query token i and head h (DeepSeek-V4.1-Flash pages, dbyun.net article
// 10794, section "KV Cache 成为这一代架构改造的核心": a Reuse layer reuses the index
// list and only runs attention; the SWA KV stays FP8, and the window is the
// last 128 tokens, prism.simon-ai.net article 7901, SWA section):
//   z_t = scale * q_h . k~_t   over the selected FP4 Main-KV rows (V = K latent)
//         and, when given, the window rows e4m3(c_t) * s_t
//   o_h = sum_t softmax(z)_t * v_t      (one softmax over both sets)
//
// One CTA per (split, query token, layer) walks its 64-row chunks of the key
// set through a warp-specialised pipeline with two shared-memory K/V tiles:
//   warps 4..11  loaders: gather the chunk's rows (codes of the next chunk are
//                already in flight while the current one is converted) and
//                dequantise them exactly to fp16 (E2M1 x E4M3 products, or
//                E4M3 window codes) into a 128B-swizzled tile
//                [64-element d-block][row][128 B];
//   warps 12,14  issue S = Q K^T on tcgen05 (kind::f16, M = 64 heads, N = 64
//                rows, K = D) into one of two TMEM score buffers, each warp
//                half of the d-blocks into its own accumulator (the softmax
//                adds the two; an MMA costs its issuing thread ~110 cycles);
//   warps 0..3   softmax, two threads per head (M = 64 keeps head h in TMEM
//                lane 32*(h/16) + h%16; the 16x32bx2 load gives lanes t and
//                t+16 of a warp the two halves of head t's scores): one pass
//                per chunk against the running (log2) max, which only moves
//                (with a second pass) when a chunk exceeds it by more than
//                2^15 (then the output accumulator is rescaled); P = 2^(z - m)
//                written as fp16 rows [head][row] (window rows carry their
//                per-token scale into P);
//   warps 13,15  issue O^T += V^T P^T (M = 128 latent dims per tile, N =
//                heads, K = 64 rows; half of the latent-dim tiles each)
//                reading the same tile as V; their commits free the tile and
//                the P buffer.
// The epilogue divides by the row sum, stages the output in shared memory and
// writes it with bulk copies (4-byte stores when the destination is not 16-byte
// aligned), or the split's unnormalised partial with its max and sum (the last
// split of a token merges them).  Every wait is bounded.
#include "internal.h"
#include "tc_common.cuh"

namespace csa2 {
namespace attend_tc {

constexpr int kRows = 64;       // rows per chunk (MMA N of S, K of PV)
constexpr int kMq = 64;         // MMA M of S: heads, padded to 64
constexpr int kSoftWarps = 4;   // warps 0..3
constexpr int kLoadWarps = 8;   // warps 4..11
constexpr int kWarpS = 12;      // S issuers: warps 12 and 14 take the two halves of the d-blocks of every
                                // chunk (a tcgen05.mma costs its issuing thread ~110 cycles)
constexpr int kWarpS2 = 14;
constexpr int kWarpPV = 13;     // PV issuers: warps 13 and 15 take the two halves of the latent-dim tiles
constexpr int kWarpPV2 = 15;
constexpr int kThreads = 512;
constexpr int kLoadThreads = kLoadWarps * 32;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 15.0f;  // P = 2^(z - m) stays <= 2^15 between rescales (fp16 holds it)

constexpr int kMaxLayers = 32;  // layers attended in one launch (grid.z), each with its own index list
constexpr int kMaxRows = 2048;  // K: selected rows per query token

struct LayerIO {
  const int32_t* idx;    // [T][K] selected Main KV positions of this layer's selector
  const int32_t* idx_n;  // [T]
  const void* q;
  void* out;
  float* lse;
  const uint8_t* swa_codes;
  const float* swa_scale;
};

struct Params {
  csa2_query_batch qb;
  int q_f32;
  csa2_fp4_cache kv;
  int K;
  int has_swa, swa_cap, swa_window;
  float scale;
  int out_f32;
  LayerIO io[kMaxLayers];
  float* part_o;   // split mode: [layers][T][S][Hq][D]
  float* part_ml;  // split mode: [layers][T][S][Hq][2] (natural-log max, sum)
  int* done;       // split mode: [layers][T] arrival counters, zero on entry, left zero on exit
  int* status;
  uint64_t wait_ns;
};

template <int D, int HQ, bool QLO, bool PLO>
struct Layout {
  static constexpr int kKB = D / 64;                    // 64-element d-blocks
  static constexpr int kMT = D / 128;                   // PV M tiles
  static constexpr int kUnitsRow = D / 32;              // 32-element units per row
  static constexpr int kPer = kRows * kUnitsRow / kLoadThreads;  // units per loader thread per chunk
  static constexpr uint32_t kTile = kRows * D * 2;      // fp16 K/V tile
  // Q [kb][HQ][128 B]; the S MMA reads kMq rows per d-block, so the last
  // d-block's rows past HQ land in a pad inside the region
  static constexpr uint32_t kQBytes = HQ * D * 2 + (kMq - HQ) * 128;
  static constexpr uint32_t kPBytes = HQ * kRows * 2;   // P [head][row] fp16
  static constexpr uint32_t kOffTile = 0;               // [2][kTile]
  static constexpr uint32_t kOffQ = kOffTile + 2 * kTile;
  static constexpr uint32_t kOffQlo = kOffQ + (kQBytes + 1023) / 1024 * 1024;
  static constexpr uint32_t kOffP = kOffQlo + (QLO ? (kQBytes + 1023) / 1024 * 1024 : 0);  // [2][kPBytes]
  // fp32 outputs: the low fp16 part of P (one buffer; see the softmax)
  static constexpr uint32_t kOffPlo = kOffP + 2 * ((kPBytes + 1023) / 1024 * 1024);
  static constexpr uint32_t kOffRows = kOffPlo + (PLO ? (kPBytes + 1023) / 1024 * 1024 : 0);  // [kMaxRows] i32 cache rows
  static constexpr uint32_t kOffRs = kOffRows + kMaxRows * 4;                              // [2][kRows] f32
  static constexpr uint32_t kOffCorr = kOffRs + 2 * kRows * 4;  // [kMq] f32
  static constexpr uint32_t kOffL = kOffCorr + kMq * 4;         // [kMq] f32 final row sums
  static constexpr uint32_t kOffM = kOffL + kMq * 4;            // [kMq] f32 final maxima (log2)
  static constexpr uint32_t kOffBar = kOffM + kMq * 4;          // 9 mbarriers
  static constexpr uint32_t kOffMisc = kOffBar + 9 * 8;         // tmem base, abort, last-split flag
  static constexpr uint32_t kBytes = kOffMisc + 16 + 1024;
  static constexpr uint32_t kColS = 0;    // score buffer b, d-block half c at kColS + c * 2 * kRows + b * kRows
  static constexpr int kPvIss = kMT >= 2 ? 2 : 1;  // PV issuing warps with work
  static constexpr uint32_t kColO = 256;  // O^T tile mt at kColO + mt * HQ
  static_assert(kPer >= 1 && kRows * kUnitsRow % kLoadThreads == 0, "loader unit split");
  static_assert(kMT * HQ <= 256 && 2 * kRows <= 256, "TMEM budget");
  static_assert((uint32_t)HQ * D * 4 <= 2 * kTile, "epilogue staging fits in the tiles");
};

// swizzled byte offset of 16-byte chunk c of row r for 128-byte rows
__device__ __forceinline__ uint32_t swz128(uint32_t r, uint32_t c) { return r * 128 + ((c ^ (r & 7)) << 4); }

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// 2^x on the special-function unit (PTX ex2.approx.ftz: relative error below
// 2^-22; -inf -> +0)
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// named barrier over the softmax warps with an OR over `pred`
__device__ __forceinline__ bool soft_sync_or(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "barrier.red.or.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred)
      : "memory");
  return r != 0;
}

// one loader thread's share of a chunk: kPer units of 32 elements
template <int kPer>
struct Pref {
  uint4 c[kPer];     // FP4 codes (16 B), or the first 16 of a window unit's 32 FP8 codes
  uint32_t s[kPer];  // E4M3 scale byte of an FP4 unit
  float rs[kPer];    // softmax row scale (units starting a row): 1 sparse, s_t window, -1 no row
  int32_t wrow[kPer];  // window unit: its row (the second 16 bytes are read at conversion)
};

template <int D, int HQ, bool QLO, bool PLO>
__global__ void __launch_bounds__(kThreads, 1) k_attend_tc(const __grid_constant__ Params P) {
  using Ly = Layout<D, HQ, QLO, PLO>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar_kv_full = sbase + Ly::kOffBar;       // [2] loaders -> S issuer (count kLoadWarps)
  const uint32_t bar_kv_empty = bar_kv_full + 16;         // [2] PV commit -> loaders, softmax rescale, epilogue
  const uint32_t bar_s_full = bar_kv_empty + 16;          // [2] S commit -> softmax
  const uint32_t bar_p_full = bar_s_full + 16;            // [2] softmax -> PV issuer (count kSoftWarps)
  const uint32_t bar_drain = bar_p_full + 16;             // issuers' final commits (count 2)
  volatile uint32_t* tmem_holder = reinterpret_cast<volatile uint32_t*>(smem + Ly::kOffMisc);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + Ly::kOffMisc + 4);
  float* rs_s = reinterpret_cast<float*>(smem + Ly::kOffRs);
  float* corr_s = reinterpret_cast<float*>(smem + Ly::kOffCorr);
  float* l_s = reinterpret_cast<float*>(smem + Ly::kOffL);
  float* m_s = reinterpret_cast<float*>(smem + Ly::kOffM);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tok = blockIdx.y, split = blockIdx.x, nsplit = gridDim.x, layer = blockIdx.z;
  const LayerIO& io = P.io[layer];  // read from parameter space where used
  const int64_t slot0 = ((int64_t)layer * P.qb.n_tok + tok) * nsplit;  // this token's partial slots

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_kv_full + 8 * i, kLoadWarps);
      mbar_init(bar_kv_empty + 8 * i, Ly::kPvIss);
      mbar_init(bar_s_full + 8 * i, 2);
      mbar_init(bar_p_full + 8 * i, kSoftWarps);
    }
    mbar_init(bar_drain, 2 + Ly::kPvIss);  // every issuing warp
    *abort = 0;
    tc::fence_barrier_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(sbase + Ly::kOffMisc, 512);
    tc::tmem_relinquish();
    tc::fence_before_sync();
  }
  grid_dep_wait();  // the previous kernel's index lists
  const int b = __ldg(P.qb.tok_seq + tok);
  const int64_t p = __ldg(P.qb.tok_pos + tok);
  // this CTA's chunks: c = split + nsplit * i (sparse chunks first, then window chunks)
  const int n_sel = min(__ldg(io.idx_n + tok), P.K);
  const int n_sp = (n_sel + kRows - 1) / kRows;
  int64_t w_lo = 0;
  int n_w = 0;
  if (P.has_swa) {
    w_lo = p - P.swa_window + 1;
    if (w_lo < 0) w_lo = 0;
    n_w = (int)(p - w_lo + 1);
  }
  const int n_chunks = n_sp + (n_w + kRows - 1) / kRows;
  const int n_mine = split < n_chunks ? (n_chunks - split + nsplit - 1) / nsplit : 0;
  const int n_mine_sp = split < n_sp ? (n_sp - split + nsplit - 1) / nsplit : 0;
  int32_t* rows_s = reinterpret_cast<int32_t*>(smem + Ly::kOffRows);
  // the cache rows of this CTA's sparse chunks (index list, then page table),
  // every load of a stage in flight together
  constexpr int kRowPer = (kMaxRows + kThreads - 1) / kThreads;
  int32_t tv[kRowPer];
#pragma unroll
  for (int u = 0; u < kRowPer; ++u) {
    const int e = threadIdx.x + u * kThreads;
    tv[u] = -2;  // no entry
    if (e < n_mine_sp * kRows) {
      const int j = (split + (e / kRows) * nsplit) * kRows + e % kRows;
      tv[u] = j < n_sel ? __ldg(io.idx + (int64_t)tok * P.K + j) : -2;
    }
  }
  // cache rows: index -> page -> row (the page loads wait for the index loads)
  int64_t pg[kRowPer];
  auto load_pages = [&]() {
#pragma unroll
    for (int u = 0; u < kRowPer; ++u) {
      const int32_t t = tv[u];
      pg[u] = 0;
      if (t >= 0 && t <= p)
        pg[u] = P.kv.page_table ? (int64_t)__ldg(P.kv.page_table + (int64_t)b * P.kv.max_pages +
                                                 (uint32_t)t / (uint32_t)P.kv.page_size)
                                : __ldg(P.kv.seq_base + b);
    }
  };
  // query -> fp16 [kb][h][128 B] (K-major, 128B swizzle); f32 queries also
  // keep the fp16 residual.  All threads, all loads in flight together.
  {
    constexpr int kUnitsQ = HQ * D / 8;  // 8 consecutive d per unit
    constexpr int kQPer = (kUnitsQ + kThreads - 1) / kThreads;
    // units in flight per batch: every unit of a bf16 query, three of an f32 one
    constexpr int kQB = QLO ? (kQPer < 3 ? kQPer : 3) : kQPer;
#pragma unroll 1
    for (int u0 = 0; u0 < kQPer; u0 += kQB) {
    // raw query units: 8 bf16 (one uint4) or, with f32 queries (QLO), 8 f32
    uint4 raw[kQB][QLO ? 2 : 1];
#pragma unroll
    for (int u = 0; u < kQB; ++u) {
      const int e = (u0 + u) * kThreads + threadIdx.x;
      if (e >= kUnitsQ) continue;
      const int h = e / (D / 8), c8 = e % (D / 8);
      const int64_t off = ((int64_t)tok * HQ + h) * D + c8 * 8;
      if constexpr (QLO) {
        const uint4* s4 = reinterpret_cast<const uint4*>(reinterpret_cast<const float*>(io.q) + off);
        raw[u][0] = __ldg(s4);
        raw[u][QLO ? 1 : 0] = __ldg(s4 + 1);
      } else {
        raw[u][0] = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(io.q) + off));
      }
    }
    // the page-table loads go out while the first query batch is in flight
    if (u0 == 0) load_pages();
#pragma unroll
    for (int u = 0; u < kQB; ++u) {
      const int e = (u0 + u) * kThreads + threadIdx.x;
      if (e >= kUnitsQ) continue;
      const int h = e / (D / 8), c8 = e % (D / 8);
      const int kb = c8 / 8, c = c8 % 8;
      float f[8];
      if constexpr (QLO) {
        const uint32_t ww[8] = {raw[u][0].x, raw[u][0].y, raw[u][0].z, raw[u][0].w,
                                raw[u][QLO ? 1 : 0].x, raw[u][QLO ? 1 : 0].y, raw[u][QLO ? 1 : 0].z,
                                raw[u][QLO ? 1 : 0].w};
#pragma unroll
        for (int k = 0; k < 8; ++k) f[k] = __uint_as_float(ww[k]);
      } else {
        const uint32_t ww[4] = {raw[u][0].x, raw[u][0].y, raw[u][0].z, raw[u][0].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          f[2 * k] = __uint_as_float(ww[k] << 16);
          f[2 * k + 1] = __uint_as_float(ww[k] & 0xFFFF0000u);
        }
      }
      uint4 hi, lo;
      uint32_t* hp = &hi.x;
      uint32_t* lp = &lo.x;
      // the MMAs take the query in fp16: a value at or beyond 65520 (or a NaN)
      // has no fp16 form; it is reported and the result is not meaningful
      bool out_of_range = false;
#pragma unroll
      for (int k = 0; k < 8; ++k) out_of_range |= !(fabsf(f[k]) < 65520.0f);
      if (out_of_range) set_status(P.status, CSA2_ERR_RANGE);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        __half2 h2 = __floats2half2_rn(f[2 * k], f[2 * k + 1]);
        hp[k] = *reinterpret_cast<uint32_t*>(&h2);
        const float2 back = __half22float2(h2);
        lp[k] = pack_half2(f[2 * k] - back.x, f[2 * k + 1] - back.y);
      }
      const uint32_t o = kb * (HQ * 128) + swz128(h, c);
      *reinterpret_cast<uint4*>(smem + Ly::kOffQ + o) = hi;
      if (QLO) *reinterpret_cast<uint4*>(smem + Ly::kOffQlo + o) = lo;
    }
    }
  }
  {
#pragma unroll
    for (int u = 0; u < kRowPer; ++u) {
      const int e = threadIdx.x + u * kThreads;
      const int32_t t = tv[u];
      if (t == -2) {
        if (e < n_mine_sp * kRows) rows_s[e] = -1;
        continue;
      }
      int64_t row = -1;
      if (t >= 0 && t <= p) {
        row = P.kv.page_table ? pg[u] * P.kv.page_size + (int64_t)((uint32_t)t % (uint32_t)P.kv.page_size)
                              : pg[u] + t;
        if (row < 0 || row >= P.kv.n_rows) row = -1;
      }
      if (row < 0) set_status(P.status, CSA2_ERR_RANGE);
      rows_s[e] = (int32_t)row;
    }
  }
  tc::fence_proxy_async_smem();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_holder;

  if (warp >= kSoftWarps && warp < kSoftWarps + kLoadWarps) {
    // ------------------------------------------------------------ loaders
    const int lt = threadIdx.x - kSoftWarps * 32;  // 0..255
    Pref<Ly::kPer> cur, nxt;
    // codes (and, for units that start a row, the softmax row scale) of local chunk i
    auto load_codes = [&](int i, Pref<Ly::kPer>& pf) {
      const int c = split + i * nsplit;
      const bool sparse = c < n_sp;
#pragma unroll
      for (int k = 0; k < Ly::kPer; ++k) {
        const int u = lt + k * kLoadThreads;
        const int r = u / Ly::kUnitsRow, g = u % Ly::kUnitsRow;
        int64_t row = -1;
        if (sparse) {
          row = rows_s[i * kRows + r];
        } else {
          const int64_t t = w_lo + (int64_t)(c - n_sp) * kRows + r;
          // 0 <= t < max_seq_len: an unsigned 32-bit remainder (a 64-bit one
          // costs the loader a long instruction sequence per unit)
          if (t <= p) row = (int64_t)b * P.swa_cap + (int64_t)((uint32_t)t % (uint32_t)P.swa_cap);
        }
        pf.c[k] = make_uint4(0, 0, 0, 0);
        pf.s[k] = 0;
        pf.rs[k] = -1.0f;
        pf.wrow[k] = (int32_t)row;
        if (row < 0) continue;
        if (sparse) {
          pf.c[k] = __ldg(reinterpret_cast<const uint4*>(P.kv.codes + row * (D / 2)) + g);
          pf.s[k] = __ldg(P.kv.scales + row * (D / 32) + g);
          pf.rs[k] = 1.0f;
        } else {
          pf.c[k] = __ldg(reinterpret_cast<const uint4*>(io.swa_codes + row * D) + 2 * g);
          if (g == 0) pf.rs[k] = __ldg(io.swa_scale + row);
        }
      }
    };
    if (n_mine > 0) load_codes(0, cur);
    bool dead = false;  // uniform over the loader warps: a wait gave up
    for (int i = 0; i < n_mine; ++i) {
      const int c = split + i * nsplit, bf = i & 1;
      // the next chunk's codes go in flight before this chunk is converted
      if (i + 1 < n_mine) load_codes(i + 1, nxt);
      // the tile is free once PV(i - 2) has completed: one loader thread
      // probes, the others park on named barrier 2
      if (i >= 2 && !dead) {
        if (!mbar_wait_group(bar_kv_empty + 8 * bf, ((i >> 1) - 1) & 1, P.wait_ns, lt == 0, *abort != 0, 2,
                             kLoadThreads)) {
          if (lt == 0) {
            set_status(P.status, CSA2_ERR_TIMEOUT);
            *abort = 1;
          }
          dead = true;
        }
      }
      if (!dead) {
        uint8_t* tile = smem + Ly::kOffTile + bf * Ly::kTile;
        const bool sparse = c < n_sp;
#pragma unroll
        for (int k = 0; k < Ly::kPer; ++k) {
          const int u = lt + k * kLoadThreads;
          const int r = u / Ly::kUnitsRow, g = u % Ly::kUnitsRow;
          // 32 values = d in [32g, 32g+32): d-block g/2, 16-byte chunks (g%2)*4 .. +4
          const int kb = g / 2, c0 = (g % 2) * 4;
          uint32_t outw[16];
          if (sparse) {
            const __half sh = __float2half_rn(e4m3_to_f32(cur.s[k]));
            const __half2 s2 = __halves2half2(sh, sh);
            const uint32_t words[4] = {cur.c[k].x, cur.c[k].y, cur.c[k].z, cur.c[k].w};
#pragma unroll
            for (int w = 0; w < 4; ++w)
#pragma unroll
              for (int bb = 0; bb < 4; ++bb) {
                uint32_t h2 = tc::e2m1x2_to_f16x2((words[w] >> (8 * bb)) & 0xFFu);
                __half2 v = __hmul2(*reinterpret_cast<__half2*>(&h2), s2);
                outw[w * 4 + bb] = *reinterpret_cast<uint32_t*>(&v);
              }
          } else {
            const uint4 c1 = cur.wrow[k] >= 0
                                 ? __ldg(reinterpret_cast<const uint4*>(io.swa_codes + (int64_t)cur.wrow[k] * D) + 2 * g + 1)
                                 : make_uint4(0, 0, 0, 0);
            const uint32_t words[8] = {cur.c[k].x, cur.c[k].y, cur.c[k].z, cur.c[k].w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
            for (int w = 0; w < 8; ++w) {
              outw[2 * w] = tc::e4m3x2_to_f16x2(words[w] & 0xFFFFu);
              outw[2 * w + 1] = tc::e4m3x2_to_f16x2(words[w] >> 16);
            }
          }
#pragma unroll
          for (int w = 0; w < 4; ++w)
            *reinterpret_cast<uint4*>(tile + kb * (kRows * 128) + swz128(r, c0 + w)) =
                make_uint4(outw[4 * w], outw[4 * w + 1], outw[4 * w + 2], outw[4 * w + 3]);
          if (g == 0) rs_s[bf * kRows + r] = cur.rs[k];  // one thread per row
        }
        tc::fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar_kv_full + 8 * bf);
      cur = nxt;
    }
  } else if (warp == kWarpS || warp == kWarpS2) {
    // ------------------------------------------------------------ S = Q K^T
    const uint32_t idesc = tc::idesc_f16(kMq, kRows, 0, 0);
    const int half = warp == kWarpS ? 0 : 1;  // d-blocks [half * kKB/2, (half + 1) * kKB/2)
    for (int i = 0; i < n_mine; ++i) {
      const int bf = i & 1;
      if (lane == 0 && !*abort) {
        if (!mbar_wait_bounded(bar_kv_full + 8 * bf, (i >> 1) & 1, P.wait_ns)) {
          set_status(P.status, CSA2_ERR_TIMEOUT);
          *abort = 1;
        } else {
          tc::fence_after_sync();
          // descriptors advance by adding (byte offset >> 4) to the start
          // address field (shared addresses stay below 2^18: no carry out)
          const uint64_t a0 = tc::smem_desc(sbase + Ly::kOffQ, 16, 1024, tc::kSwizzle128B);
          const uint64_t al0 = tc::smem_desc(sbase + Ly::kOffQlo, 16, 1024, tc::kSwizzle128B);
          const uint64_t b0 = tc::smem_desc(sbase + Ly::kOffTile + bf * Ly::kTile, 16, 1024, tc::kSwizzle128B);
          const uint32_t dcol = tmem + Ly::kColS + half * 2 * kRows + bf * kRows;
          constexpr int kHalf = Ly::kKB / 2;
#pragma unroll
          for (int k2 = 0; k2 < kHalf; ++k2)
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              const int kb = half * kHalf + k2;
              const uint64_t ao = (uint64_t)((kb * (HQ * 128) + ks * 32) >> 4);
              const uint64_t bd = b0 + (uint64_t)((kb * (kRows * 128) + ks * 32) >> 4);
              tc::mma_f16(dcol, a0 + ao, bd, idesc, (k2 | ks) ? 1u : 0u);
              if (QLO) tc::mma_f16(dcol, al0 + ao, bd, idesc, 1u);
            }
          tc::commit(bar_s_full + 8 * bf);
        }
      }
      __syncwarp();
    }
    if (lane == 0) tc::commit(bar_drain);
    __syncwarp();
  } else if (warp == kWarpPV || warp == kWarpPV2) {
    // ------------------------------------------------------------ O^T += V^T P^T
    const uint32_t idesc = tc::idesc_f16(128, HQ, 1, 0);
    const int ph = warp == kWarpPV ? 0 : 1;  // latent-dim tiles [ph * kMT/2, (ph + 1) * kMT/2)
    const int mt0 = Ly::kPvIss == 2 ? ph * (Ly::kMT / 2) : 0;
    const int mt1 = Ly::kPvIss == 2 ? mt0 + Ly::kMT / 2 : (ph == 0 ? Ly::kMT : 0);
    for (int i = 0; i < (mt1 > mt0 ? n_mine : 0); ++i) {
      const int bf = i & 1;
      if (lane == 0 && !*abort) {
        if (!mbar_wait_bounded(bar_p_full + 8 * bf, (i >> 1) & 1, P.wait_ns)) {
          set_status(P.status, CSA2_ERR_TIMEOUT);
          *abort = 1;
        } else {
          tc::fence_after_sync();
          const uint64_t a0 =
              tc::smem_desc(sbase + Ly::kOffTile + bf * Ly::kTile, kRows * 128, 1024, tc::kSwizzle128B);
          const uint64_t b0 =
              tc::smem_desc(sbase + Ly::kOffP + bf * ((Ly::kPBytes + 1023) / 1024 * 1024), 16, 1024, tc::kSwizzle128B);
          const uint64_t bl0 = tc::smem_desc(sbase + Ly::kOffPlo, 16, 1024, tc::kSwizzle128B);
#pragma unroll 1
          for (int mt = mt0; mt < mt1; ++mt)
#pragma unroll
            for (int ks = 0; ks < kRows / 16; ++ks) {
              const uint64_t ad = a0 + (uint64_t)(((2 * mt) * (kRows * 128) + ks * 2048) >> 4);
              const uint64_t bd = b0 + (uint64_t)((ks * 32) >> 4);
              tc::mma_f16(tmem + Ly::kColO + mt * HQ, ad, bd, idesc, (i > 0 || ks > 0) ? 1u : 0u);
              if (PLO) tc::mma_f16(tmem + Ly::kColO + mt * HQ, ad, bl0 + (uint64_t)((ks * 32) >> 4), idesc, 1u);
            }
          tc::commit(bar_kv_empty + 8 * bf);
        }
      }
      __syncwarp();
    }
    if (lane == 0 && mt1 > mt0) tc::commit(bar_drain);
    __syncwarp();
  } else if (warp < kSoftWarps) {
    // ------------------------------------------------------------ softmax
    // head h = 16 * warp + (lane & 15); lane half `hf` takes rows [32 hf, 32 hf + 32)
    // of each chunk (the 16x32bx2 TMEM load hands them over)
    const int hf = lane >> 4;
    const int h = 16 * warp + (lane & 15);
    const bool act = h < HQ;
    const uint32_t s_lane = tmem + ((uint32_t)(warp * 32) << 16);
    const float zs = P.scale * kLog2e;
    float m = -INFINITY, l = 0.0f;  // l: this half's rows
    bool dead = false;              // uniform over the softmax warps: a wait gave up
    for (int i = 0; i < n_mine; ++i) {
      const int bf = i & 1;
      // one thread probes, the other softmax threads park on named barrier 1
      const bool ok = !dead && mbar_wait_group(bar_s_full + 8 * bf, (i >> 1) & 1, P.wait_ns, threadIdx.x == 0,
                                               *abort != 0, 1, 128);
      if (!ok && !dead) {
        if (threadIdx.x == 0 && !*abort) {
          set_status(P.status, CSA2_ERR_TIMEOUT);
          *abort = 1;
        }
        dead = true;
      }
      tc::fence_after_sync();
      const float* rsb = rs_s + bf * kRows + 32 * hf;  // this half's rows
      const uint32_t s_col = s_lane + Ly::kColS + bf * kRows;
      // every row a valid sparse row (row scale 1): the common case, no per-row scale
      const bool plain = __all_sync(0xffffffffu, rs_s[bf * kRows + lane] == 1.0f && rs_s[bf * kRows + lane + 32] == 1.0f);
      // P = 2^(z - mu) as fp16 [head][row] for this half's 32 rows, their sum,
      // and the largest z seen; window rows carry s_t into P.  The TMEM loads
      // are warp-collective: every lane issues them (ok is uniform), only the
      // lanes that carry a head write P.
      uint8_t* prow = smem + Ly::kOffP + bf * ((Ly::kPBytes + 1023) / 1024 * 1024);
      uint8_t* plow = smem + Ly::kOffPlo;
      // fp32 outputs: P is written as two fp16 parts, hi = fp16(e) and
      // lo = fp16(e - hi), and PV runs over both (relative error of the
      // weights ~2^-22 instead of the 2^-12 of one fp16), while the sum adds
      // the fp32 weights.  The one lo buffer is free once PV(i - 1) is done.
      if (PLO && i > 0 && ok) {
        if (!mbar_wait_group(bar_kv_empty + 8 * ((i - 1) & 1), ((i - 1) >> 1) & 1, P.wait_ns, threadIdx.x == 0,
                             *abort != 0, 1, 128)) {
          if (threadIdx.x == 0 && !*abort) {
            set_status(P.status, CSA2_ERR_TIMEOUT);
            *abort = 1;
          }
        }
      }
      auto p_pass = [&](float mu_, float& sum_, float& zmax_) {
        const float nmu = mu_ == -INFINITY ? 0.0f : -mu_;
        sum_ = 0.0f;
        zmax_ = -INFINITY;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          uint32_t v[8], v2[8];  // the two d-block halves of S
          tc::ld_16x32bx2_x8<32>(s_col + g * 8, v);
          tc::ld_16x32bx2_x8<32>(s_col + 2 * kRows + g * 8, v2);
          tc::ld_wait();
#pragma unroll
          for (int k = 0; k < 8; ++k) v[k] = __float_as_uint(__uint_as_float(v[k]) + __uint_as_float(v2[k]));
          {
            uint32_t pk[4], pl[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int jj = 2 * k, j0 = g * 8 + jj;
              if (plain) {
                const float z0 = __uint_as_float(v[jj]) * zs, z1 = __uint_as_float(v[jj + 1]) * zs;
                zmax_ = fmaxf(zmax_, fmaxf(z0, z1));
                const float e0 = mu_ == -INFINITY ? 0.0f : ex2_approx(z0 + nmu);
                const float e1 = mu_ == -INFINITY ? 0.0f : ex2_approx(z1 + nmu);
                __half2 w2 = __floats2half2_rn(e0, e1);
                pk[k] = *reinterpret_cast<uint32_t*>(&w2);
                const float2 back = __half22float2(w2);
                if (PLO) {
                  pl[k] = pack_half2(e0 - back.x, e1 - back.y);
                  sum_ += e0 + e1;
                } else {
                  // the fp16 weights are what PV uses and what the sum adds
                  sum_ += back.x + back.y;
                }
              } else {
                const float r0 = rsb[j0], r1 = rsb[j0 + 1];
                const float z0 = r0 >= 0.0f ? __uint_as_float(v[jj]) * (zs * r0) : -INFINITY;
                const float z1 = r1 >= 0.0f ? __uint_as_float(v[jj + 1]) * (zs * r1) : -INFINITY;
                zmax_ = fmaxf(zmax_, fmaxf(z0, z1));
                float e0 = (mu_ == -INFINITY) ? 0.0f : ex2_approx(z0 + nmu);
                float e1 = (mu_ == -INFINITY) ? 0.0f : ex2_approx(z1 + nmu);
                const float w0 = r0 > 0.0f ? r0 : 0.0f, w1 = r1 > 0.0f ? r1 : 0.0f;
                __half2 w2 = __floats2half2_rn(e0 * w0, e1 * w1);
                pk[k] = *reinterpret_cast<uint32_t*>(&w2);
                const float2 back = __half22float2(w2);
                if (PLO) {
                  pl[k] = pack_half2(e0 * w0 - back.x, e1 * w1 - back.y);
                } else {
                  // sparse rows: sum exactly the fp16 weights the PV product uses
                  if (r0 == 1.0f) e0 = back.x;
                  if (r1 == 1.0f) e1 = back.y;
                }
                sum_ += e0 + e1;
              }
            }
            // 16-byte chunk of 8 rows: rows 32 hf + 8 g ..
            if (act) *reinterpret_cast<uint4*>(prow + swz128(h, 4 * hf + g)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            if (PLO && act)
              *reinterpret_cast<uint4*>(plow + swz128(h, 4 * hf + g)) = make_uint4(pl[0], pl[1], pl[2], pl[3]);
          }
        }
        zmax_ = fmaxf(zmax_, __shfl_xor_sync(0xffffffffu, zmax_, 16));  // both halves of the head
      };
      float mu = m, sum = 0.0f;
      if (ok) {
        // a head without a running max yet starts from this chunk's maximum
        const bool first = __any_sync(0xffffffffu, act && m == -INFINITY);
        float zmax;
        if (first) {
          p_pass(-INFINITY, sum, zmax);  // max only (no weights: every e is 0)
          if (m == -INFINITY) mu = zmax;
        }
        p_pass(mu, sum, zmax);
        // the running max moves only when the chunk exceeds it by more than
        // 2^15 (rare after the first chunk): the chunk is redone
        const bool redo = act && mu != -INFINITY && zmax > mu + kRescaleLog2;
        if (__any_sync(0xffffffffu, redo)) {
          if (redo) mu = zmax;
          p_pass(mu, sum, zmax);
        }
      }
      const bool resc = act && m != -INFINITY && mu != m;
      const float corr = resc ? exp2f(m - mu) : 1.0f;
      if (act && hf == 0) corr_s[h] = corr;
      const bool any = soft_sync_or(resc);  // also publishes corr_s
      if (any && i > 0 && ok) {
        // rescale the output accumulator of earlier chunks (rare): PV(i - 1)
        // must have completed first
        if (!mbar_wait_group(bar_kv_empty + 8 * ((i - 1) & 1), ((i - 1) >> 1) & 1, P.wait_ns, threadIdx.x == 0,
                             *abort != 0, 1, 128)) {
          if (threadIdx.x == 0 && !*abort) {
            set_status(P.status, CSA2_ERR_TIMEOUT);
            *abort = 1;
          }
        } else {
          tc::fence_after_sync();
#pragma unroll 1
          for (int mt = 0; mt < Ly::kMT; ++mt)
#pragma unroll
            for (int g = 0; g < HQ / 16; ++g) {
              const uint32_t ta = s_lane + Ly::kColO + mt * HQ + g * 16;
              uint32_t v[16];
              tc::ld_32x32b_x16(ta, v);
              tc::ld_wait();
#pragma unroll
              for (int k = 0; k < 16; ++k) v[k] = __float_as_uint(__uint_as_float(v[k]) * corr_s[g * 16 + k]);
              tc::st_32x32b_x16(ta, v);
            }
          tc::st_wait();
        }
      }
      if (ok && act) {
        l = l * corr + sum;
        m = mu;
      }
      tc::fence_proxy_async_smem();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar_p_full + 8 * bf);
    }
    const float lt = l + __shfl_xor_sync(0xffffffffu, l, 16);  // both halves of the head
    if (act && hf == 0) {
      l_s[h] = lt;
      m_s[h] = m;
      corr_s[h] = lt > 0.0f ? 1.0f / lt : 0.0f;  // reciprocal row sum for the epilogue
    }
  }
  // ---- epilogue: every warp; the tiles are free once the last PV completed
  if (threadIdx.x == 0 && n_mine > 0 && !*abort) {
    const int il = n_mine - 1;
    if (!mbar_wait_bounded(bar_kv_empty + 8 * (il & 1), (il >> 1) & 1, P.wait_ns)) {
      set_status(P.status, CSA2_ERR_TIMEOUT);
      *abort = 1;
    }
  }
  __syncthreads();
  tc::fence_after_sync();
  const bool have = n_mine > 0 && !*abort;
  // O^T (TMEM lanes = latent dims) -> staging [h][d] in the tile region:
  // fp32 partials (split mode) or the normalised output in the output dtype
  {
    const bool f32_stage = nsplit > 1 || P.out_f32;
    float* st32 = reinterpret_cast<float*>(smem + Ly::kOffTile);
    __nv_bfloat16* st16 = reinterpret_cast<__nv_bfloat16*>(smem + Ly::kOffTile);
    const int q = warp & 3;
    const int nw_q = (kThreads / 32 - q + 3) / 4;  // warps sharing this lane quarter
    const int wi = warp >> 2;
    constexpr int kItems = Ly::kMT * (HQ / 16);
    for (int item = wi; item < kItems; item += nw_q) {
      const int mt = item / (HQ / 16), g = item % (HQ / 16);
      const int d = mt * 128 + q * 32 + lane;
      uint32_t v[16];
      if (have) {
        tc::ld_32x32b_x16(tmem + ((uint32_t)(q * 32) << 16) + Ly::kColO + mt * HQ + g * 16, v);
        tc::ld_wait();
      }
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const int hh = g * 16 + k;
        float o = have ? __uint_as_float(v[k]) : 0.0f;
        if (nsplit == 1) o = have ? o * corr_s[hh] : 0.0f;
        if (f32_stage)
          st32[hh * D + d] = o;
        else
          st16[hh * D + d] = __float2bfloat16_rn(o);
      }
    }
    tc::fence_proxy_async_smem();  // the staging is read by the bulk copy
    __syncthreads();
    // staging -> global: the contiguous [HQ][D] block in one bulk copy (16-byte
    // stores by every thread when the destination is not 16-byte aligned)
    uint8_t* dst = nsplit > 1 ? reinterpret_cast<uint8_t*>(P.part_o + (slot0 + split) * HQ * D)
                              : reinterpret_cast<uint8_t*>(io.out) + (int64_t)tok * HQ * D * (P.out_f32 ? 4 : 2);
    const uint32_t bytes = (uint32_t)HQ * D * (f32_stage ? 4 : 2);
    if ((reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
      if (threadIdx.x == 0) {
        for (uint32_t off = 0; off < bytes; off += 32768)
          tc::bulk_store(dst + off, sbase + Ly::kOffTile + off, min(32768u, bytes - off));
        tc::bulk_commit();
        if (nsplit > 1) {
          tc::bulk_wait_all();
          tc::fence_proxy_async_global();  // before the split-arrival atomic below
        } else {
          tc::bulk_wait_read();  // final output: only the staging must stay valid
        }
      }
    } else {
      const uint32_t* src = reinterpret_cast<const uint32_t*>(smem + Ly::kOffTile);
      for (uint32_t e = threadIdx.x; e < bytes / 4; e += kThreads) {
        const uint32_t v = src[e];
        memcpy(dst + 4 * e, &v, 4);
      }
    }
    if (threadIdx.x < HQ) {
      const int hh = threadIdx.x;
      const float lh = have ? l_s[hh] : 0.0f;
      const float m2 = have ? m_s[hh] : -INFINITY;
      if (nsplit == 1) {
        if (io.lse) io.lse[(int64_t)tok * HQ + hh] = lh > 0.0f ? (m2 + log2f(lh)) * 0.6931471805599453f : -INFINITY;
      } else {
        float* ml = P.part_ml + ((slot0 + split) * HQ + hh) * 2;
        ml[0] = lh > 0.0f ? m2 * 0.6931471805599453f : -INFINITY;
        ml[1] = lh;
      }
    }
  }
  // split mode: the last CTA of this token to finish merges the partials
  // (log-sum-exp weights) and restores the arrival counter to zero
  if (nsplit > 1) {
    volatile int* s_last = reinterpret_cast<volatile int*>(smem + Ly::kOffMisc + 8);
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) *s_last = atomicAdd(P.done + (int64_t)layer * P.qb.n_tok + tok, 1) == nsplit - 1;
    __syncthreads();
    if (*s_last) {
      __threadfence();
      float* wgt = reinterpret_cast<float*>(smem + Ly::kOffTile);  // [nsplit][HQ] weights (tiles are free)
      for (int hh = threadIdx.x; hh < HQ; hh += kThreads) {
        float M = -INFINITY;
        for (int sp = 0; sp < nsplit; ++sp) {
          const float* ml = P.part_ml + ((slot0 + sp) * HQ + hh) * 2;
          if (__ldcg(ml + 1) > 0.0f) M = fmaxf(M, __ldcg(ml));
        }
        float L = 0.0f;
        for (int sp = 0; sp < nsplit; ++sp) {
          const float* ml = P.part_ml + ((slot0 + sp) * HQ + hh) * 2;
          const float lv = __ldcg(ml + 1);
          const float a = lv > 0.0f ? __expf(__ldcg(ml) - M) : 0.0f;
          wgt[sp * HQ + hh] = a;
          L += a * lv;
        }
        const float inv = L > 0.0f ? 1.0f / L : 0.0f;
        for (int sp = 0; sp < nsplit; ++sp) wgt[sp * HQ + hh] *= inv;
        if (io.lse) io.lse[(int64_t)tok * HQ + hh] = L > 0.0f ? M + logf(L) : -INFINITY;
      }
      __syncthreads();
      // 16-byte loads, all splits of 2 groups in flight per thread (nsplit <= 4)
      constexpr int kTot4 = HQ * D / 4;
      const float4* po = reinterpret_cast<const float4*>(P.part_o) + slot0 * kTot4;
      for (int e0 = threadIdx.x; e0 < kTot4; e0 += kThreads * 2) {
        float4 v[2][4];
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
          for (int sp = 0; sp < 4; ++sp) {
            const int e = e0 + u * kThreads;
            v[u][sp] = (sp < nsplit && e < kTot4) ? __ldcg(po + (int64_t)sp * kTot4 + e) : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int e = e0 + u * kThreads;
          if (e >= kTot4) continue;
          const int hh = (e * 4) / D;
          float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int sp = 0; sp < 4; ++sp) {
            if (sp >= nsplit) continue;
            const float wv = wgt[sp * HQ + hh];
            a.x += wv * v[u][sp].x;
            a.y += wv * v[u][sp].y;
            a.z += wv * v[u][sp].z;
            a.w += wv * v[u][sp].w;
          }
          const int64_t oi = (int64_t)tok * HQ * D + (int64_t)e * 4;
          if (P.out_f32) {
            *reinterpret_cast<float4*>(reinterpret_cast<float*>(io.out) + oi) = a;
          } else {
            __nv_bfloat162 lo2 = __floats2bfloat162_rn(a.x, a.y), hi2 = __floats2bfloat162_rn(a.z, a.w);
            uint2 pk;
            pk.x = *reinterpret_cast<uint32_t*>(&lo2);
            pk.y = *reinterpret_cast<uint32_t*>(&hi2);
            *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(io.out) + oi) = pk;
          }
        }
      }
      if (threadIdx.x == 0) P.done[(int64_t)layer * P.qb.n_tok + tok] = 0;
    }
  }
  // no MMA of ours may be in flight when TMEM is released
  grid_dep_launch();
  if (threadIdx.x == 0) {
    if (!mbar_wait_bounded(bar_drain, 0, P.wait_ns)) set_status(P.status, CSA2_ERR_TIMEOUT);
  }
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

template <int D, int HQ, bool QLO, bool PLO>
int launch_t(const Params& p, int nsplit, int n_layers, cudaStream_t st) {
  using Ly = Layout<D, HQ, QLO, PLO>;
  static_assert(Ly::kBytes <= 232448, "attention shared memory");
  static bool attr[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr[dev]) {
    if (int rc = cuda_check(cudaFuncSetAttribute(k_attend_tc<D, HQ, QLO, PLO>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 Ly::kBytes),
                            "attend smem attribute"))
      return rc;
    int fit = 0;
    if (int rc = cuda_check(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&fit, k_attend_tc<D, HQ, QLO, PLO>, kThreads,
                                                                          Ly::kBytes),
                            "attend occupancy"))
      return rc;
    if (fit < 1) return fail(CSA2_ERR_UNSUPPORTED, "attention kernel does not fit on an SM");
    attr[dev] = true;
  }
  Launch L_("attend_tc", st);
  return cuda_check(launch_overlapped(kOverlapAttend, k_attend_tc<D, HQ, QLO, PLO>,
                                      dim3(nsplit, p.qb.n_tok, n_layers), dim3(kThreads), Ly::kBytes, st, p),
                    "k_attend_tc");
}

// fp32 queries (the fp16 residual copy) exist for D * Hq <= 16384 only
template <int D, int HQ, bool PLO>
int launch_q(const Params& p, int nsplit, int n_layers, cudaStream_t st) {
  if constexpr (D * HQ <= 16384) {
    return launch_t<D, HQ, true, PLO>(p, nsplit, n_layers, st);
  } else {
    (void)p, (void)nsplit, (void)n_layers, (void)st;
    return fail(CSA2_ERR_UNSUPPORTED, "fp32 queries need D * Hq <= 16384");
  }
}

}  // namespace attend_tc

// shapes of the attention kernel: D in {128, 512}, Hq in {16, 32, 64}; fp32
// queries keep an fp16 residual copy next to the fp16 query, which fits in
// shared memory for D * Hq <= 16384.
bool attend_tc_supported(int D, int Hq, int q_dtype) {
  if (!((D == 512 || D == 128) && (Hq == 64 || Hq == 32 || Hq == 16))) return false;
  if (q_dtype == CSA2_F32 && D * Hq > 16384) return false;
  return true;
}

int launch_attend_tc(const csa2_query_batch* qb, int q_dtype, int Hq, const csa2_fp4_cache* kv, int K,
                     const AttendLayer* layers, int n_layers, float scale, int out_dtype, float* part_o,
                     float* part_ml, int* done, int nsplit, cudaStream_t st) {
  using namespace attend_tc;
  if (n_layers < 1 || n_layers > kMaxLayers) return fail(CSA2_ERR_UNSUPPORTED, "1..%d layers per launch", kMaxLayers);
  if (nsplit < 1 || nsplit > 4) return fail(CSA2_ERR_UNSUPPORTED, "1..4 attention splits");
  if (K < 1 || K > kMaxRows) return fail(CSA2_ERR_UNSUPPORTED, "K must be 1..%d", kMaxRows);
  if (kv->n_rows >= (int64_t(1) << 31)) return fail(CSA2_ERR_UNSUPPORTED, "Main KV too large for 32-bit rows");
  Params p{};
  p.qb = *qb;
  p.q_f32 = q_dtype == CSA2_F32;
  p.kv = *kv;
  p.K = K;
  p.has_swa = layers[0].swa != nullptr;
  if (p.has_swa) {
    p.swa_cap = layers[0].swa->cap;
    p.swa_window = layers[0].swa->window;
  }
  for (int l = 0; l < n_layers; ++l) {
    if ((layers[l].swa != nullptr) != (p.has_swa != 0)) return fail(CSA2_ERR_INVALID_ARG, "mixed sliding-window layers");
    if (layers[l].swa && (layers[l].swa->cap != p.swa_cap || layers[l].swa->window != p.swa_window))
      return fail(CSA2_ERR_INVALID_ARG, "sliding-window shapes differ between layers");
    p.io[l].idx = layers[l].idx;
    p.io[l].idx_n = layers[l].idx_n;
    p.io[l].q = layers[l].q;
    p.io[l].out = layers[l].out;
    p.io[l].lse = layers[l].lse;
    p.io[l].swa_codes = layers[l].swa ? layers[l].swa->codes : nullptr;
    p.io[l].swa_scale = layers[l].swa ? layers[l].swa->scale : nullptr;
  }
  p.scale = scale;
  p.out_f32 = out_dtype == CSA2_F32;
  p.part_o = part_o;
  p.part_ml = part_ml;
  p.done = done;
  p.status = status_ptr();
  p.wait_ns = 1000000000ull;
  const int D = kv->dim;
  const bool qlo = p.q_f32 != 0;
  // fp32 outputs take the two-part P (see the softmax)
  const bool plo = p.out_f32 != 0;
#define CSA2_ATT_CASE(d, hq)                                                                                   \
  if (D == d && Hq == hq) {                                                                                   \
    if (plo) return qlo ? launch_q<d, hq, true>(p, nsplit, n_layers, st) : launch_t<d, hq, false, true>(p, nsplit, n_layers, st); \
    return qlo ? launch_q<d, hq, false>(p, nsplit, n_layers, st) : launch_t<d, hq, false, false>(p, nsplit, n_layers, st); \
  }
  CSA2_ATT_CASE(512, 64)
  CSA2_ATT_CASE(512, 32)
  CSA2_ATT_CASE(512, 16)
  CSA2_ATT_CASE(128, 64)
  CSA2_ATT_CASE(128, 32)
  CSA2_ATT_CASE(128, 16)
#undef CSA2_ATT_CASE
  return fail(CSA2_ERR_UNSUPPORTED, "attend_tc shape");
}

}  // namespace csa2
