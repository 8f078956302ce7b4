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
// One CTA per (query token, split); each walks its 128-row chunks of the key
// set.  Per chunk:
//   1. all 8 warps gather the chunk's rows and dequantise them exactly to
//      fp16 (E2M1 x E4M3 products, or E4M3 window codes) into a 128B-swizzled
//      shared tile [64-element d-block][row][128 B];
//   2. one thread issues S^T = K q^T on tcgen05 (kind::f16, M = 128 rows,
//      N = heads, K = D) into TMEM;
//   3. warps 0..3 (one row each) scale and mask S^T, reduce per-head maxima and
//      sums across rows with a halving shuffle transpose, keep a running
//      (log2) max that only moves when a chunk exceeds it by more than 2^8
//      (then the TMEM output accumulator is rescaled), and write
//      P = 2^(z - m) as fp16 rows into shared memory (window rows carry their
//      per-token scale into P);
//   4. one thread issues O^T += V^T P^T (M = 128 latent dims per tile, N =
//      heads, K = 128 rows) reading the same dequantised tile as V.
// The epilogue divides by the row sum and writes the output (or the split's
// unnormalised partial with its max and sum for the merge kernel).
#include "internal.h"
#include "tc_common.cuh"

namespace csa2 {
namespace attend_tc {

constexpr int kRows = 128;
constexpr int kThreads = 256;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.0f;  // P stays <= 2^8 between rescales (fp16-safe)

constexpr int kMaxLayers = 32;  // layers attended in one launch (grid.z), each with its own index list

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

template <int D, int HQ, bool QLO>
struct Layout {
  static constexpr int kKB = D / 64;   // 64-element d-blocks
  static constexpr int kMT = D / 128;  // PV M tiles
  static constexpr int kPRow = HQ * 2; // bytes per P row
  static constexpr uint32_t kOffK = 0;
  static constexpr uint32_t kOffQ = kOffK + kRows * D * 2;
  static constexpr uint32_t kOffQlo = kOffQ + HQ * D * 2;
  static constexpr uint32_t kOffP = kOffQlo + (QLO ? HQ * D * 2 : 0);
  static constexpr uint32_t kOffRed = kOffP + kRows * kPRow;     // [4][HQ] f32
  static constexpr uint32_t kOffM = kOffRed + 4 * HQ * 4;        // running max (log2) [HQ]
  static constexpr uint32_t kOffL = kOffM + HQ * 4;              // running sum [HQ]
  static constexpr uint32_t kOffRs = kOffL + HQ * 4;             // row scale [128] f32
  static constexpr uint32_t kOffValid = kOffRs + kRows * 4;      // row valid [128] i32
  static constexpr uint32_t kOffRows = kOffValid + kRows * 4;    // gathered row index [128] i64
  static constexpr uint32_t kOffMu = kOffRows + kRows * 8;       // max used for this chunk [HQ]
  static constexpr uint32_t kOffCorr = kOffMu + HQ * 4;          // rescale factor [HQ]
  static constexpr uint32_t kOffBar = kOffCorr + HQ * 4;         // 3 mbarriers (S, PV, drain)
  static constexpr uint32_t kOffMisc = kOffBar + 24;             // tmem base, abort, rescale flag
  static constexpr uint32_t kBytes = kOffMisc + 16 + 1024;
  static constexpr int kChains = kKB < 4 ? kKB : 4;  // S = K q^T split over this many issuing threads
  static constexpr uint32_t kColS = 0;                // chain c accumulates at kColS + c * HQ
  static constexpr uint32_t kColO = 256;              // O^T tile mt at kColO + mt * HQ
  static_assert(kChains * HQ <= 256 && kMT * HQ <= 256, "TMEM budget");
};

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// swizzled byte offset of 16-byte chunk c of row r for rows of `rb` bytes
__device__ __forceinline__ uint32_t swz(uint32_t r, uint32_t c, uint32_t rb) {
  uint32_t x = rb == 128 ? (r & 7) : rb == 64 ? ((r >> 1) & 3) : ((r >> 2) & 1);
  return r * rb + ((c ^ x) << 4);
}

// reduce v[0..N) across the 32 lanes of a warp by repeated halving; afterwards
// lane L holds, in v[0..max(1,N/32)), the warp-wide result for heads
// N >= 32: 2L.. (N/32 of them, here N = 64 -> heads 2L, 2L+1);
// N < 32: head L / (32/N) (lanes sharing a head hold the same value)
template <int N, bool MAX>
__device__ __forceinline__ void warp_transpose_reduce(float (&v)[N], int lane) {
  int size = N;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    if (size > 1) {
      const bool up = (lane & o) != 0;
      const int half = size / 2;
#pragma unroll
      for (int i = 0; i < N / 2; ++i) {
        if (i < half) {
          float send = up ? v[i] : v[i + half];
          float keep = up ? v[i + half] : v[i];
          float got = __shfl_xor_sync(0xffffffffu, send, o);
          v[i] = MAX ? fmaxf(keep, got) : keep + got;
        }
      }
      size = half;
    } else {
      float got = __shfl_xor_sync(0xffffffffu, v[0], o);
      v[0] = MAX ? fmaxf(v[0], got) : v[0] + got;
    }
  }
}

template <int HQ>
__device__ __forceinline__ int reduced_head(int lane, int i) {
  if constexpr (HQ >= 32) {
    return lane * (HQ / 32) + i;
  } else {
    return lane / (32 / HQ);
  }
}

template <int D, int HQ, bool QLO>
__global__ void __launch_bounds__(kThreads, 1) k_attend_tc(const __grid_constant__ Params P) {
  using Ly = Layout<D, HQ, QLO>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar_s = sbase + Ly::kOffBar, bar_pv = bar_s + 8, bar_drain = bar_s + 16;
  volatile uint32_t* tmem_holder = reinterpret_cast<volatile uint32_t*>(smem + Ly::kOffMisc);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + Ly::kOffMisc + 4);
  volatile int* any_rescale = reinterpret_cast<volatile int*>(smem + Ly::kOffMisc + 8);
  float* mu_s = reinterpret_cast<float*>(smem + Ly::kOffMu);
  float* corr_s = reinterpret_cast<float*>(smem + Ly::kOffCorr);
  float* red = reinterpret_cast<float*>(smem + Ly::kOffRed);
  float* m_s = reinterpret_cast<float*>(smem + Ly::kOffM);
  float* l_s = reinterpret_cast<float*>(smem + Ly::kOffL);
  float* rs = reinterpret_cast<float*>(smem + Ly::kOffRs);
  int* valid = reinterpret_cast<int*>(smem + Ly::kOffValid);
  int64_t* rows_s = reinterpret_cast<int64_t*>(smem + Ly::kOffRows);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tok = blockIdx.y, split = blockIdx.x, nsplit = gridDim.x, layer = blockIdx.z;
  const LayerIO& io = P.io[layer];  // read from parameter space where used
  const int64_t slot0 = ((int64_t)layer * P.qb.n_tok + tok) * nsplit;  // this token's partial slots
  const int b = __ldg(P.qb.tok_seq + tok);
  const int64_t p = __ldg(P.qb.tok_pos + tok);

  if (threadIdx.x == 0) {
    mbar_init(bar_s, Ly::kChains);
    mbar_init(bar_pv, Ly::kMT);
    mbar_init(bar_drain, 4);
    *abort = 0;
    *any_rescale = 0;
    tc::fence_barrier_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(sbase + Ly::kOffMisc, 512);
    tc::tmem_relinquish();
    tc::fence_before_sync();
  }
  for (int h = threadIdx.x; h < HQ; h += kThreads) {
    m_s[h] = -INFINITY;
    l_s[h] = 0.0f;
  }
  // query -> fp16 (K-major, 128B swizzle); f32 queries also keep the residual.
  // Loads are issued in batches of 8 independent 16-byte reads per thread.
  {
    constexpr int kUnitsQ = HQ * D / 8;  // 8 consecutive d per unit
    constexpr int kBatch = 8;
    for (int e0 = 0; e0 < kUnitsQ; e0 += kThreads * kBatch) {
      float f[kBatch][8];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int e = e0 + u * kThreads + threadIdx.x;
        if (e >= kUnitsQ) continue;
        const int h = e / (D / 8), c8 = e % (D / 8);
        const int64_t off = ((int64_t)tok * HQ + h) * D + c8 * 8;
        if (P.q_f32) {
          const float4* s4 = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(io.q) + off);
          float4 a = __ldg(s4), bb = __ldg(s4 + 1);
          f[u][0] = a.x; f[u][1] = a.y; f[u][2] = a.z; f[u][3] = a.w;
          f[u][4] = bb.x; f[u][5] = bb.y; f[u][6] = bb.z; f[u][7] = bb.w;
        } else {
          uint4 w4 = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(io.q) + off));
          const uint32_t ww[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            f[u][2 * k] = __uint_as_float(ww[k] << 16);
            f[u][2 * k + 1] = __uint_as_float(ww[k] & 0xFFFF0000u);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int e = e0 + u * kThreads + threadIdx.x;
        if (e >= kUnitsQ) continue;
        const int h = e / (D / 8), c8 = e % (D / 8);
        const int kb = c8 / 8, c = c8 % 8;
        uint4 hi, lo;
        uint32_t* hp = &hi.x;
        uint32_t* lp = &lo.x;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          __half2 h2 = __floats2half2_rn(f[u][2 * k], f[u][2 * k + 1]);
          hp[k] = *reinterpret_cast<uint32_t*>(&h2);
          float2 back = __half22float2(h2);
          lp[k] = pack_half2(f[u][2 * k] - back.x, f[u][2 * k + 1] - back.y);
        }
        const uint32_t o = kb * (HQ * 128) + swz(h, c, 128);
        *reinterpret_cast<uint4*>(smem + Ly::kOffQ + o) = hi;
        if (QLO) *reinterpret_cast<uint4*>(smem + Ly::kOffQlo + o) = lo;
      }
    }
  }
  tc::fence_proxy_async_smem();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_holder;

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
  const uint32_t idesc_s = tc::idesc_f16(128, HQ, 0, 0);
  const uint32_t idesc_pv = tc::idesc_f16(128, HQ, 1, 1);
  const tc::SmemLayout p_sw = HQ == 64 ? tc::kSwizzle128B : HQ == 32 ? tc::kSwizzle64B : tc::kSwizzle32B;

  int it = 0;
  for (int chunk = split; chunk < n_chunks; chunk += nsplit, ++it) {
    if (it > 0) {  // the previous chunk's PV still reads the tile (thread 0 probes, the rest park)
      if (threadIdx.x == 0 && !mbar_wait_bounded(bar_pv, (it - 1) & 1, P.wait_ns)) {
        set_status(P.status, CSA2_ERR_TIMEOUT);
        *abort = 1;
      }
      __syncthreads();
      if (*abort) break;
      tc::fence_after_sync();
    }
    // ---- 1. gather + dequantise the chunk into the K/V tile
    const bool swa_chunk = chunk >= n_sp;
    // row addresses first (one index load per row), so the code loads below
    // are independent of each other and all in flight together
    if (threadIdx.x < kRows) {
      const int r = threadIdx.x;
      int64_t row = -1;
      float scale_r = 1.0f;
      if (!swa_chunk) {
        const int j = chunk * kRows + r;
        if (j < n_sel) {
          const int32_t t = __ldg(io.idx + (int64_t)tok * P.K + j);
          if (t >= 0 && t <= p) {
            row = cache_row(P.kv, b, t);
            if (row < 0 || row >= P.kv.n_rows) row = -1;
          }
          if (row < 0) set_status(P.status, CSA2_ERR_RANGE);
        }
      } else {
        const int64_t t = w_lo + (int64_t)(chunk - n_sp) * kRows + r;
        if (t <= p) {
          row = (int64_t)b * P.swa_cap + t % P.swa_cap;
          scale_r = __ldg(io.swa_scale + row);
        } else {
          scale_r = 0.0f;
        }
      }
      rows_s[r] = row;
      valid[r] = row >= 0;
      rs[r] = scale_r;
    }
    __syncthreads();
    if (!swa_chunk) {
      constexpr int kUnits = D / 32;  // 16-byte code units (32 values, one scale) per row
      constexpr int kPer = kRows * kUnits / kThreads;
      uint4 cw[kPer];
      uint32_t sb[kPer];
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        const int u = threadIdx.x + i * kThreads;
        const int r = u / kUnits, g = u % kUnits;
        const int64_t row = rows_s[r];
        if (row >= 0) {
          cw[i] = __ldg(reinterpret_cast<const uint4*>(P.kv.codes + row * (D / 2)) + g);
          sb[i] = __ldg(P.kv.scales + row * (D / 32) + g);
        } else {
          cw[i] = make_uint4(0, 0, 0, 0);
          sb[i] = 0;
        }
      }
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        const int u = threadIdx.x + i * kThreads;
        const int r = u / kUnits, g = u % kUnits;
        const __half sh = __float2half_rn(e4m3_to_f32(sb[i]));
        const __half2 s2 = __halves2half2(sh, sh);
        const uint32_t words[4] = {cw[i].x, cw[i].y, cw[i].z, cw[i].w};
        uint32_t outw[16];
#pragma unroll
        for (int k = 0; k < 4; ++k)
#pragma unroll
          for (int bb = 0; bb < 4; ++bb) {
            uint32_t h2 = tc::e2m1x2_to_f16x2((words[k] >> (8 * bb)) & 0xFFu);
            __half2 v = __hmul2(*reinterpret_cast<__half2*>(&h2), s2);
            outw[k * 4 + bb] = *reinterpret_cast<uint32_t*>(&v);
          }
        // 32 values = d in [32g, 32g+32): d-block g/2, 16-byte chunks (g%2)*4 .. +4
        const int kb = g / 2, c0 = (g % 2) * 4;
#pragma unroll
        for (int k = 0; k < 4; ++k)
          *reinterpret_cast<uint4*>(smem + Ly::kOffK + kb * (kRows * 128) + swz(r, c0 + k, 128)) =
              make_uint4(outw[4 * k], outw[4 * k + 1], outw[4 * k + 2], outw[4 * k + 3]);
      }
    } else {
      constexpr int kUnits = D / 16;  // 16 FP8 codes per unit
      constexpr int kPer = kRows * kUnits / kThreads;
      uint4 cw[kPer];
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        const int u = threadIdx.x + i * kThreads;
        const int r = u / kUnits, g = u % kUnits;
        const int64_t row = rows_s[r];
        cw[i] = row >= 0 ? __ldg(reinterpret_cast<const uint4*>(io.swa_codes + row * D) + g) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        const int u = threadIdx.x + i * kThreads;
        const int r = u / kUnits, g = u % kUnits;
        const uint32_t words[4] = {cw[i].x, cw[i].y, cw[i].z, cw[i].w};
        uint32_t outw[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          outw[2 * k] = tc::e4m3x2_to_f16x2(words[k] & 0xFFFFu);
          outw[2 * k + 1] = tc::e4m3x2_to_f16x2(words[k] >> 16);
        }
        const int kb = g / 4, c0 = (g % 4) * 2;
#pragma unroll
        for (int k = 0; k < 2; ++k)
          *reinterpret_cast<uint4*>(smem + Ly::kOffK + kb * (kRows * 128) + swz(r, c0 + k, 128)) =
              make_uint4(outw[4 * k], outw[4 * k + 1], outw[4 * k + 2], outw[4 * k + 3]);
      }
    }
    tc::fence_proxy_async_smem();
    __syncthreads();

    // ---- 2. S^T = K q^T, the K chain split over kChains issuing threads
    //         (chain c: d-blocks c, c + kChains, ...; its own accumulator)
    if (warp == 0 && lane < Ly::kChains) {
      tc::fence_after_sync();
      const int c = lane;
#pragma unroll 1
      for (int kb = c; kb < Ly::kKB; kb += Ly::kChains)
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t ad = tc::smem_desc(sbase + Ly::kOffK + kb * (kRows * 128) + ks * 32, 16, 1024, tc::kSwizzle128B);
          const uint64_t bd = tc::smem_desc(sbase + Ly::kOffQ + kb * (HQ * 128) + ks * 32, 16, 1024, tc::kSwizzle128B);
          tc::mma_f16(tmem + Ly::kColS + c * HQ, ad, bd, idesc_s, (kb != c || ks) ? 1u : 0u);
          if (QLO) {
            const uint64_t bl =
                tc::smem_desc(sbase + Ly::kOffQlo + kb * (HQ * 128) + ks * 32, 16, 1024, tc::kSwizzle128B);
            tc::mma_f16(tmem + Ly::kColS + c * HQ, ad, bl, idesc_s, 1u);
          }
        }
      tc::commit(bar_s);
    }
    __syncwarp();

    // ---- 3. softmax over the rows (warps 0..3: one row per thread)
    if (warp < 4) {
      if (!mbar_wait_warp(bar_s, it & 1, P.wait_ns)) {
        set_status(P.status, CSA2_ERR_TIMEOUT);
        *abort = 1;
      }
      tc::fence_after_sync();
      const int r = warp * 32 + lane;
      const bool rv = valid[r] != 0;
      const float zscale = P.scale * kLog2e * rs[r];  // log2-domain score scale (window rows: * s_t)
      constexpr int kPer = HQ >= 32 ? HQ / 32 : 1;
      const uint32_t s_addr = tmem + ((uint32_t)(warp * 32) << 16) + Ly::kColS;
      // the chunk's scores (sum of the chains), scaled to the log2 domain
      // (window rows: * s_t); invalid rows -inf
      auto load_scores = [&](float (&z)[HQ]) {
#pragma unroll
        for (int g = 0; g < HQ / 16; ++g) {
          uint32_t v[Ly::kChains][16];
#pragma unroll
          for (int c = 0; c < Ly::kChains; ++c) tc::ld_32x32b_x16(s_addr + c * HQ + g * 16, v[c]);
          tc::ld_wait();
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            float acc = __uint_as_float(v[0][k]);
#pragma unroll
            for (int c = 1; c < Ly::kChains; ++c) acc += __uint_as_float(v[c][k]);
            z[g * 16 + k] = rv ? acc * zscale : -INFINITY;
          }
        }
      };
      // per-head maximum of this chunk
      {
        float mx[HQ];
        load_scores(mx);
        warp_transpose_reduce<HQ, true>(mx, lane);
#pragma unroll
        for (int i = 0; i < kPer; ++i) red[warp * HQ + reduced_head<HQ>(lane, i)] = mx[i];
      }
      tc::named_sync(1, 128);
      // running max: moves only when the chunk exceeds it by more than 2^8
      if (threadIdx.x < HQ) {
        const int h = threadIdx.x;
        const float cm = fmaxf(fmaxf(red[h], red[HQ + h]), fmaxf(red[2 * HQ + h], red[3 * HQ + h]));
        const float mo = m_s[h];
        float mu = mo;
        if (mo == -INFINITY || cm > mo + kRescaleLog2) mu = cm;
        mu_s[h] = mu;
        corr_s[h] = (mo == -INFINITY || mu == mo) ? 1.0f : exp2f(mo - mu);
        if (mo != -INFINITY && mu != mo) *any_rescale = 1;
      }
      tc::named_sync(1, 128);
      // rescale the output accumulator of earlier chunks (rare)
      if (*any_rescale && it > 0) {
#pragma unroll 1
        for (int mt = 0; mt < Ly::kMT; ++mt)
#pragma unroll
          for (int g = 0; g < HQ / 16; ++g) {
            const uint32_t ta = tmem + ((uint32_t)(warp * 32) << 16) + Ly::kColO + mt * HQ + g * 16;
            uint32_t v[16];
            tc::ld_32x32b_x16(ta, v);
            tc::ld_wait();
#pragma unroll
            for (int k = 0; k < 16; ++k) v[k] = __float_as_uint(__uint_as_float(v[k]) * corr_s[g * 16 + k]);
            tc::st_32x32b_x16(ta, v);
          }
        tc::st_wait();
      }
      // P = 2^(z - m) as fp16 rows [row][head]; window rows carry s_t into P.
      // z[] is reused for the weights entering the row sum.
      uint8_t* prow = smem + Ly::kOffP;
      const float rsr = rs[r];
      float z[HQ];
      load_scores(z);
#pragma unroll
      for (int c = 0; c < HQ / 8; ++c) {
        uint32_t pk[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int h0 = c * 8 + 2 * k;
          const float m0 = mu_s[h0], m1 = mu_s[h0 + 1];
          float e0 = (m0 == -INFINITY) ? 0.0f : exp2f(z[h0] - m0);
          float e1 = (m1 == -INFINITY) ? 0.0f : exp2f(z[h0 + 1] - m1);
          __half2 w2 = __floats2half2_rn(e0 * rsr, e1 * rsr);
          pk[k] = *reinterpret_cast<uint32_t*>(&w2);
          if (rsr == 1.0f) {  // sparse rows: sum exactly the fp16 weights the PV product uses
            float2 back = __half22float2(w2);
            e0 = back.x;
            e1 = back.y;
          }
          z[h0] = e0;
          z[h0 + 1] = e1;
        }
        *reinterpret_cast<uint4*>(prow + swz(r, c, Ly::kPRow)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      warp_transpose_reduce<HQ, false>(z, lane);
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        const int h = reduced_head<HQ>(lane, i);
        bool writer = true;
        if constexpr (HQ < 32) writer = (lane % (32 / HQ)) == 0;
        if (writer) red[warp * HQ + h] = z[i];
      }
      tc::named_sync(1, 128);
      if (threadIdx.x < HQ) {
        const int h = threadIdx.x;
        l_s[h] = l_s[h] * corr_s[h] + (red[h] + red[HQ + h]) + (red[2 * HQ + h] + red[3 * HQ + h]);
        m_s[h] = mu_s[h];
      }
      if (threadIdx.x == 0) *any_rescale = 0;
      tc::fence_proxy_async_smem();
      tc::fence_before_sync();
    }
    __syncthreads();
    if (*abort) break;

    // ---- 4. O^T += V^T P^T, one M tile (128 latent dims) per issuing thread
    if (warp == 0 && lane < Ly::kMT) {
      tc::fence_after_sync();
      const int mt = lane;
#pragma unroll
      for (int ks = 0; ks < kRows / 16; ++ks) {
        const uint64_t ad =
            tc::smem_desc(sbase + Ly::kOffK + (2 * mt) * (kRows * 128) + ks * 2048, kRows * 128, 1024, tc::kSwizzle128B);
        const uint64_t bd = tc::smem_desc(sbase + Ly::kOffP + ks * 16 * Ly::kPRow, 8 * Ly::kPRow, 8 * Ly::kPRow, p_sw);
        tc::mma_f16(tmem + Ly::kColO + mt * HQ, ad, bd, idesc_pv, (it > 0 || ks > 0) ? 1u : 0u);
      }
      tc::commit(bar_pv);
    }
    __syncwarp();
  }
  // ---- epilogue
  if (it > 0 && !*abort && threadIdx.x == 0) {
    if (!mbar_wait_bounded(bar_pv, (it - 1) & 1, P.wait_ns)) {
      set_status(P.status, CSA2_ERR_TIMEOUT);
      *abort = 1;
    }
  }
  __syncthreads();
  tc::fence_after_sync();
  const bool have = it > 0 && !*abort;
  if (warp < 4) {
#pragma unroll 1
    for (int mt = 0; mt < Ly::kMT; ++mt) {
      const int d = mt * 128 + warp * 32 + lane;
#pragma unroll
      for (int g = 0; g < HQ / 16; ++g) {
        uint32_t v[16];
        if (have) {
          tc::ld_32x32b_x16(tmem + ((uint32_t)(warp * 32) << 16) + Ly::kColO + mt * HQ + g * 16, v);
          tc::ld_wait();
        }
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const int h = g * 16 + k;
          const float o = have ? __uint_as_float(v[k]) : 0.0f;
          if (nsplit == 1) {
            const float l = l_s[h];
            const float val = l > 0.0f ? o / l : 0.0f;
            const int64_t oi = ((int64_t)tok * HQ + h) * D + d;
            if (P.out_f32)
              reinterpret_cast<float*>(io.out)[oi] = val;
            else
              reinterpret_cast<__nv_bfloat16*>(io.out)[oi] = __float2bfloat16_rn(val);
          } else {
            P.part_o[((slot0 + split) * HQ + h) * D + d] = o;
          }
        }
      }
    }
    if (threadIdx.x < HQ) {
      const int h = threadIdx.x;
      const float l = have ? l_s[h] : 0.0f;
      const float m2 = have ? m_s[h] : -INFINITY;
      if (nsplit == 1) {
        if (io.lse) io.lse[(int64_t)tok * HQ + h] = l > 0.0f ? (m2 + log2f(l)) * 0.6931471805599453f : -INFINITY;
      } else {
        float* ml = P.part_ml + ((slot0 + split) * HQ + h) * 2;
        ml[0] = l > 0.0f ? m2 * 0.6931471805599453f : -INFINITY;
        ml[1] = l;
      }
    }
  }
  // split mode: the last CTA of this token to finish merges the partials
  // (log-sum-exp weights) and restores the arrival counter to zero
  if (nsplit > 1) {
    __shared__ int s_last;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(P.done + (int64_t)layer * P.qb.n_tok + tok, 1) == nsplit - 1;
    __syncthreads();
    if (s_last) {
      __threadfence();
      float* wgt = red;  // [nsplit][HQ] weights, reusing the reduction scratch (nsplit <= 4 here)
      for (int h = threadIdx.x; h < HQ; h += kThreads) {
        float M = -INFINITY;
        for (int sp = 0; sp < nsplit; ++sp) {
          const float* ml = P.part_ml + ((slot0 + sp) * HQ + h) * 2;
          if (__ldcg(ml + 1) > 0.0f) M = fmaxf(M, __ldcg(ml));
        }
        float L = 0.0f;
        for (int sp = 0; sp < nsplit; ++sp) {
          const float* ml = P.part_ml + ((slot0 + sp) * HQ + h) * 2;
          const float l = __ldcg(ml + 1);
          const float a = l > 0.0f ? __expf(__ldcg(ml) - M) : 0.0f;
          wgt[sp * HQ + h] = a;
          L += a * l;
        }
        const float inv = L > 0.0f ? 1.0f / L : 0.0f;
        for (int sp = 0; sp < nsplit; ++sp) wgt[sp * HQ + h] *= inv;
        if (io.lse) io.lse[(int64_t)tok * HQ + h] = L > 0.0f ? M + logf(L) : -INFINITY;
      }
      __syncthreads();
      // 16-byte loads, all splits of 4 groups in flight per thread (nsplit <= 4)
      constexpr int kTot4 = HQ * D / 4;
      const float4* po = reinterpret_cast<const float4*>(P.part_o) + slot0 * kTot4;
      for (int e0 = threadIdx.x; e0 < kTot4; e0 += kThreads * 4) {
        float4 v[4][4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int sp = 0; sp < 4; ++sp) {
            const int e = e0 + u * kThreads;
            v[u][sp] = (sp < nsplit && e < kTot4) ? __ldcg(po + (int64_t)sp * kTot4 + e) : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int e = e0 + u * kThreads;
          if (e >= kTot4) continue;
          const int h = (e * 4) / D;
          float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int sp = 0; sp < 4; ++sp) {
            if (sp >= nsplit) continue;
            const float wv = wgt[sp * HQ + h];
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
  if (warp == 0 && lane < 4) tc::commit(bar_drain);  // every issuing thread
  __syncwarp();
  if (threadIdx.x == 0) {
    if (!mbar_wait_bounded(bar_drain, 0, P.wait_ns)) set_status(P.status, CSA2_ERR_TIMEOUT);
  }
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

template <int D, int HQ, bool QLO>
int launch_t(const Params& p, int nsplit, int n_layers, cudaStream_t st) {
  using Ly = Layout<D, HQ, QLO>;
  static bool attr[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr[dev]) {
    if (int rc = cuda_check(cudaFuncSetAttribute(k_attend_tc<D, HQ, QLO>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 Ly::kBytes),
                            "attend smem attribute"))
      return rc;
    attr[dev] = true;
  }
  Launch L_("attend_tc", st);
  k_attend_tc<D, HQ, QLO><<<dim3(nsplit, p.qb.n_tok, n_layers), kThreads, Ly::kBytes, st>>>(p);
  return cuda_check(cudaGetLastError(), "k_attend_tc");
}

}  // namespace attend_tc

// tensor-core attention is used for (D, Hq) in {(512, 64), (128, 16), (128, 64), (512, 16)};
// fp32 queries need the residual copy, which fits for D * Hq <= 16384.
bool attend_tc_supported(int D, int Hq, int q_dtype) {
  if (!((D == 512 || D == 128) && (Hq == 64 || Hq == 16))) return false;
  if (q_dtype == CSA2_F32 && D * Hq > 16384) return false;
  return true;
}

int launch_attend_tc(const csa2_query_batch* qb, int q_dtype, int Hq, const csa2_fp4_cache* kv, int K,
                     const AttendLayer* layers, int n_layers, float scale, int out_dtype, float* part_o,
                     float* part_ml, int* done, int nsplit, cudaStream_t st) {
  using namespace attend_tc;
  if (n_layers < 1 || n_layers > kMaxLayers) return fail(CSA2_ERR_UNSUPPORTED, "1..%d layers per launch", kMaxLayers);
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
  if (D == 512 && Hq == 64)
    return qlo ? fail(CSA2_ERR_UNSUPPORTED, "f32 q") : launch_t<512, 64, false>(p, nsplit, n_layers, st);
  if (D == 512 && Hq == 16)
    return qlo ? launch_t<512, 16, true>(p, nsplit, n_layers, st) : launch_t<512, 16, false>(p, nsplit, n_layers, st);
  if (D == 128 && Hq == 64)
    return qlo ? launch_t<128, 64, true>(p, nsplit, n_layers, st) : launch_t<128, 64, false>(p, nsplit, n_layers, st);
  if (D == 128 && Hq == 16)
    return qlo ? launch_t<128, 16, true>(p, nsplit, n_layers, st) : launch_t<128, 16, false>(p, nsplit, n_layers, st);
  return fail(CSA2_ERR_UNSUPPORTED, "attend_tc shape");
}

}  // namespace csa2
