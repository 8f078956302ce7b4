// kernels_simt.cuh -- FP4 quantiser, selection, and the CUDA-core scoring and
// attention kernels of the CSA2 decode step.
#pragma once

#include "common.cuh"

namespace csa2 {

// ============================================================================
// K1: FP4 quantiser.  One thread = 8 consecutive elements, 4 threads = one
// 32-element group.  scale = E4M3_rne_satfinite(amax / 6) (one fp32 RN
// division); codes = round-to-nearest-even of the exact |x|/scale on the E2M1
// grid, found by comparing |x| with scale * {.25,.75,1.25,1.75,2.5,3.5,5}
// (products exact in fp32), ties to the even code.
// ============================================================================
// Quantisation jobs of one launch: each a row-major fp32 matrix [rows][dim]
// written as codes [row][dim/2] + scales [row][dim/32], rows remapped through
// `slot` when given (cache append).  A thread takes 8 consecutive elements
// ("unit"); job j owns units [begin[j], begin[j+1]), multiples of 4, so the 4
// threads of a 32-element scale group never straddle two jobs.
constexpr int kQuantJobs = 12;
struct QuantJob {
  const float* x;
  const int64_t* slot;
  uint8_t* codes;
  uint8_t* scales;
  int dim;
};
struct QuantJobs {
  QuantJob job[kQuantJobs];
  int64_t begin[kQuantJobs + 1];
  int n;
};

__global__ void __launch_bounds__(256) k_quantize_fp4(const __grid_constant__ QuantJobs J, int* status) {
  const int64_t total = J.begin[J.n];
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t base = (int64_t)blockIdx.x * blockDim.x; base < total; base += stride) {
    int64_t i = base + threadIdx.x;
    bool active = i < total;
    float v[8];
    float amax = 0.0f;
    bool bad = false;
    int64_t r = 0, c8 = 0;
    int jb = 0;
    if (active) {
      while (jb + 1 < J.n && i >= J.begin[jb + 1]) ++jb;
      const int64_t per_row = J.job[jb].dim / 8;
      const int64_t li = i - J.begin[jb];
      r = li / per_row;
      c8 = li - r * per_row;
      const float4* xp = reinterpret_cast<const float4*>(J.job[jb].x + r * J.job[jb].dim + c8 * 8);
      float4 a = __ldg(xp), b = __ldg(xp + 1);
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
      v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        float m = fabsf(v[k]);
        bad |= !(m <= 3.402823466e38f);
        amax = fmaxf(amax, m);
      }
    }
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    int badq = __shfl_xor_sync(0xffffffffu, (int)bad, 1) | (int)bad;
    badq |= __shfl_xor_sync(0xffffffffu, badq, 2);
    if (!active) continue;
    const QuantJob& jo = J.job[jb];
    const int dim = jo.dim;
    int64_t orow = jo.slot ? __ldg(jo.slot + r) : r;
    uint32_t packed = 0;
    uint8_t sc = 0;
    if (!badq) {
      float q = __fdiv_rn(amax, 6.0f);
      sc = (uint8_t)__nv_cvt_float_to_fp8(q, __NV_SATFINITE, __NV_E4M3);
      float s = e4m3_to_f32(sc);
      const float t0 = s * 0.25f, t1 = s * 0.75f, t2 = s * 1.25f, t3 = s * 1.75f, t4 = s * 2.5f,
                  t5 = s * 3.5f, t6 = s * 5.0f;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        float a = fabsf(v[k]);
        uint32_t idx = (uint32_t)(a > t0) + (uint32_t)(a >= t1) + (uint32_t)(a > t2) + (uint32_t)(a >= t3) +
                       (uint32_t)(a > t4) + (uint32_t)(a >= t5) + (uint32_t)(a > t6);
        if (s == 0.0f) idx = 0;
        uint32_t nib = idx | ((__float_as_uint(v[k]) >> 28) & 8u);
        packed |= nib << (4 * k);
      }
    } else {
      set_status(status, CSA2_ERR_NONFINITE);
    }
    *reinterpret_cast<uint32_t*>(jo.codes + orow * (dim / 2) + c8 * 4) = packed;
    if ((c8 & 3) == 0) jo.scales[orow * (dim / 32) + c8 / 4] = sc;
  }
}

// ============================================================================
// Indexer scoring on CUDA cores.  One thread = one position: dequantise the
// key row, s = sum_h w_h * max(0, q_h . k) with q staged in shared memory.
// ============================================================================
template <int DI>
__device__ __forceinline__ void load_key_row(const csa2_fp4_cache& c, int64_t row, float* k) {
  const uint32_t* cw = reinterpret_cast<const uint32_t*>(c.codes + row * (DI / 2));
  const uint8_t* sp = c.scales + row * (DI / 32);
#pragma unroll
  for (int g = 0; g < DI / 32; ++g) {
    float s = e4m3_to_f32(__ldg(sp + g));
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      uint32_t word = __ldg(cw + g * 4 + w);
#pragma unroll
      for (int n = 0; n < 8; ++n) k[g * 32 + w * 8 + n] = e2m1_to_f32(word >> (4 * n)) * s;
    }
  }
}

template <int DI>
__device__ __forceinline__ float score_row(const float* k, const float* qs, const float* ws, int H) {
  float acc = 0.0f;
  for (int h = 0; h < H; ++h) {
    const float* qh = qs + h * DI;
    float dot = 0.0f;
#pragma unroll
    for (int c = 0; c < DI; ++c) dot = fmaf(qh[c], k[c], dot);
    acc = fmaf(ws[h], fmaxf(dot, 0.0f), acc);
  }
  return acc;
}

// stage the dequantised query of token `tok` and its head weights
template <int DI>
__device__ __forceinline__ void stage_query(const uint8_t* q_codes, const uint8_t* q_scales, const float* w, int H,
                                            int tok, float* qs, float* ws) {
  for (int e = threadIdx.x; e < H * DI; e += blockDim.x) {
    int h = e / DI, c = e % DI;
    uint8_t byte = q_codes[((int64_t)tok * H + h) * (DI / 2) + c / 2];
    uint32_t nib = (c & 1) ? (byte >> 4) : (byte & 15);
    qs[e] = e2m1_to_f32(nib) * e4m3_to_f32(q_scales[((int64_t)tok * H + h) * (DI / 32) + c / 32]);
  }
  for (int h = threadIdx.x; h < H; h += blockDim.x) ws[h] = w[(int64_t)tok * H + h];
  __syncthreads();
}

// Full scan: grid (position chunks of 128, T); block scores of every visible block
template <int DI>
__global__ void __launch_bounds__(128) k_scan_simt(csa2_query_batch qb, const uint8_t* __restrict__ q_codes,
                                                   const uint8_t* __restrict__ q_scales, const float* __restrict__ w,
                                                   int H, csa2_fp4_cache kc, float* __restrict__ bscore,
                                                   int64_t ld_bs, int* status) {
  extern __shared__ float sm[];
  float* qs = sm;
  float* ws = sm + H * DI;
  const int tok = blockIdx.y;
  const int b = __ldg(qb.tok_seq + tok);
  const int64_t p = __ldg(qb.tok_pos + tok);
  const int64_t t0 = (int64_t)blockIdx.x * 128;
  if (t0 > p) return;
  stage_query<DI>(q_codes, q_scales, w, H, tok, qs, ws);
  const int64_t t = t0 + threadIdx.x;
  float s = -INFINITY;
  if (t <= p) {
    int64_t row = cache_row(kc, b, t);
    if (row < 0 || row >= kc.n_rows) {
      set_status(status, CSA2_ERR_RANGE);
    } else {
      float k[DI];
      load_key_row<DI>(kc, row, k);
      s = score_row<DI>(k, qs, ws, H);
    }
  }
  s = fmaxf(s, __shfl_xor_sync(0xffffffffu, s, 1));
  s = fmaxf(s, __shfl_xor_sync(0xffffffffu, s, 2));
  s = fmaxf(s, __shfl_xor_sync(0xffffffffu, s, 4));
  if ((threadIdx.x & 7) == 0 && t <= p) bscore[(int64_t)tok * ld_bs + t / kBlock] = s;
}

// Pool rescoring: grid (chunks of 128 pool positions, T); score of pool entry
// i (position pool[i/8]*8 + i%8), -inf where invalid
template <int DI>
__global__ void __launch_bounds__(128) k_rescore_simt(csa2_query_batch qb, const uint8_t* __restrict__ q_codes,
                                                      const uint8_t* __restrict__ q_scales, const float* __restrict__ w,
                                                      int H, csa2_fp4_cache kc, const int32_t* __restrict__ pool,
                                                      const int32_t* __restrict__ pool_n, int P,
                                                      float* __restrict__ scores, int* status) {
  extern __shared__ float sm[];
  float* qs = sm;
  float* ws = sm + H * DI;
  const int tok = blockIdx.y;
  const int b = __ldg(qb.tok_seq + tok);
  const int64_t p = __ldg(qb.tok_pos + tok);
  const int np = min(__ldg(pool_n + tok), P);
  const int i0 = blockIdx.x * 128;
  if (i0 >= np * kBlock) {
    for (int i = i0 + threadIdx.x; i < i0 + 128 && i < P * kBlock; i += blockDim.x)
      scores[(int64_t)tok * P * kBlock + i] = -INFINITY;
    return;
  }
  stage_query<DI>(q_codes, q_scales, w, H, tok, qs, ws);
  const int i = i0 + threadIdx.x;
  float s = -INFINITY;
  if (i < np * kBlock) {
    int32_t blk = __ldg(pool + (int64_t)tok * P + i / kBlock);
    int64_t t = (int64_t)blk * kBlock + (i % kBlock);
    if (blk >= 0 && t <= p) {
      int64_t row = cache_row(kc, b, t);
      if (row < 0 || row >= kc.n_rows) {
        set_status(status, CSA2_ERR_RANGE);
      } else {
        float k[DI];
        load_key_row<DI>(kc, row, k);
        s = score_row<DI>(k, qs, ws, H);
      }
    }
  }
  if (i < P * kBlock) scores[(int64_t)tok * P * kBlock + i] = s;
}

// ============================================================================
// Attention partials on CUDA cores.  Grid (splits, T); each CTA stages up to
// 64 rows of the key set (sparse FP4 rows of the index list, or FP8 window
// rows) dequantised in shared memory, and each warp runs an online softmax for
// its heads; writes (m, l, o~ = sum e^{z-m} v) per (token, split, head).
// ============================================================================
constexpr int kAttRows = 64;

template <int D>
__global__ void __launch_bounds__(256) k_attend_simt(csa2_query_batch qb, const void* __restrict__ q, int q_dtype,
                                                     int Hq, csa2_fp4_cache kv, const int32_t* __restrict__ idx,
                                                     const int32_t* __restrict__ idx_n, int K, csa2_swa_desc swa,
                                                     int n_sparse_split, float scale, float* __restrict__ part_o,
                                                     float* __restrict__ part_ml, int n_split, int* status) {
  extern __shared__ float sm[];
  float* rows = sm;                         // [kAttRows][D]
  int* valid = reinterpret_cast<int*>(sm + kAttRows * D);
  const int tok = blockIdx.y, split = blockIdx.x;
  const int b = __ldg(qb.tok_seq + tok);
  const int64_t p = __ldg(qb.tok_pos + tok);
  const bool is_swa = split >= n_sparse_split;
  // stage rows
  for (int r = threadIdx.x >> 5; r < kAttRows; r += blockDim.x >> 5) {
    const int lane = threadIdx.x & 31;
    bool ok = false;
    if (!is_swa) {
      int j = split * kAttRows + r;
      int n = min(__ldg(idx_n + tok), K);
      if (j < n) {
        int32_t t = __ldg(idx + (int64_t)tok * K + j);
        if (t >= 0 && t <= p) {
          int64_t row = cache_row(kv, b, t);
          if (row >= 0 && row < kv.n_rows) {
            ok = true;
            const uint8_t* cp = kv.codes + row * (D / 2);
            const uint8_t* sp = kv.scales + row * (D / 32);
            for (int c = lane; c < D; c += 32) {
              uint8_t byte = __ldg(cp + c / 2);
              rows[r * D + c] = e2m1_to_f32((c & 1) ? (byte >> 4) : (byte & 15)) * e4m3_to_f32(__ldg(sp + c / 32));
            }
          } else if (lane == 0) {
            set_status(status, CSA2_ERR_RANGE);
          }
        } else if (lane == 0) {
          set_status(status, CSA2_ERR_RANGE);
        }
      }
    } else {
      int64_t lo = p - swa.window + 1;
      if (lo < 0) lo = 0;
      int64_t t = lo + (int64_t)(split - n_sparse_split) * kAttRows + r;
      if (t <= p) {
        ok = true;
        int64_t row = (int64_t)b * swa.cap + t % swa.cap;
        float s = __ldg(swa.scale + row);
        for (int c = lane; c < D; c += 32) rows[r * D + c] = e4m3_to_f32(__ldg(swa.codes + row * D + c)) * s;
      }
    }
    if (lane == 0) valid[r] = ok;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  constexpr int PER = D / 32;
  for (int h = wid; h < Hq; h += nw) {
    float qv[PER];
    const int64_t qoff = ((int64_t)tok * Hq + h) * D;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      int c = lane + 32 * j;
      qv[j] = q_dtype == CSA2_F32 ? __ldg(reinterpret_cast<const float*>(q) + qoff + c)
                                  : __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(q)[qoff + c]);
    }
    float m = -INFINITY, l = 0.0f, o[PER];
#pragma unroll
    for (int j = 0; j < PER; ++j) o[j] = 0.0f;
    for (int r = 0; r < kAttRows; ++r) {
      if (!valid[r]) continue;
      float d = 0.0f;
#pragma unroll
      for (int j = 0; j < PER; ++j) d = fmaf(qv[j], rows[r * D + lane + 32 * j], d);
      float z = warp_sum(d) * scale;
      if (z > m) {
        float a = __expf(m - z);
        l *= a;
#pragma unroll
        for (int j = 0; j < PER; ++j) o[j] *= a;
        m = z;
      }
      float e = __expf(z - m);
      l += e;
#pragma unroll
      for (int j = 0; j < PER; ++j) o[j] = fmaf(e, rows[r * D + lane + 32 * j], o[j]);
    }
    const int64_t pidx = ((int64_t)tok * n_split + split) * Hq + h;
#pragma unroll
    for (int j = 0; j < PER; ++j) part_o[pidx * D + lane + 32 * j] = o[j];
    if (lane == 0) {
      part_ml[pidx * 2] = m;
      part_ml[pidx * 2 + 1] = l;
    }
  }
}

// LSE merge of the split partials: grid (Hq, T), one thread per channel group
__global__ void __launch_bounds__(128) k_merge(const float* __restrict__ part_o, const float* __restrict__ part_ml,
                                               int n_split, int Hq, int D, void* __restrict__ out, int out_dtype,
                                               float* __restrict__ lse) {
  const int h = blockIdx.x, tok = blockIdx.y;
  const int64_t base = (int64_t)tok * n_split * Hq;
  float M = -INFINITY;
  for (int s = 0; s < n_split; ++s) {
    float l = part_ml[((base + (int64_t)s * Hq + h) * 2) + 1];
    if (l > 0.0f) M = fmaxf(M, part_ml[(base + (int64_t)s * Hq + h) * 2]);
  }
  float L = 0.0f;
  for (int s = 0; s < n_split; ++s) {
    const float* ml = part_ml + (base + (int64_t)s * Hq + h) * 2;
    if (ml[1] > 0.0f) L += ml[1] * __expf(ml[0] - M);
  }
  const float inv = L > 0.0f ? 1.0f / L : 0.0f;
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    float acc = 0.0f;
    for (int s = 0; s < n_split; ++s) {
      const float* ml = part_ml + (base + (int64_t)s * Hq + h) * 2;
      if (ml[1] > 0.0f) acc += __expf(ml[0] - M) * part_o[(base + (int64_t)s * Hq + h) * D + c];
    }
    float v = acc * inv;
    const int64_t oi = ((int64_t)tok * Hq + h) * D + c;
    if (out_dtype == CSA2_F32)
      reinterpret_cast<float*>(out)[oi] = v;
    else
      reinterpret_cast<__nv_bfloat16*>(out)[oi] = __float2bfloat16_rn(v);
  }
  if (lse && threadIdx.x == 0) lse[(int64_t)tok * Hq + h] = L > 0.0f ? M + logf(L) : -INFINITY;
}

// copies used by the stack for the optional per-layer outputs
__global__ void k_copy_i32(const int32_t* __restrict__ src, int32_t* __restrict__ dst, int64_t n) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    dst[i] = src[i];
}

// bounded-wait self test: waits on an mbarrier that nothing completes
__global__ void k_selftest_wait(int64_t limit_ns, int* status) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    if (!mbar_wait_bounded(smem_u32(&bar), 0, (uint64_t)limit_ns)) set_status(status, CSA2_ERR_TIMEOUT);
  }
}

}  // namespace csa2
