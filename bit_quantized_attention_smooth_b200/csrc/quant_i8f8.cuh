// Quantisation kernels of the INT8-QK / FP8-PV mode.
//
// The TurboDiffusion explainer (wxsanhe.com post 64219, section 1 "hybrid
// attention") puts QK^T in INT8 and PV in FP8 and recovers accuracy with
// outlier smoothing; the SageAttention tag page (reportify.cn), SageAttention3
// summary, bullet [17], quantises Q/K per block.  Readings used here:
//   mu[c]   = (float)( sum_n K[n,c] (exact float64 sum) / N )      per (b,h)
//   s_q, s_k = max|x| / 127 per 128-token block (1 for an all-zero block);
//             optionally s_q per token (max over the token's channels)
//   q8      = RNE(x / s) clamped to [-127, 127], division in IEEE float32
//   s_v[c]  = max_n |V[n,c]| / 448 per channel (1 for an all-zero channel)
//   v8      = E4M3_RNE_satfinite(V / s_v), written transposed [d, Nv]
//
// NaN inputs: every maximum above propagates NaN (fmax_nan), so a NaN makes
// the scale it feeds NaN: a Q block's (or token's) rows, a K channel's mean
// (and with it every K scale of the head), a V channel's scale.
//
// HBM-bound.  Pass 1 (kv_stats) reads K and V once and reduces per-channel
// sums in float64 atomics and per-channel |V| maxima.  Each bf16/fp16 value is
// exact in float64, and so is every partial sum while the sum's magnitude
// stays below 2^53 times the smallest quantum among the summands (true for
// the workloads here: values above 2^-30 in magnitude, sums below 2^21), so
// the mean does not depend on the order of the atomics; a head holding values
// as small as fp16/bf16 subnormals next to sums near 2^30 can differ in the
// mean's last bit between runs.  Pass 2 reads Q, K, V once more and writes
// the codes; every load is a coalesced 16-byte vector.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ptx.cuh"

namespace sattn {

constexpr int kBlockTokens = 128;   // quantisation block = attention tile height
constexpr int kQuantThreads = 256;
// Threads of the per-block quantizers: a block of 128 tokens is spread over
// 512 threads so that each holds few values and an SM keeps more loads in flight.
constexpr int kBlockQuantThreads = 512;

template <typename T>
__device__ __forceinline__ void load8(const T *p, float (&f)[8]);

template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16 *p, float (&f)[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[i]));
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

template <>
__device__ __forceinline__ void load8<__half>(const __half *p, float (&f)[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __half22float2(*reinterpret_cast<const __half2 *>(&w[i]));
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

// Pass 1: per-channel float64 sums of K and float32 maxima of |V|.
// grid (ceil(N / tokens_per_cta), B*H), block 256.
template <typename T, int D>
__global__ void __launch_bounds__(kQuantThreads) kv_stats_kernel(const T *__restrict__ k, const T *__restrict__ v,
                                                                 double *__restrict__ ksum,
                                                                 unsigned *__restrict__ vmax, int N,
                                                                 int tokens_per_cta) {
  constexpr int LPR = D / 8;                  // threads per row (8 channels each)
  constexpr int RPI = kQuantThreads / LPR;    // rows per iteration
  __shared__ double s_sum[RPI][D];
  __shared__ float s_max[RPI][D];

  const int bh = blockIdx.y;
  const int cg = threadIdx.x % LPR;
  const int r0 = threadIdx.x / LPR;
  const int n_begin = blockIdx.x * tokens_per_cta;
  const int n_end = min(N, n_begin + tokens_per_cta);
  const size_t head = static_cast<size_t>(bh) * N * D;

  double acc[8];
  float vm[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    acc[i] = 0.0;
    vm[i] = 0.f;
  }
#pragma unroll 4
  for (int n = n_begin + r0; n < n_end; n += RPI) {
    float kf[8], vf[8];
    load8<T>(k + head + static_cast<size_t>(n) * D + cg * 8, kf);
    load8<T>(v + head + static_cast<size_t>(n) * D + cg * 8, vf);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      acc[i] += static_cast<double>(kf[i]);
      vm[i] = fmax_nan(vm[i], fabsf(vf[i]));
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    s_sum[r0][cg * 8 + i] = acc[i];
    s_max[r0][cg * 8 + i] = vm[i];
  }
  __syncthreads();
  if (threadIdx.x < D) {
    const int c = threadIdx.x;
    double s = 0.0;
    float m = 0.f;
    for (int r = 0; r < RPI; ++r) {
      s += s_sum[r][c];
      m = fmax_nan(m, s_max[r][c]);
    }
    atomicAdd(ksum + static_cast<size_t>(bh) * D + c, s);
    atomicMax(vmax + static_cast<size_t>(bh) * D + c, __float_as_uint(m));  // m >= 0: bit order = value order
  }
}

template <int NT>
__device__ __forceinline__ float block_max(float v, float *s_red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmax_nan(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int warp = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) s_red[warp] = v;
  __syncthreads();
  float m = s_red[0];
#pragma unroll
  for (int w = 1; w < NT / 32; ++w) m = fmax_nan(m, s_red[w]);
  return m;
}

// Pass 2a: per-block INT8 of Q (IS_K = false) or of K - mu (IS_K = true).
// grid (ceil(N/128), B*H), block kBlockQuantThreads.  Each thread owns a
// fixed group of 8 channels and (128 * D / 8) / kBlockQuantThreads row positions.
template <typename T, int D, bool IS_K>
__global__ void __launch_bounds__(kBlockQuantThreads, 2) quant_qk_kernel(const T *__restrict__ x, int8_t *__restrict__ out,
                                                                 float *__restrict__ scale,
                                                                 const double *__restrict__ ksum,
                                                                 float *__restrict__ mu_out, int N, int nblk) {
  constexpr int LPR = D / 8;
  constexpr int RPI = kBlockQuantThreads / LPR;
  constexpr int ITERS = kBlockTokens / RPI;
  __shared__ float s_red[kBlockQuantThreads / 32];

  const int bh = blockIdx.y;
  const int blk = blockIdx.x;
  const int cg = threadIdx.x % LPR;
  const int r0 = threadIdx.x / LPR;
  const size_t head = static_cast<size_t>(bh) * N * D;

  // every load first, so that the mean's float64 division below overlaps them
  float val[ITERS][8];
#pragma unroll
  for (int it = 0; it < ITERS; ++it) {
    const int n = blk * kBlockTokens + it * RPI + r0;
    if (n < N) {
      load8<T>(x + head + static_cast<size_t>(n) * D + cg * 8, val[it]);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) val[it][i] = 0.f;
    }
  }
  float amax = 0.f;
  if (IS_K) {
    float mu[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      mu[i] = static_cast<float>(ksum[static_cast<size_t>(bh) * D + cg * 8 + i] / static_cast<double>(N));
    if (blk == 0 && r0 == 0) {
#pragma unroll
      for (int i = 0; i < 8; ++i) mu_out[static_cast<size_t>(bh) * D + cg * 8 + i] = mu[i];
    }
#pragma unroll
    for (int it = 0; it < ITERS; ++it) {
      const bool valid = blk * kBlockTokens + it * RPI + r0 < N;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        val[it][i] = valid ? __fsub_rn(val[it][i], mu[i]) : 0.f;
        amax = fmax_nan(amax, fabsf(val[it][i]));
      }
    }
  } else {
#pragma unroll
    for (int it = 0; it < ITERS; ++it)
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmax_nan(amax, fabsf(val[it][i]));
  }
  amax = block_max<kBlockQuantThreads>(amax, s_red);
  const float s = amax == 0.f ? 1.f : __fdiv_rn(amax, 127.f);
  if (threadIdx.x == 0) scale[static_cast<size_t>(bh) * nblk + blk] = s;

#pragma unroll
  for (int it = 0; it < ITERS; ++it) {
    const int n = blk * kBlockTokens + it * RPI + r0;
    if (n < N) {
      uint32_t w[2] = {0u, 0u};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        int qi = __float2int_rn(__fdiv_rn(val[it][i], s));
        qi = max(-127, min(127, qi));
        w[i >> 2] |= (static_cast<uint32_t>(qi) & 0xFFu) << (8 * (i & 3));
      }
      *reinterpret_cast<uint2 *>(out + head + static_cast<size_t>(n) * D + cg * 8) = make_uint2(w[0], w[1]);
    }
  }
}

// Pass 2a, per-token variant: INT8 of Q with one scale per token ("thread-level"
// granularity: the attention kernel gives each query row its own thread), s =
// max|x[n, :]| / 127.  grid (ceil(N / kTokRows), B*H), block kQuantThreads;
// D/8 consecutive lanes share a token (8 channels each) and every thread takes
// kTokIters tokens, loaded before any is reduced.
constexpr int kTokIters = 4;
template <int D>
__host__ __device__ constexpr int tok_rows_per_cta() { return kQuantThreads / (D / 8) * kTokIters; }

template <typename T, int D>
__global__ void __launch_bounds__(kQuantThreads) quant_q_token_kernel(const T *__restrict__ x, int8_t *__restrict__ out,
                                                                      float *__restrict__ scale, int N) {
  constexpr int LPR = D / 8;                  // lanes per token (16 or 8); divides 32
  constexpr int RPI = kQuantThreads / LPR;    // tokens per iteration of the CTA
  const int bh = blockIdx.y;
  const int cg = threadIdx.x % LPR;
  const size_t head = static_cast<size_t>(bh) * N * D;
  const int n0 = blockIdx.x * tok_rows_per_cta<D>() + threadIdx.x / LPR;
  float val[kTokIters][8];
#pragma unroll
  for (int it = 0; it < kTokIters; ++it) {
    const int n = n0 + it * RPI;
    if (n < N) {
      load8<T>(x + head + static_cast<size_t>(n) * D + cg * 8, val[it]);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) val[it][i] = 0.f;
    }
  }
#pragma unroll
  for (int it = 0; it < kTokIters; ++it) {
    const int n = n0 + it * RPI;
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmax_nan(amax, fabsf(val[it][i]));
    // every lane of the warp takes part (tokens past N hold zeros)
#pragma unroll
    for (int o = LPR / 2; o > 0; o >>= 1) amax = fmax_nan(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float s = amax == 0.f ? 1.f : __fdiv_rn(amax, 127.f);
    if (n < N) {
      if (cg == 0) scale[static_cast<size_t>(bh) * N + n] = s;
      uint32_t w[2] = {0u, 0u};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        int qi = __float2int_rn(__fdiv_rn(val[it][i], s));
        qi = max(-127, min(127, qi));
        w[i >> 2] |= (static_cast<uint32_t>(qi) & 0xFFu) << (8 * (i & 3));
      }
      *reinterpret_cast<uint2 *>(out + head + static_cast<size_t>(n) * D + cg * 8) = make_uint2(w[0], w[1]);
    }
  }
}

// Pass 2b: per-channel FP8 E4M3 of V, stored transposed vt[bh][c][token]
// with row length Nv (N rounded up to 16).  grid (ceil(N/128), B*H), block
// 4 D threads.  Thread t takes the 4 tokens 4 (t mod 32) .. + 3 of the block
// and the 8 channels of group t / 32, packs the 4 codes of each channel into one word
// (lowest token in the low byte), and the block is written out row by row:
// every shared-memory access of a warp touches 32 consecutive words and every
// global store is a full 128-byte row segment.
template <typename T, int D>
__global__ void __launch_bounds__(4 * D, 2) quant_v_kernel(const T *__restrict__ v, uint8_t *__restrict__ vt,
                                                                float *__restrict__ sv_out,
                                                                const unsigned *__restrict__ vmax, int N,
                                                                int Nv) {
  constexpr int CPT = 8;                     // channels per thread
  constexpr int NT = 4 * D;                  // threads
  constexpr int WPR = kBlockTokens / 4;      // words per channel row of the block (32)
  __shared__ uint32_t tile[D][WPR];

  const int bh = blockIdx.y;
  const int blk = blockIdx.x;
  const int tq = threadIdx.x % WPR;          // token quad
  const int c0 = (threadIdx.x / WPR) * CPT;  // first channel of this thread
  const size_t head = static_cast<size_t>(bh) * N * D;

  float sv[CPT];
#pragma unroll
  for (int i = 0; i < CPT; ++i) {
    const float m = __uint_as_float(vmax[static_cast<size_t>(bh) * D + c0 + i]);
    sv[i] = m == 0.f ? 1.f : __fdiv_rn(m, 448.f);
  }
  if (blk == 0 && tq == 0) {
#pragma unroll
    for (int i = 0; i < CPT; ++i) sv_out[static_cast<size_t>(bh) * D + c0 + i] = sv[i];
  }

  float f[4][CPT];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int n = blk * kBlockTokens + 4 * tq + r;
#pragma unroll
    for (int g = 0; g < CPT; g += 8) {
      float t8[8];
      if (n < N) {
        load8<T>(v + head + static_cast<size_t>(n) * D + c0 + g, t8);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) t8[i] = 0.f;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) f[r][g + i] = t8[i];
    }
  }
#pragma unroll
  for (int i = 0; i < CPT; ++i) {
    const uint32_t lo = cvt_e4m3x2(__fdiv_rn(f[0][i], sv[i]), __fdiv_rn(f[1][i], sv[i]));
    const uint32_t hi = cvt_e4m3x2(__fdiv_rn(f[2][i], sv[i]), __fdiv_rn(f[3][i], sv[i]));
    tile[c0 + i][tq] = lo | (hi << 16);
  }
  __syncthreads();
  const int tok0 = blk * kBlockTokens;
  const int valid_words = min(kBlockTokens, Nv - tok0) / 4;
  for (int idx = threadIdx.x; idx < D * WPR; idx += NT) {
    const int c = idx / WPR;
    const int w = idx % WPR;
    if (w < valid_words)
      *reinterpret_cast<uint32_t *>(vt + (static_cast<size_t>(bh) * D + c) * Nv + tok0 + 4 * w) = tile[c][w];
  }
}

}  // namespace sattn
