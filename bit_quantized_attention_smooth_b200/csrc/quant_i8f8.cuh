// Quantisation of the INT8-QK / FP8-PV mode: the per-tile work of the fused
// quantiser (quant_fused.cuh schedules it).
//
// The TurboDiffusion explainer (wxsanhe.com post 64219, section 1 "hybrid
// attention") puts QK^T in INT8 and PV in FP8 and recovers accuracy with
// outlier smoothing; the SageAttention tag page (reportify.cn), SageAttention3
// summary, bullet [17], quantises Q/K per block.  Readings used here:
//   mu[c]   = (float)( sum_n K[n,c] (float64 sum) / N )      per (b,h)
//   s_q, s_k = max|x| / 127 per 128-token block (1 for an all-zero block);
//             optionally s_q per token (max over the token's channels)
//   q8      = RNE(x / s) clamped to [-127, 127], x / s the IEEE float32 quotient
//   s_v[c]  = max_n |V[n,c]| / 448 per channel (1 for an all-zero channel)
//   v8      = E4M3_RNE_satfinite(V / s_v), written transposed [d, Nv]
//
// NaN inputs: every maximum above propagates NaN (fmax_nan), so a NaN makes
// the scale it feeds NaN: a Q block's (or token's) rows, a K channel's mean
// (and with it every K scale of the head), a V channel's scale.
//
// A "tile" is 128 tokens x d channels of one tensor of one (b,h), staged in
// shared memory row-major by a bulk copy; rows at and past `rows` are stale
// and never read as data.  The 256 compute threads of a CTA take part in each
// tile; every warp arrives once on the stage's `empty` barrier after its last
// read of the tile.
//
// Statistics tiles add float64 column sums of K and float32 column maxima of
// |V| into per-head accumulators with atomics.  Each bf16/fp16 value is exact
// in float64, and so is every partial sum while the sum's magnitude stays
// below 2^53 times the smallest quantum among the summands (true for the
// workloads here: values above 2^-30 in magnitude, sums below 2^21), so the
// mean does not depend on the order of the atomics; a head holding values as
// small as fp16/bf16 subnormals next to sums near 2^30 can differ in the
// mean's last bit between runs.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <type_traits>

#include "ptx.cuh"

namespace sattn {

constexpr int kBlockTokens = 128;      // quantisation block = attention tile height
constexpr int kQuantConsumers = 256;   // compute threads of a quantiser CTA (8 warps)
constexpr int kQuantWarps = kQuantConsumers / 32;
constexpr int kQuantBar = 1;           // named barrier of the compute threads

// Shared scratch of the compute threads.
template <int D>
struct QuantScratch {
  union {
    double sum[kQuantWarps][D];        // per-warp partial column sums of a K tile
    float max[kQuantWarps][D];         // per-warp partial column maxima of a V tile
  } red;
  float red_max[kQuantWarps];          // per-warp maxima of a quantisation block
  float row_scale[kBlockTokens];       // per-token Q scales of the tile (its rare exact path)
  float2 e4m3_recip[256];              // NVFP4: bracket multipliers of 1/scale per E4M3 scale code
};

// 8 values (one 16-byte word) -> float, exact.
template <typename T>
__device__ __forceinline__ void cvt8(const uint4 &u, float (&f)[8]);

template <>
__device__ __forceinline__ void cvt8<__nv_bfloat16>(const uint4 &u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

template <>
__device__ __forceinline__ void cvt8<__half>(const uint4 &u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __half22float2(*reinterpret_cast<const __half2 *>(&w[i]));
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

// Value i (0..7) of one 16-byte word of T -> float, exact.
template <typename T>
__device__ __forceinline__ float elem8(const uint4 &u, int i) {
  const uint32_t w = i < 2 ? u.x : i < 4 ? u.y : i < 6 ? u.z : u.w;
  if (std::is_same<T, __nv_bfloat16>::value) return __uint_as_float((i & 1) ? (w & 0xFFFF0000u) : (w << 16));
  const __half2 h = *reinterpret_cast<const __half2 *>(&w);
  return (i & 1) ? __high2float(h) : __low2float(h);
}

// 8 consecutive values of a shared-memory tile (16-byte aligned) -> float.
template <typename T>
__device__ __forceinline__ void lds8(const T *p, float (&f)[8]) {
  cvt8<T>(*reinterpret_cast<const uint4 *>(p), f);
}

// Lane-wise operations on two packed values of T (exact: maxima and minima
// of representable values are representable), NaN-propagating.
template <typename T>
struct Packed;
template <>
struct Packed<__nv_bfloat16> {
  using P = __nv_bfloat162;
  static constexpr uint32_t kNegInf = 0xFF80FF80u, kPosInf = 0x7F807F80u;
};
template <>
struct Packed<__half> {
  using P = __half2;
  static constexpr uint32_t kNegInf = 0xFC00FC00u, kPosInf = 0x7C007C00u;
};
template <typename T>
__device__ __forceinline__ uint32_t absmax2(uint32_t acc, uint32_t w) {   // max(acc, |w|)
  using P = typename Packed<T>::P;
  const P r = __hmax2_nan(*reinterpret_cast<const P *>(&acc), __habs2(*reinterpret_cast<const P *>(&w)));
  return *reinterpret_cast<const uint32_t *>(&r);
}
template <typename T>
__device__ __forceinline__ uint32_t max2(uint32_t a, uint32_t b) {
  using P = typename Packed<T>::P;
  const P r = __hmax2_nan(*reinterpret_cast<const P *>(&a), *reinterpret_cast<const P *>(&b));
  return *reinterpret_cast<const uint32_t *>(&r);
}
template <typename T>
__device__ __forceinline__ uint32_t min2(uint32_t a, uint32_t b) {
  using P = typename Packed<T>::P;
  const P r = __hmin2_nan(*reinterpret_cast<const P *>(&a), *reinterpret_cast<const P *>(&b));
  return *reinterpret_cast<const uint32_t *>(&r);
}
// Both values of a packed pair as floats.
template <typename T>
__device__ __forceinline__ float2 unpack2(uint32_t w) {
  const uint4 u = make_uint4(w, 0u, 0u, 0u);
  return make_float2(elem8<T>(u, 0), elem8<T>(u, 1));
}

__device__ __forceinline__ float fmax3_nan(float a, float b, float c) {
  float d;
  asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ void release_stage(uint64_t *empty) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(empty);
}

// This thread's rows of a tile, loaded into registers before any arithmetic
// (so that the rows can be processed with full instruction-level
// parallelism): row r0 + p (256 / (d/8)), channels 8 cg .. + 7, zeros for
// rows at and past `rows`.
template <typename T, int D>
constexpr int kRowPasses = kBlockTokens * D / (8 * kQuantConsumers);

template <typename T, int D>
__device__ __forceinline__ void load_rows(const T *tile, int rows, int r0, int cg, uint4 (&u)[kRowPasses<T, D>]) {
  constexpr int RPP = kQuantConsumers / (D / 8);
#pragma unroll
  for (int p = 0; p < kRowPasses<T, D>; ++p) {
    const int r = r0 + p * RPP;
    u[p] = r < rows ? *reinterpret_cast<const uint4 *>(tile + r * D + cg * 8) : make_uint4(0u, 0u, 0u, 0u);
  }
}

// The same rows, with row 0 (always valid) standing in for rows at and past
// `rows`: a copy of valid data changes no maximum or minimum.
template <typename T, int D>
__device__ __forceinline__ void load_rows_dup(const T *tile, int rows, int r0, int cg, uint4 (&u)[kRowPasses<T, D>]) {
  constexpr int RPP = kQuantConsumers / (D / 8);
#pragma unroll
  for (int p = 0; p < kRowPasses<T, D>; ++p) {
    const int r = r0 + p * RPP;
    u[p] = *reinterpret_cast<const uint4 *>(tile + (r < rows ? r : 0) * D + cg * 8);
  }
}

// One tile of a statistics item (several consecutive 128-token blocks of one
// tensor of one head): per-channel sums of K (IS_V = false) or maxima of |V|
// (IS_V = true) over the tile's rows (zero rows past `rows` change neither),
// reduced within each warp and kept per warp in sc.red (first = the item's
// first tile: overwrite, else accumulate).  Thread ct takes the 8 channels
// 8 (ct mod d/8) .. + 7 of every (256 / (d/8))-th row; each (warp, channel)
// slot has one writer.
template <typename T, int D, bool IS_V>
__device__ __forceinline__ void stat_tile(const T *tile, int rows, bool first, QuantScratch<D> &sc,
                                          uint64_t *empty) {
  constexpr int LPR = D / 8;
  constexpr int PASSES = kRowPasses<T, D>;
  const int ct = threadIdx.x;
  const int lane = ct & 31;
  const int warp = ct >> 5;
  const int cg = ct % LPR;
  uint4 u[PASSES];
  load_rows<T, D>(tile, rows, ct / LPR, cg, u);
  release_stage(empty);
  if (IS_V) {
    uint32_t vm[4] = {0u, 0u, 0u, 0u};             // packed max |V| of the 8 channels
#pragma unroll
    for (int p = 0; p < PASSES; ++p) {
      vm[0] = absmax2<T>(vm[0], u[p].x);
      vm[1] = absmax2<T>(vm[1], u[p].y);
      vm[2] = absmax2<T>(vm[2], u[p].z);
      vm[3] = absmax2<T>(vm[3], u[p].w);
    }
    float m[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 t = unpack2<T>(vm[i]);
      m[2 * i] = t.x;
      m[2 * i + 1] = t.y;
    }
#pragma unroll
    for (int o = LPR; o < 32; o <<= 1)
#pragma unroll
      for (int i = 0; i < 8; ++i) m[i] = fmax_nan(m[i], __shfl_xor_sync(0xffffffffu, m[i], o));
    if (lane < LPR) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float &slot = sc.red.max[warp][cg * 8 + i];
        slot = first ? m[i] : fmax_nan(slot, m[i]);
      }
    }
  } else {
    double acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0;
#pragma unroll
    for (int p = 0; p < PASSES; ++p) {
      float f[8];
      cvt8<T>(u[p], f);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += static_cast<double>(f[i]);
    }
#pragma unroll
    for (int o = LPR; o < 32; o <<= 1)
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
    if (lane < LPR) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        double &slot = sc.red.sum[warp][cg * 8 + i];
        slot = first ? acc[i] : slot + acc[i];
      }
    }
  }
}

// End of a statistics item: the per-warp slots are summed (maximised) over
// the CTA and added into the head's accumulator (ksum_h or vmax_h, d
// entries) by threads ct < d; each of their warps then fences its atomics
// and bumps *done_h once (a warp-level publication: no barrier across warps).
template <int D, bool IS_V>
__device__ __forceinline__ void stat_publish(QuantScratch<D> &sc, double *ksum_h, unsigned *vmax_h,
                                             unsigned *done_h) {
  const int ct = threadIdx.x;
  named_bar_sync(kQuantBar, kQuantConsumers);
  if (ct < D) {
    if (IS_V) {
      float m = sc.red.max[0][ct];
#pragma unroll
      for (int w = 1; w < kQuantWarps; ++w) m = fmax_nan(m, sc.red.max[w][ct]);
      atomicMax(vmax_h + ct, __float_as_uint(m));   // m >= 0 or NaN: bit order = value order
    } else {
      double s = sc.red.sum[0][ct];
#pragma unroll
      for (int w = 1; w < kQuantWarps; ++w) s += sc.red.sum[w][ct];
      atomicAdd(ksum_h + ct, s);
    }
    __threadfence();
    __syncwarp();                                   // d is a multiple of 32: whole warps
    if ((ct & 31) == 0) {
      __threadfence();
      atomicAdd(done_h, 1u);
    }
  }
}

// INT8 codes RNE(x / s) (s > 0 finite, r = 1/s correctly rounded, the IEEE
// float32 quotient being the reference) of 8 values, packed lowest index in
// the lowest byte, by the product x * r: for |x / s| <= 128, x * r lies within
// 2.5e-5 of the exact quotient and the IEEE quotient within 7.7e-6, so both
// round to the same integer unless x * r is within 1e-4 of a half-integer.
// Returns false in that case (the caller then takes int8_codes8_exact).  The
// rounding adds 1.5 * 2^23, which puts RNE(y) in the low mantissa bits (exact
// for |y| < 2^22): the code byte is the low byte of the sum's bit pattern.
__device__ __forceinline__ bool int8_codes8_fast(const float (&x)[8], float r, uint2 &codes) {
  constexpr float kRound = 12582912.0f;            // 1.5 * 2^23
  const float2 r2 = make_float2(r, r);
  const float2 k2 = make_float2(kRound, kRound);
  const float2 m1 = make_float2(-1.f, -1.f);
  uint32_t c[8];
  float worst = 0.f;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 y = fmul2(make_float2(x[2 * j], x[2 * j + 1]), r2);
    const float2 m = fadd2(y, k2);
    const float2 t = fadd2(y, ffma2(m, m1, k2));  // y - RNE(y), exact
    worst = fmax3(worst, fabsf(t.x), fabsf(t.y));
    c[2 * j] = __float_as_uint(m.x);
    c[2 * j + 1] = __float_as_uint(m.y);
  }
  codes = make_uint2(__byte_perm(__byte_perm(c[0], c[1], 0x0040), __byte_perm(c[2], c[3], 0x0040), 0x5410),
                     __byte_perm(__byte_perm(c[4], c[5], 0x0040), __byte_perm(c[6], c[7], 0x0040), 0x5410));
  return worst <= 0.4999f;
}

// The same codes through the IEEE quotient (near ties, and scales whose
// reciprocal is not a positive normal number); a NaN quotient gives code 0.
__device__ __forceinline__ uint2 int8_codes8_exact(const float (&x)[8], float s) {
  uint32_t w[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    int qi = __float2int_rn(__fdiv_rn(x[i], s));
    qi = max(-127, min(127, qi));
    w[i >> 2] |= (static_cast<uint32_t>(qi) & 0xFFu) << (8 * (i & 3));
  }
  return make_uint2(w[0], w[1]);
}

__device__ __forceinline__ bool fast_reciprocal(float r) { return r > 0.f && r < 3.0e38f; }

// Per-block INT8 of a Q tile (IS_K = false) or of K - mu (IS_K = true, mu =
// the stage's per-channel values): one scale for the tile's valid rows, codes
// into out_blk (row r at out_blk + r d), the scale into *scale_slot.  The
// block maximum is taken on the packed inputs: max |x| for Q, and for K
// max(RN(max x - mu), RN(mu - min x)) per channel, which equals the maximum
// of |RN(x - mu)| because rounding is monotone.
template <typename T, int D, bool IS_K>
__device__ __forceinline__ void qk_block_tile(const T *tile, int rows, const float *mu_s, QuantScratch<D> &sc,
                                              int8_t *out_blk, float *scale_slot, uint64_t *empty) {
  constexpr int LPR = D / 8;
  constexpr int RPP = kQuantConsumers / LPR;
  constexpr int PASSES = kRowPasses<T, D>;
  const int ct = threadIdx.x;
  const int lane = ct & 31;
  const int warp = ct >> 5;
  const int cg = ct % LPR;
  const int r0 = ct / LPR;
  float nmu[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) nmu[i] = IS_K ? -mu_s[cg * 8 + i] : 0.f;
  uint4 u[PASSES];
  load_rows_dup<T, D>(tile, rows, r0, cg, u);      // rows past `rows`: copies of row 0 (codes not stored)

  const uint32_t w0[4] = {u[0].x, u[0].y, u[0].z, u[0].w};
  uint32_t hi[4], lo[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    hi[i] = IS_K ? w0[i] : 0u;
    lo[i] = w0[i];
  }
#pragma unroll
  for (int p = 0; p < PASSES; ++p) {
    const uint32_t w[4] = {u[p].x, u[p].y, u[p].z, u[p].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (IS_K) {
        hi[i] = max2<T>(hi[i], w[i]);
        lo[i] = min2<T>(lo[i], w[i]);
      } else {
        hi[i] = absmax2<T>(hi[i], w[i]);
      }
    }
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 h = unpack2<T>(hi[i]);
    if (IS_K) {
      const float2 l = unpack2<T>(lo[i]);
      amax = fmax3_nan(amax, __fadd_rn(h.x, nmu[2 * i]), __fsub_rn(-nmu[2 * i], l.x));
      amax = fmax3_nan(amax, __fadd_rn(h.y, nmu[2 * i + 1]), __fsub_rn(-nmu[2 * i + 1], l.y));
    } else {
      amax = fmax3_nan(amax, h.x, h.y);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmax_nan(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (lane == 0) sc.red_max[warp] = amax;
  named_bar_sync(kQuantBar, kQuantConsumers);
  amax = sc.red_max[0];
#pragma unroll
  for (int w = 1; w < kQuantWarps; ++w) amax = fmax_nan(amax, sc.red_max[w]);
  const float s = amax == 0.f ? 1.f : __fdiv_rn(amax, 127.f);
  const float rcp = __frcp_rn(s);
  if (ct == 0) *scale_slot = s;

  unsigned redo = fast_reciprocal(rcp) ? 0u : (1u << PASSES) - 1u;
#pragma unroll
  for (int p = 0; p < PASSES; ++p) {
    float f[8];
    cvt8<T>(u[p], f);
    if (IS_K) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 d = fadd2(make_float2(f[2 * j], f[2 * j + 1]), make_float2(nmu[2 * j], nmu[2 * j + 1]));
        f[2 * j] = d.x;
        f[2 * j + 1] = d.y;
      }
    }
    uint2 codes;
    if (!int8_codes8_fast(f, rcp, codes)) redo |= 1u << p;
    const int r = r0 + p * RPP;
    if (r < rows) __stcs(reinterpret_cast<uint2 *>(out_blk + r * D + cg * 8), codes);
  }
  // rare: rows near a rounding tie again, through the IEEE quotient (from the stage)
  for (; redo != 0u; redo &= redo - 1u) {
    const int r = r0 + (__ffs(redo) - 1) * RPP;
    if (r >= rows) continue;
    float f[8];
    lds8<T>(tile + r * D + cg * 8, f);
    if (IS_K) {
#pragma unroll
      for (int i = 0; i < 8; ++i) f[i] = __fadd_rn(f[i], nmu[i]);
    }
    *reinterpret_cast<uint2 *>(out_blk + r * D + cg * 8) = int8_codes8_exact(f, s);
  }
  release_stage(empty);
}

// Per-token INT8 of a Q tile ("thread-level" granularity: the attention
// kernel gives each query row its own thread): s = max|x[n, :]| / 127 for
// every valid row, into scale_blk[r].  The d/8 lanes of a row reduce its
// maximum with shuffles; every lane takes part (rows past `rows` hold zeros).
template <typename T, int D>
__device__ __forceinline__ void q_token_tile(const T *tile, int rows, QuantScratch<D> &sc, int8_t *out_blk,
                                             float *scale_blk, uint64_t *empty) {
  constexpr int LPR = D / 8;
  constexpr int RPP = kQuantConsumers / LPR;
  constexpr int PASSES = kRowPasses<T, D>;
  const int ct = threadIdx.x;
  const int cg = ct % LPR;
  const int r0 = ct / LPR;
  uint4 u[PASSES];
  load_rows<T, D>(tile, rows, r0, cg, u);
  unsigned redo = 0u;
#pragma unroll
  for (int p = 0; p < PASSES; ++p) {
    const float2 mf = unpack2<T>(absmax2<T>(absmax2<T>(absmax2<T>(absmax2<T>(0u, u[p].x), u[p].y), u[p].z), u[p].w));
    float amax = fmax_nan(mf.x, mf.y);
#pragma unroll
    for (int o = LPR / 2; o > 0; o >>= 1) amax = fmax_nan(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float s = amax == 0.f ? 1.f : __fdiv_rn(amax, 127.f);
    const float rcp = __frcp_rn(s);
    float f[8];
    cvt8<T>(u[p], f);
    uint2 codes;
    if (!int8_codes8_fast(f, rcp, codes) || !fast_reciprocal(rcp)) redo |= 1u << p;
    const int r = r0 + p * RPP;
    if (cg == 0) sc.row_scale[r] = s;
    if (r < rows) {
      if (cg == 0) scale_blk[r] = s;
      __stcs(reinterpret_cast<uint2 *>(out_blk + r * D + cg * 8), codes);
    }
  }
  __syncwarp();                                    // a row's lanes share a warp: its scale is visible
  // rare: rows near a rounding tie again, through the IEEE quotient (from the stage)
  for (; redo != 0u; redo &= redo - 1u) {
    const int r = r0 + (__ffs(redo) - 1) * RPP;
    if (r >= rows) continue;
    float f[8];
    lds8<T>(tile + r * D + cg * 8, f);
    *reinterpret_cast<uint2 *>(out_blk + r * D + cg * 8) = int8_codes8_exact(f, sc.row_scale[r]);
  }
  release_stage(empty);
}

// The bracket multipliers of a divisor: rlo = RN(r (1 - 2^-20)), rhi =
// RN(r (1 + 2^-20)), r = RN(1/sv).  For any x, the products x rlo and x rhi
// bracket both the exact quotient x / sv and its float32 rounding (their
// relative error is below 2^-22), and rounding to a narrower format is
// monotone: when the two ends give the same code, that is the quotient's
// code.  False when r is not a positive normal number below 1e38.
__device__ __forceinline__ bool bracket(float sv, float &rlo, float &rhi) {
  const float r = __frcp_rn(sv);
  rlo = r * 0.99999904632568359375f;               // 1 - 2^-20
  rhi = r * 1.00000095367431640625f;               // 1 + 2^-20
  return r > 1.2e-38f && r < 1.0e38f;
}

// E4M3 codes of 4 values of one channel by the bracket: returns the codes of
// the upper end; sets bit j of `bad` where value j's two ends round apart
// (the quotient then lies next to a rounding boundary, typically exactly on
// it: bf16 values over a scale with few significant bits often land on an
// E4M3 midpoint).
__device__ __forceinline__ uint32_t e4m3_codes4_fast(const float (&x)[4], float rlo, float rhi, unsigned &bad) {
  const float2 a = make_float2(x[0], x[1]);
  const float2 b = make_float2(x[2], x[3]);
  const float2 alo = fmul2(a, make_float2(rlo, rlo));
  const float2 blo = fmul2(b, make_float2(rlo, rlo));
  const float2 ahi = fmul2(a, make_float2(rhi, rhi));
  const float2 bhi = fmul2(b, make_float2(rhi, rhi));
  const uint32_t clo = cvt_e4m3x4(alo, blo);
  const uint32_t chi = cvt_e4m3x4(ahi, bhi);
  const uint32_t d = clo ^ chi;
  bad = ((d & 0xFFu) != 0u) | (((d >> 8) & 0xFFu) != 0u) << 1 | (((d >> 16) & 0xFFu) != 0u) << 2 |
        ((d >> 24) != 0u) << 3;
  return chi;
}

template <int G>
__device__ __forceinline__ void store_codes(uint8_t *dst, const uint32_t (&w)[G]) {
  if (G == 2)
    __stcs(reinterpret_cast<uint2 *>(dst), make_uint2(w[0], w[G - 1]));
  else
    __stcs(reinterpret_cast<unsigned int *>(dst), w[0]);
}

// Per-channel FP8 E4M3 of a V tile (the stage's per-channel values: s_v in
// sv_s[0 .. d), the bracket multipliers of s_v in sv_s[d .. 2d) and [2d ..
// 3d), 0 where 1/s_v has no safe bracket),
// written transposed into vt_h[c * Nv + tok0 + t] for the tile's tokens below
// Nv (tokens at and past N get code 0).  Warp w takes 4 TPT tokens of 64
// channels; lane l the 8 channels 8 (l mod 8) .. + 7 of that half and the TPT
// tokens TPT (l / 8) ..; it packs the TPT codes of each channel (lowest token
// in the lowest byte) and stores them with one vector store, so that the four
// lanes of a channel write 4 TPT consecutive bytes.
template <typename T, int D>
__device__ __forceinline__ void v_tile(const T *tile, int rows, int tok0, int Nv, const float *sv_s, uint8_t *vt_h,
                                       uint64_t *empty) {
  constexpr int TPT = D == 128 ? 8 : 4;            // tokens per thread
  constexpr int TPW = 4 * TPT;                     // tokens per warp
  constexpr int WPT = kBlockTokens / TPW;          // warps along the tokens
  constexpr int G = TPT / 4;                       // 4-token groups per thread
  static_assert(WPT * (D / 64) == kQuantWarps, "one V task per warp");
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int c0 = (warp / WPT) * 64 + (lane % 8) * 8;
  const int t0 = (warp % WPT) * TPW + (lane / 8) * TPT;
  uint4 raw[TPT];                                  // the tokens' 8 channels, unconverted (zeros past `rows`)
#pragma unroll
  for (int t = 0; t < TPT; ++t)
    raw[t] = t0 + t < rows ? *reinterpret_cast<const uint4 *>(tile + (t0 + t) * D + c0) : make_uint4(0u, 0u, 0u, 0u);
  if (tok0 + t0 < Nv) {                            // Nv is a multiple of 16: all TPT tokens in or out
    uint64_t redo = 0u;                            // bit TPT i + t: channel c0 + i, token t0 + t
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float rlo = sv_s[D + c0 + i], rhi = sv_s[2 * D + c0 + i];
      uint32_t w[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float x[4] = {elem8<T>(raw[4 * g], i), elem8<T>(raw[4 * g + 1], i), elem8<T>(raw[4 * g + 2], i),
                            elem8<T>(raw[4 * g + 3], i)};
        unsigned bad;
        w[g] = e4m3_codes4_fast(x, rlo, rhi, bad);
        if (!(rlo > 0.f)) bad = 0xFu;              // no safe bracket for this channel
        redo |= static_cast<uint64_t>(bad) << (TPT * i + 4 * g);
      }
      store_codes<G>(vt_h + static_cast<size_t>(c0 + i) * Nv + tok0 + t0, w);
    }
    // values whose ends disagree: the code of the IEEE quotient, over the byte just stored
    for (; redo != 0u; redo &= redo - 1u) {
      const int e = __ffsll(static_cast<long long>(redo)) - 1;
      const int c = c0 + e / TPT, t = t0 + e % TPT;
      const float x = t < rows ? static_cast<float>(tile[t * D + c]) : 0.f;
      vt_h[static_cast<size_t>(c) * Nv + tok0 + t] = static_cast<uint8_t>(cvt_e4m3x2(__fdiv_rn(x, sv_s[c]), 0.f));
    }
  }
  release_stage(empty);
}

}  // namespace sattn
