// Quantisation of the NVFP4 mode: the per-tile work of the fused quantiser
// (quant_fused.cuh schedules it).
//
// SageAttention tag page (reportify.cn), SageAttention3 summary, FP4 bullet
// [15]: microscaled FP4 with the NVFP4 format -- E2M1 values, one E4M3 scale
// per 16 consecutive values.  Readings used here (no per-tensor scale):
//   Q and K' = K - mu: blocks of 16 channels of one token;
//   V: blocks of 16 tokens of one channel (the contraction axis of P V),
//      stored transposed [d, Nv] with Nv = N rounded up to 32;
//   scale = E4M3_RNE(max|x| / 6)  (float32 division, then E4M3 rounding);
//   code  = E2M1_RNE_satfinite(x / scale)  (float32 division); a block whose
//           scale rounds to 0 gets zero codes.
// Codes are packed two per byte, the lower-index value in the low nibble.
//
// The MXFP4 mode (the format the same bullet [15] compares NVFP4 with; OCP
// Microscaling) uses the same tiles with blocks of 32 values (32 channels of a
// Q/K token, 32 tokens of a V channel) and one E8M0 scale per block:
//   scale = 2^(floor(log2 max|x|) - 2)  (E8M0 code = biased exponent of max|x| - 2,
//           0 for max|x| < 2^-124, 255 = NaN);
//   code  = E2M1_RNE_satfinite(x * 2^(127 - scale code))  (exact: a power of two).
// The MMA reads the E8M0 scale per 16 values, so each block's code is stored
// in both of its 16-value slots of the layout below.
//
// Scale factors are written directly in the layout the block-scaled MMA reads
// after a 32x128b.warpx4 tensor-memory copy: for every 128-row tile and every
// 64-value slice kk of the contraction axis, a 512-byte block in which the
// scale of row m (0..127) and 16-value block b (0..3 of the slice) sits at byte
// 16 * (m % 32) + 4 * (m / 32) + b.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ptx.cuh"
#include "quant_i8f8.cuh"

namespace sattn {

// Byte offset of a scale factor inside its 512-byte block.
__host__ __device__ __forceinline__ int sf_offset(int row, int blk) {
  return 16 * (row & 31) + 4 * ((row >> 5) & 3) + (blk & 3);
}

// E4M3 code -> float (exact, via the fp16 conversion).
__device__ __forceinline__ float e4m3_to_float(uint32_t code) {
  uint32_t h2;
  const uint16_t c16 = static_cast<uint16_t>(code & 0xFFu);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(c16));
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
}

// Two floats -> one byte of two E2M1 codes, `lo` in the low nibble.
__device__ __forceinline__ uint32_t cvt_e2m1x2(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
      "cvt.u32.u8 %0, t;\n\t}"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  return r;
}

// Eight floats -> one word of eight E2M1 codes (RNE, saturating), the values
// of a, b, c, d in that order from the lowest nibble up.
__device__ __forceinline__ uint32_t cvt_e2m1x8(float2 a, float2 b, float2 c, float2 d) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y), "f"(d.x), "f"(d.y));
  return r;
}

// The bracket multipliers of 1/v for every E4M3 code v (entry = (RN(r (1 -
// 2^-20)), RN(r (1 + 2^-20))), r = RN(1/v); (0, 0) for zero, NaN, negative
// and codes without a safe bracket), one code per thread of the CTA's first
// 256.
__device__ __forceinline__ void fill_e4m3_recip(float2 *tab) {
  if (threadIdx.x < 256) {
    const float v = e4m3_to_float(threadIdx.x);
    float rlo = 0.f, rhi = 0.f;
    if (!(v > 0.f) || !bracket(v, rlo, rhi)) rlo = rhi = 0.f;
    tab[threadIdx.x] = make_float2(rlo, rhi);
  }
}

// One NVFP4 block of 16 values (reading: scale = E4M3_RNE(max|x| / 6), code =
// E2M1_RNE_satfinite(x / scale), both quotients the IEEE float32 ones; a
// scale of 0 or NaN gives zero codes), by brackets (see `bracket`): the
// scale code from amax RN(RN(1/6) (1 -+ 2^-20)), both ends converted by one
// instruction (when they differ, the quotient amax / 6 is computed); the
// codes from x times the scale's entry of `recip`.  E4M3 and E2M1 rounding
// are monotone, so equal codes at both ends are the quotient's codes.
// Returns the scale code; w = the codes, two words of 8 nibbles (value k of
// the block in nibble k mod 8 of word k / 8); bad[i] has bit 4 (k mod 8) set
// where value k's two ends disagree (the caller then puts in the code of the
// quotient, see nvfp4_code).
__device__ __forceinline__ uint32_t nvfp4_block_fast(const float (&x)[16], const float2 *recip, uint32_t (&w)[2],
                                                     uint32_t (&bad)[2]) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmax_nan(amax, fabsf(x[i]));
  const uint32_t ends = cvt_e4m3x2(amax * __uint_as_float(0x3e2aaaa0u), amax * __uint_as_float(0x3e2aaab6u));
  uint32_t sc_code = ends >> 8;
  if ((ends & 0xFFu) != sc_code) sc_code = cvt_e4m3x2(__fdiv_rn(amax, 6.f), 0.f) & 0xFFu;
  w[0] = w[1] = 0u;
  bad[0] = bad[1] = 0u;
  if ((sc_code & 0x7Fu) == 0u || sc_code == 0x7Fu) return sc_code;   // zero scale, or NaN: zero codes
  const float2 rr = recip[sc_code];
  if (!(rr.x > 0.f)) {
    bad[0] = bad[1] = 0x11111111u;
    return sc_code;
  }
  uint32_t lo[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    float2 pl[4], ph[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 v = make_float2(x[8 * k + 2 * j], x[8 * k + 2 * j + 1]);
      pl[j] = fmul2(v, make_float2(rr.x, rr.x));
      ph[j] = fmul2(v, make_float2(rr.y, rr.y));
    }
    lo[k] = cvt_e2m1x8(pl[0], pl[1], pl[2], pl[3]);
    w[k] = cvt_e2m1x8(ph[0], ph[1], ph[2], ph[3]);
  }
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    uint32_t d = lo[k] ^ w[k];
    d |= d >> 1;
    d |= d >> 2;
    bad[k] = d & 0x11111111u;
  }
  return sc_code;
}

// E2M1 code of x / scale through the IEEE quotient.
__device__ __forceinline__ uint32_t nvfp4_code(float x, uint32_t sc_code) {
  return cvt_e2m1x2(__fdiv_rn(x, e4m3_to_float(sc_code)), 0.f) & 0xFu;
}

// E8M0 code of the MXFP4 scale of a block with largest magnitude amax (>= 0
// or NaN): floor(log2 amax) - 2 + 127 = (biased exponent of amax) - 2, at
// least 0 (amax below 2^-124, zero included; the codes are then 0 or exact
// small values); NaN -> 255.  A finite float32 amax gives at most 253.
__device__ __forceinline__ uint32_t mx_scale_code(float amax) {
  if (amax != amax) return 255u;
  const uint32_t e = (__float_as_uint(amax) >> 23) & 0xFFu;
  return e > 2u ? e - 2u : 0u;
}

// 2^(127 - code) for a scale code in [0, 253]: the exact reciprocal of the scale.
__device__ __forceinline__ float mx_inv_scale(uint32_t code) { return __uint_as_float((254u - code) << 23); }

// E2M1 codes of 16 values of an MXFP4 block with scale code `code`: x times
// the exact reciprocal, RNE satfinite; two words of 8 nibbles as in
// nvfp4_block_fast.  A NaN scale gives zero codes.
__device__ __forceinline__ void mxfp4_codes16(const float (&x)[16], uint32_t code, uint32_t (&w)[2]) {
  if (code == 255u) {
    w[0] = w[1] = 0u;
    return;
  }
  const float r = mx_inv_scale(code);
  const float2 r2 = make_float2(r, r);
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    float2 p[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) p[j] = fmul2(make_float2(x[8 * k + 2 * j], x[8 * k + 2 * j + 1]), r2);
    w[k] = cvt_e2m1x8(p[0], p[1], p[2], p[3]);
  }
}

// NVFP4 of a Q tile (IS_K = false) or of K - mu (IS_K = true, mu = the
// stage's per-channel values): thread ct takes the 16-channel block ct mod
// (d/16) of every (256 / (d/16))-th row.  Codes of valid rows into codes_blk
// (row r at codes_blk + r d/2); the scale of every row (0 for rows past
// `rows`) into the tile's scale-factor blocks sf_tile.
//
// MX = true: the MXFP4 variant; the thread pair ct, ct ^ 1 holds the two
// 16-channel halves of a 32-channel block and shares its maximum by a shuffle.
template <typename T, int D, bool IS_K, bool MX = false>
__device__ __forceinline__ void nvfp4_rows_tile(const T *tile, int rows, const float *mu_s, const float2 *recip,
                                                uint8_t *codes_blk, uint8_t *sf_tile, uint64_t *empty) {
  constexpr int BPR = D / 16;                      // blocks per row
  constexpr int RPP = kQuantConsumers / BPR;
  constexpr int PASSES = kBlockTokens / RPP;
  const int ct = threadIdx.x;
  const int b = ct % BPR;
  const int r0 = ct / BPR;
  float mu[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) mu[i] = IS_K ? mu_s[b * 16 + i] : 0.f;
  uint4 u[PASSES][2];                              // every row first
#pragma unroll
  for (int p = 0; p < PASSES; ++p) {
    const int r = r0 + p * RPP;
#pragma unroll
    for (int h = 0; h < 2; ++h)
      u[p][h] = r < rows ? *reinterpret_cast<const uint4 *>(tile + r * D + b * 16 + 8 * h) : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int p = 0; p < PASSES; ++p) {
    const int r = r0 + p * RPP;
    float v[16];
    float a[8], c[8];
    cvt8<T>(u[p][0], a);
    cvt8<T>(u[p][1], c);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[i] = a[i];
      v[8 + i] = c[i];
    }
    if (IS_K && r < rows) {                        // rows past `rows` stay zero
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = __fsub_rn(v[i], mu[i]);
    }
    uint32_t w[2];
    uint32_t sc_code;
    if constexpr (MX) {
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i) amax = fmax_nan(amax, fabsf(v[i]));
      amax = fmax_nan(amax, __shfl_xor_sync(0xffffffffu, amax, 1));   // the block's other 16 channels
      sc_code = mx_scale_code(amax);
      mxfp4_codes16(v, sc_code, w);
    } else {
      uint32_t bad[2];
      sc_code = nvfp4_block_fast(v, recip, w, bad);
#pragma unroll
      for (int k = 0; k < 2; ++k) {                // values next to an E2M1 rounding boundary
        for (uint32_t m = bad[k]; m != 0u; m &= m - 1u) {
          const int nib = (__ffs(m) - 1) >> 2;
          const int j = 8 * k + nib;
          float xj = static_cast<float>(tile[r * D + b * 16 + j]);
          if (IS_K) xj = __fsub_rn(xj, mu_s[b * 16 + j]);
          w[k] = (w[k] & ~(0xFu << (4 * nib))) | (nvfp4_code(xj, sc_code) << (4 * nib));
        }
      }
    }
    if (r < rows) __stcs(reinterpret_cast<uint2 *>(codes_blk + r * (D / 2) + b * 8), make_uint2(w[0], w[1]));
    sf_tile[(b >> 2) * 512 + sf_offset(r, b)] = static_cast<uint8_t>(sc_code);
  }
  release_stage(empty);
}

// NVFP4 of a V tile: blocks of 16 tokens of one channel, written transposed
// into vt_h[c * Nv/2 + (tok0 + t)/2] for tokens below Nv (tokens at and past
// N are zeros).  Warp w < 4 d/64 takes 32 tokens of 64 channels; lane l the
// channel pair 2 l, 2 l + 1 of that half, read as one 32-bit word per token
// (a warp reads 128 consecutive bytes of a row), and stores 16 code bytes
// per channel.
// MX = true: the MXFP4 variant, one block of 32 tokens per (warp, channel).
template <typename T, int D, bool MX = false>
__device__ __forceinline__ void nvfp4_v_tile(const T *tile, int rows, int tok0, int Nv, const float2 *recip,
                                             uint8_t *vt_h, uint8_t *sf_tile, uint64_t *empty) {
  constexpr int NCH = D / 64;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  if (warp < 4 * NCH) {
    const int tg = warp / NCH;                     // 32-token group of the tile
    const int c = 2 * ((warp % NCH) * 32 + lane);  // first channel of the pair
    float x[2][32];
#pragma unroll
    for (int t = 0; t < 32; ++t) {
      const int r = tg * 32 + t;
      const uint32_t u = r < rows ? *reinterpret_cast<const uint32_t *>(tile + r * D + c) : 0u;
      const float2 f = unpack2<T>(u);
      x[0][t] = f.x;
      x[1][t] = f.y;
    }
#pragma unroll
    for (int ch = 0; ch < 2; ++ch) {
      uint32_t w[4];
      uint32_t mx_code = 0u;
      if constexpr (MX) {
        float amax = 0.f;
#pragma unroll
        for (int t = 0; t < 32; ++t) amax = fmax_nan(amax, fabsf(x[ch][t]));
        mx_code = mx_scale_code(amax);
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float blk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) blk[i] = x[ch][16 * h + i];
        uint32_t wh[2];
        uint32_t sc_code = mx_code;
        if constexpr (MX) {
          mxfp4_codes16(blk, sc_code, wh);
        } else {
          uint32_t bad[2];
          sc_code = nvfp4_block_fast(blk, recip, wh, bad);
#pragma unroll
          for (int k = 0; k < 2; ++k) {            // values next to an E2M1 rounding boundary
            for (uint32_t m = bad[k]; m != 0u; m &= m - 1u) {
              const int nib = (__ffs(m) - 1) >> 2;
              const int r = tg * 32 + 16 * h + 8 * k + nib;
              const float xj = r < rows ? static_cast<float>(tile[r * D + c + ch]) : 0.f;
              wh[k] = (wh[k] & ~(0xFu << (4 * nib))) | (nvfp4_code(xj, sc_code) << (4 * nib));
            }
          }
        }
        w[2 * h] = wh[0];
        w[2 * h + 1] = wh[1];
        const int t16 = 2 * tg + h;                // 16-token block of the tile
        sf_tile[(t16 >> 2) * 512 + sf_offset(c + ch, t16)] = static_cast<uint8_t>(sc_code);
      }
      if (tok0 + tg * 32 < Nv)                     // Nv is a multiple of 32
        __stcs(reinterpret_cast<uint4 *>(vt_h + static_cast<size_t>(c + ch) * (Nv / 2) + (tok0 + tg * 32) / 2),
               make_uint4(w[0], w[1], w[2], w[3]));
    }
  }
  release_stage(empty);
}

}  // namespace sattn
