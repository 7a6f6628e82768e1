// Quantisation kernels of the NVFP4 mode.
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

// One NVFP4 block of 16 values: returns the E4M3 scale code and writes the 8
// code bytes (as two 32-bit words).
__device__ __forceinline__ uint32_t nvfp4_block(const float (&x)[16], uint32_t (&w)[2]) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmax_nan(amax, fabsf(x[i]));
  const uint32_t sc_code = cvt_e4m3x2(__fdiv_rn(amax, 6.f), 0.f) & 0xFFu;
  const float sc = e4m3_to_float(sc_code);
  w[0] = w[1] = 0u;
  if (sc > 0.f) {
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
      const uint32_t b = cvt_e2m1x2(__fdiv_rn(x[i], sc), __fdiv_rn(x[i + 1], sc));
      w[i >> 3] |= b << (4 * (i & 7));
    }
  }
  return sc_code;
}

// Q (IS_K = false) or K - mu (IS_K = true): one thread per (row, 16-channel
// block).  grid (ceil(N/128), B*H), block 256.
template <typename T, int D, bool IS_K>
__global__ void __launch_bounds__(kQuantThreads) quant_rows_nvfp4_kernel(const T *__restrict__ x,
                                                                         uint8_t *__restrict__ codes,
                                                                         uint8_t *__restrict__ sf,
                                                                         const double *__restrict__ ksum,
                                                                         float *__restrict__ mu_out, int N) {
  constexpr int BPR = D / 16;                      // blocks per row
  constexpr int SF_TILE = (D / 64) * 512;          // scale bytes per 128-row tile
  __shared__ float s_mu[D];
  const int bh = blockIdx.y;
  const int tile = blockIdx.x;
  const size_t head = static_cast<size_t>(bh) * N * D;
  const int ntiles = gridDim.x;
  if (IS_K) {
    if (threadIdx.x < D) {
      const float mu = static_cast<float>(ksum[static_cast<size_t>(bh) * D + threadIdx.x] / static_cast<double>(N));
      s_mu[threadIdx.x] = mu;
      if (tile == 0) mu_out[static_cast<size_t>(bh) * D + threadIdx.x] = mu;
    }
    __syncthreads();
  }
  uint8_t *sf_tile = sf + (static_cast<size_t>(bh) * ntiles + tile) * SF_TILE;
  for (int idx = threadIdx.x; idx < kBlockTokens * BPR; idx += kQuantThreads) {
    const int r = idx / BPR;
    const int b = idx % BPR;
    const int n = tile * kBlockTokens + r;
    float v[16];
    if (n < N) {
      float a[8], c[8];
      load8<T>(x + head + static_cast<size_t>(n) * D + b * 16, a);
      load8<T>(x + head + static_cast<size_t>(n) * D + b * 16 + 8, c);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        v[i] = a[i];
        v[8 + i] = c[i];
      }
      if (IS_K) {
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = __fsub_rn(v[i], s_mu[b * 16 + i]);
      }
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = 0.f;
    }
    uint32_t w[2];
    const uint32_t sc = nvfp4_block(v, w);
    if (n < N) *reinterpret_cast<uint2 *>(codes + (head + static_cast<size_t>(n) * D) / 2 + b * 8) = make_uint2(w[0], w[1]);
    sf_tile[(b >> 2) * 512 + sf_offset(r, b)] = static_cast<uint8_t>(sc);
  }
}

// V: blocks of 16 tokens of one channel, written transposed vt[bh][c][Nv/2].
// grid (ceil(N/128), B*H), block 256.
template <typename T, int D>
__global__ void __launch_bounds__(kQuantThreads) quant_v_nvfp4_kernel(const T *__restrict__ v, uint8_t *__restrict__ vt,
                                                                      uint8_t *__restrict__ sf, int N, int Nv) {
  __shared__ T tile_v[kBlockTokens][D + 2];
  const int bh = blockIdx.y;
  const int tile = blockIdx.x;
  const size_t head = static_cast<size_t>(bh) * N * D;
  const int ntiles = gridDim.x;
  for (int idx = threadIdx.x; idx < kBlockTokens * D / 8; idx += kQuantThreads) {
    const int r = idx / (D / 8);
    const int cg = idx % (D / 8);
    const int n = tile * kBlockTokens + r;
    float a[8];
    if (n < N) {
      load8<T>(v + head + static_cast<size_t>(n) * D + cg * 8, a);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) a[i] = 0.f;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) tile_v[r][cg * 8 + i] = static_cast<T>(a[i]);
  }
  __syncthreads();
  uint8_t *sf_tile = sf + (static_cast<size_t>(bh) * ntiles + tile) * 1024;
  for (int idx = threadIdx.x; idx < D * (kBlockTokens / 16); idx += kQuantThreads) {
    const int c = idx % D;
    const int t = idx / D;                         // 16-token block within the tile
    float x[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) x[i] = static_cast<float>(tile_v[t * 16 + i][c]);
    uint32_t w[2];
    const uint32_t sc = nvfp4_block(x, w);
    const int tok0 = tile * kBlockTokens + t * 16;
    if (tok0 < Nv)
      *reinterpret_cast<uint2 *>(vt + (static_cast<size_t>(bh) * D + c) * (Nv / 2) + tok0 / 2) = make_uint2(w[0], w[1]);
    sf_tile[(t >> 2) * 512 + sf_offset(c, t)] = static_cast<uint8_t>(sc);
  }
}

}  // namespace sattn
