// Test accessor of the INT8 tensor-core product of the I8QK_F8PV mode: the
// integer scores S_int = q8 . k8^T of a quantised workspace, exported to
// global memory so that a test can compare them bit for bit with an exact
// integer matrix product (TurboDiffusion explainer, wxsanhe.com post 64219,
// section 1: QK^T in INT8).
//
// One CTA per (query tile, key tile, head): the 128 x d tiles of q8 and k8 come
// in by the same TMA tensor maps (128- or 64-byte swizzle) and the product is
// issued with the same shared-memory and instruction descriptors
// (sdesc_kmajor, idesc_i8_s32, tcgen05.mma kind::i8, D/32 steps of K = 32) as
// in attn_i8f8_kernel; the int32 accumulator is read back from tensor memory
// by the four warps (warp w: rows 32 w .. 32 w + 31).  Not on the attention
// path: only tests call it.
//
// The FP4 modes have the same accessor (debug_scores_fp4_kernel): the E2M1
// codes by the attention kernel's tensor maps, the block scales (E4M3, or the
// MXFP4 mode's E8M0 codes stored per 16 values) by 1-D bulk copies and
// tcgen05.cp into tensor memory, and tcgen05.mma kind::mxf4nvf4 block16 with
// the same instruction descriptor: the exported float32 S is the product of
// the dequantised operands (SageAttention tag page, SageAttention3 summary,
// FP4 bullet [15]).
#pragma once

#include "attn_i8f8.cuh"
#include "attn_nvfp4.cuh"
#include "ptx.cuh"

namespace sattn {

constexpr int kDebugThreads = 128;

template <int D>
struct DebugScoresSmem {
  static constexpr int kQ = 0;
  static constexpr int kK = kTile * D;             // both tiles 1024-byte aligned (D = 64 or 128)
  static constexpr int kBar = 2 * kTile * D;       // [2] mbarriers: tiles loaded, product done
  static constexpr int kMisc = kBar + 16;          // TMEM address, abort flag
  static constexpr int kAlloc = kMisc + 16 + 1024; // slack for the 1024-byte alignment
};

// out: int32 [gridDim.z][np][np], row = query token, column = key token of
// head blockIdx.z (np = tiles x 128; rows and columns past N hold the
// products of the zero-filled rows).
template <int D>
__global__ void __launch_bounds__(kDebugThreads, 1)
    debug_scores_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        int32_t *out, int np) {
  using L = DebugScoresSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *loaded = reinterpret_cast<uint64_t *>(smem + L::kBar);
  uint64_t *done = loaded + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMisc + 4);
  const int qt = blockIdx.x, kt = blockIdx.y, bh = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (warp == 0) {
    tmem_alloc(tmem_slot, kTile);
    tmem_relinquish();
  }
  if (threadIdx.x == 32) {
    mbar_init(loaded, 1);
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  bool issued = false;                            // thread 0: the product is in flight
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(loaded, 2 * kTile * D);
    tma_load_3d(smem + L::kQ, &tm_q, loaded, 0, qt * kTile, bh);
    tma_load_3d(smem + L::kK, &tm_k, loaded, 0, kt * kTile, bh);
    if (mbar_wait(loaded, 0, abort_flag)) {
      tc_fence_after();
      constexpr uint32_t kIdesc = idesc_i8_s32(kTile, kTile);
      const uint32_t sQ = smem_u32(smem + L::kQ), sK = smem_u32(smem + L::kK);
#pragma unroll
      for (int kk = 0; kk < D / 32; ++kk)
        mma_i8(tmem, sdesc_kmajor<D>(sQ + kk * 32), sdesc_kmajor<D>(sK + kk * 32), kIdesc, kk > 0 ? 1u : 0u);
      mma_commit(done);
      issued = true;
    } else {
      drain_wait(loaded, 0);                      // the copies complete before the CTA exits
    }
  }
  __syncwarp();
  // warp-uniform decision: the TMEM loads below are warp-collective
  if (__all_sync(0xffffffffu, mbar_wait(done, 0, abort_flag))) {
    tc_fence_after();
    const int row = qt * kTile + warp * 32 + lane;
    int32_t *orow = out + (static_cast<size_t>(bh) * np + row) * np + kt * kTile;
#pragma unroll 1
    for (int c = 0; c < kTile / 32; ++c) {
      uint32_t s[32];
      tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + c * 32, s);
      tmem_ld_wait(s);
#pragma unroll
      for (int i = 0; i < 32; i += 4)
        *reinterpret_cast<int4 *>(orow + c * 32 + i) =
            make_int4(static_cast<int>(s[i]), static_cast<int>(s[i + 1]), static_cast<int>(s[i + 2]),
                      static_cast<int>(s[i + 3]));
    }
  }
  if (issued) drain_wait(done, 0);                // the MMA completes before its TMEM is released
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTile);
  }
}

template <int D>
struct DebugScoresF4Smem {
  static constexpr int kRowB = D / 2;              // bytes of one row of codes
  static constexpr int kQ = 0;
  static constexpr int kK = 1024 * ((kTile * kRowB + 1023) / 1024);
  static constexpr int kSfQ = kK + 1024 * ((kTile * kRowB + 1023) / 1024);
  static constexpr int kSfBytes = (D / 64) * 512; // scale bytes of a 128-row tile
  static constexpr int kSfK = kSfQ + kSfBytes;
  static constexpr int kBar = kSfK + kSfBytes;
  static constexpr int kMisc = kBar + 16;
  static constexpr int kAlloc = kMisc + 16 + 1024;
};

// out: float32 [gridDim.z][np][np]; sfq, sfk: the workspace's scale blocks
// [heads][tiles][D/64][512].
template <int D, bool MX>
__global__ void __launch_bounds__(kDebugThreads, 1)
    debug_scores_fp4_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                            const uint8_t *sfq, const uint8_t *sfk, int nblk, float *out, int np) {
  using L = DebugScoresF4Smem<D>;
  constexpr int kNK = D / 64;                      // 64-value slices of the contraction axis
  constexpr uint32_t kCols = 256;                  // S [0, 128), scale factors from 128
  constexpr int kSfQc = kTile, kSfKc = kTile + 4 * kNK;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *loaded = reinterpret_cast<uint64_t *>(smem + L::kBar);
  uint64_t *done = loaded + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMisc + 4);
  const int qt = blockIdx.x, kt = blockIdx.y, bh = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (warp == 0) {
    tmem_alloc(tmem_slot, kCols);
    tmem_relinquish();
  }
  if (threadIdx.x == 32) {
    mbar_init(loaded, 1);
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  bool issued = false;                            // thread 0: the product is in flight
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(loaded, 2 * kTile * L::kRowB + 2 * L::kSfBytes);
    tma_load_3d(smem + L::kQ, &tm_q, loaded, 0, qt * kTile, bh);
    tma_load_3d(smem + L::kK, &tm_k, loaded, 0, kt * kTile, bh);
    bulk_load(smem + L::kSfQ, sfq + (static_cast<size_t>(bh) * nblk + qt) * L::kSfBytes, L::kSfBytes, loaded);
    bulk_load(smem + L::kSfK, sfk + (static_cast<size_t>(bh) * nblk + kt) * L::kSfBytes, L::kSfBytes, loaded);
    if (mbar_wait(loaded, 0, abort_flag)) {
      tc_fence_after();
      constexpr uint32_t kIdesc = idesc_nvfp4(kTile, kTile) | (MX ? (1u << 23) : 0u);
      const uint32_t sQ = smem_u32(smem + L::kQ), sK = smem_u32(smem + L::kK);
#pragma unroll
      for (int kk = 0; kk < kNK; ++kk) {
        tmem_cp_sf(tmem + kSfQc + 4 * kk, sdesc_sf_block(smem_u32(smem + L::kSfQ + 512 * kk)));
        tmem_cp_sf(tmem + kSfKc + 4 * kk, sdesc_sf_block(smem_u32(smem + L::kSfK + 512 * kk)));
      }
#pragma unroll
      for (int kk = 0; kk < kNK; ++kk)
        mma_nvfp4(tmem, sdesc_f4<L::kRowB>(sQ + 32 * kk), sdesc_f4<L::kRowB>(sK + 32 * kk), kIdesc,
                  tmem + kSfQc + 4 * kk, tmem + kSfKc + 4 * kk, kk > 0 ? 1u : 0u);
      mma_commit(done);
      issued = true;
    } else {
      drain_wait(loaded, 0);                      // the copies complete before the CTA exits
    }
  }
  __syncwarp();
  // warp-uniform decision: the TMEM loads below are warp-collective
  if (__all_sync(0xffffffffu, mbar_wait(done, 0, abort_flag))) {
    tc_fence_after();
    const int row = qt * kTile + warp * 32 + lane;
    float *orow = out + (static_cast<size_t>(bh) * np + row) * np + kt * kTile;
#pragma unroll 1
    for (int c = 0; c < kTile / 32; ++c) {
      uint32_t s[32];
      tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + c * 32, s);
      tmem_ld_wait(s);
#pragma unroll
      for (int i = 0; i < 32; i += 4)
        *reinterpret_cast<float4 *>(orow + c * 32 + i) =
            make_float4(__uint_as_float(s[i]), __uint_as_float(s[i + 1]), __uint_as_float(s[i + 2]),
                        __uint_as_float(s[i + 3]));
    }
  }
  if (issued) drain_wait(done, 0);                // the MMA completes before its TMEM is released
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kCols);
  }
}

}  // namespace sattn
