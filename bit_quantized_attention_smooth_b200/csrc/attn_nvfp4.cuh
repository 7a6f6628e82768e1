// Fused attention of the NVFP4 mode on sm_100a block-scaled tensor cores.
//
// Method (SageAttention tag page, reportify.cn, SageAttention3 summary, FP4
// bullets [15][16]): Q, K' = K - mean, V and P in NVFP4 (E2M1 values, one E4M3
// scale per 16 values), with a two-stage quantisation of P.  Per query tile of
// 128 rows and key tile j of 128 keys:
//   S      = Q^ K'^T                   tcgen05.mma kind::mxf4nvf4 block16 -> fp32 TMEM
//                                       (the MMA applies both operands' block scales)
//   S2     = S * sm_scale * log2(e);  m = running row max;  m_t = row max of the tile
//   stage 1: s1 = 2^(m_t - m) / 2688, P2 = P~ / s1 = 2688 * 2^(S2 - m_t)  (row max -> 6 * 448)
//   stage 2: per 16 keys, scale = E4M3(max P2 / 6), codes = E2M1(P2 / scale)
//   O_in   = P2^ V^                     tcgen05.mma kind::mxf4nvf4 block16 -> fp32 TMEM
//   O_out  = alpha O_out + s1 O_in  (every tile: s1 changes per tile),  l = alpha l + rowsum(P~)
//   O      = O_out / l
//
// CTA = one 128-row query tile of one (b, h); 18 warps:
//   warps 0-15 softmax: warp w serves row 32 (w mod 4) + lane (TMEM lane
//              quarter w mod 4) and key quarter k = w / 4: keys 32 k .. 32 k + 31
//              of each key tile (two 16-key scale blocks) and output columns
//              [k D / 4, (k + 1) D / 4)
//   warp 16    TMA producer (codes by tensor maps, scale factors by 1-D bulk copies)
//   warp 17    TMEM allocator and single-thread MMA issuer; it also moves the
//              scale factors from shared to tensor memory (tcgen05.cp 32x128b.warpx4)
// The four threads of a row exchange their quarters' maxima through shared
// memory (a bounded four-warp mbarrier per lane quarter); each quantises its
// 32 keys of P and keeps its quarter of the outer accumulator in registers.
// Four softmax warps per SM sub-partition hide each other's latency.
// TMEM columns: S [0,128) [128,256), O_in [256,256+D), scale factors from 384.
// Scale factors of a 128-row operand and a 64-value slice of the contraction
// axis occupy 4 columns: row m at lane m % 32 of every sub-partition, column
// m / 32, byte = 16-value block within the slice.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "attn_i8f8.cuh"
#include "ptx.cuh"
#include "quant_nvfp4.cuh"

namespace sattn {

constexpr int kF4Threads = 576;
constexpr int kF4SoftmaxWarps = 16;
constexpr float kLog2_2688 = 11.392317422778761f;   // log2(448 * 6)
constexpr float kLog2_6 = 2.584962500721156f;       // log2(6)

struct AttnF4Args {
  const uint8_t *sfq;   // [BH][nblk][D/64][512]
  const uint8_t *sfk;   // [BH][nblk][D/64][512]
  const uint8_t *sfv;   // [BH][nblk][2][512]
  void *out;            // [BH, N, D]
  int N;
  int nblk;
  float sm_log2;
  const uint8_t *block_mask;   // [BH, nblk, nblk], nonzero = keep the 128x128 block; nullptr = dense
};

template <int D>
struct AttnF4Smem {
  static constexpr int kRowB = D / 2;                 // bytes of one Q/K row of codes
  static constexpr int kQBytes = kTile * kRowB;
  static constexpr int kKBytes = kTile * kRowB;
  static constexpr int kVBytes = D * (kTile / 2);
  static constexpr int kPBytes = kTile * (kTile / 2);
  static constexpr int kSfQK = (D / 64) * 512;        // scale bytes of a Q or K tile
  static constexpr int kSfV = 1024;                   // scale bytes of a V tile (2 slices)
  static constexpr int kSfP = 1024;
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + 1024 * ((kQBytes + 1023) / 1024);
  static constexpr int kV = kK + kKVStages * kKBytes;
  static constexpr int kP = kV + kKVStages * kVBytes;
  static constexpr int kSfQ = kP + 2 * kPBytes;
  static constexpr int kSfK = kSfQ + kSfQK;
  static constexpr int kSfVo = kSfK + kKVStages * kSfQK;
  static constexpr int kSfPo = kSfVo + kKVStages * kSfV;
  static constexpr int kX = kSfPo + 2 * kSfP;          // float [2 phases][4 quarters][128] + [4][128]
  static constexpr int kLsc = kX + (2 * 4 * 128 + 4 * 128) * 4;   // float2 [128]: (value, log2 value) of E4M3 codes
  static constexpr int kMask = kLsc + 128 * 8;        // [kMaxMaskTiles] bytes (block-sparse calls)
  static constexpr int kBar = kMask + kMaxMaskTiles;
  // q_full, k_full[S], k_empty[S], v_full[S], v_empty[S], s_full[2], s_free[2],
  // p_full[2], pv_done[2], quad[4], drain
  static constexpr int kNumBars = 1 + 4 * kKVStages + 8 + 4 + 1;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kBytes = kMisc + 16 + 256;     // 256 bytes of slack after the last buffer
  static constexpr int kAlloc = kBytes + 1024;
};

// 1-D bulk copy global -> shared, completion counted in bytes on `bar`.
__device__ __forceinline__ void bulk_load(void *smem_dst, const void *gsrc, uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(gsrc)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Shared-memory descriptor of a [32 rows][16 bytes] block without swizzle:
// 8-row core matrices of 128 bytes stacked at 128 bytes.
__device__ __forceinline__ uint64_t sdesc_sf_block(uint32_t smem_addr) {
  return static_cast<uint64_t>((smem_addr & 0x3FFFF) >> 4) | (uint64_t(1) << 16) | (uint64_t(128 >> 4) << 32) |
         (uint64_t(1) << 46);
}

// Scale factors of one 64-value slice: 32 x 16 bytes from shared memory to 4
// TMEM columns of all four sub-partitions.
__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T with E2M1 operands and one block scale per
// 16 values in TMEM (UE4M3, or UE8M0 when the descriptor's bit 23 is set).
__device__ __forceinline__ void mma_nvfp4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Instruction descriptor of kind::mxf4nvf4: A and B E2M1 (format 1) K-major,
// UE4M3 scales (bit 23 = 0; the MXFP4 variant sets it for UE8M0), N >> 3 in [17,23), M >> 4 in [24,29), scale ids 0,
// dense K = 64.
__host__ __device__ constexpr uint32_t idesc_nvfp4(int M, int N) {
  return (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// K-major descriptor for 64-byte (SW64) or 32-byte (SW32) rows of FP4 codes.
template <int ROW_BYTES>
__device__ __forceinline__ uint64_t sdesc_f4(uint32_t smem_addr) {
  static_assert(ROW_BYTES == 32 || ROW_BYTES == 64, "fp4 row width");
  constexpr uint64_t sbo = (8 * ROW_BYTES) >> 4;
  constexpr uint64_t mode = ROW_BYTES == 64 ? 4 : 6;
  return static_cast<uint64_t>((smem_addr & 0x3FFFF) >> 4) | (uint64_t(1) << 16) | (sbo << 32) |
         (uint64_t(1) << 46) | (mode << 61);
}

// MX = true: the MXFP4 ablation (tag page, SageAttention3 summary, FP4 bullet
// [15]): every FP4 operand in blocks of 32 with E8M0 scales.  The MMA runs in
// its 16-value scale mode with UE8M0 scales (each 32-block's scale stored
// twice), which computes the same products; P's second stage takes the E8M0
// scale of its 32-key block.
template <int D, bool CAUSAL, typename OutT, bool SPARSE, bool MX = false>
__global__ void __launch_bounds__(kF4Threads, 1)
    attn_nvfp4_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const AttnF4Args args) {
  using L = AttnF4Smem<D>;
  static_assert(D == 64 || D == 128, "head dim");
  constexpr uint32_t kTmemCols = 512;
  constexpr int kOin = 256;
  constexpr int kNK = D / 64;                         // 64-channel slices of Q/K
  constexpr int kSfQc = 384;                          // TMEM scale-factor columns
  constexpr int kSfKc = kSfQc + 4 * kNK;              // [2]
  constexpr int kSfVc = kSfKc + 2 * 4 * kNK;          // [2] x 8
  constexpr int kSfPc = kSfVc + 2 * 8;                // [2] x 8
  static_assert(kSfPc + 16 <= 512, "TMEM columns");

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kBar);
  uint64_t *q_full = bars;
  uint64_t *k_full = bars + 1;
  uint64_t *k_empty = k_full + kKVStages;
  uint64_t *v_full = k_empty + kKVStages;
  uint64_t *v_empty = v_full + kKVStages;
  uint64_t *s_full = v_empty + kKVStages;   // [2]
  uint64_t *s_free = s_full + 2;            // [2]
  uint64_t *p_full = s_free + 2;            // [2]
  uint64_t *pv_done = p_full + 2;           // [2]
  uint64_t *quad = pv_done + 2;             // [lane quarter]: the four key quarters of the rows
  uint64_t *drain_bar = quad + 4;
  float *xmax = reinterpret_cast<float *>(smem + L::kX);                  // [2][4][128]
  float *xl = reinterpret_cast<float *>(smem + L::kX + 2 * 4 * 128 * 4);  // [4][128]
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMisc + 4);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int bh = blockIdx.y;
  const int N = args.N;
  const int nkv_all = args.nblk;
  const int qt = CAUSAL ? (static_cast<int>(gridDim.x) - 1 - static_cast<int>(blockIdx.x))
                        : static_cast<int>(blockIdx.x);
  const int nkv = CAUSAL ? min(qt + 1, nkv_all) : nkv_all;
  // Block-sparse skipping: key tile j is processed iff need(j); every role
  // walks the same sequence of needed tiles, and the barriers and buffers
  // advance per position n in it (n == j for dense calls).
  const uint8_t *smask = smem + L::kMask;
  auto need = [&](int jj) -> bool { return !SPARSE || smask[jj] != 0; };
  if (SPARSE) {
    uint8_t *sm = smem + L::kMask;
    for (int i = tid; i < nkv_all; i += kF4Threads)
      sm[i] = args.block_mask[(static_cast<size_t>(bh) * nkv_all + qt) * nkv_all + i];
  }

  if (warp == 17) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (tid == 512) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kKVStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_free[b], kF4SoftmaxWarps);   // one arrival per softmax warp
      mbar_init(&p_full[b], kF4SoftmaxWarps);
      mbar_init(&pv_done[b], 1);
    }
    for (int i = 0; i < 4; ++i) mbar_init(&quad[i], 4);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (tid == 544) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (!MX && tid < 128) {
    // every non-negative E4M3 code's value and log2 (the stage-2 scales of P)
    const float v = e4m3_to_float(static_cast<uint32_t>(tid));
    reinterpret_cast<float2 *>(smem + L::kLsc)[tid] = make_float2(v, v > 0.f ? __log2f(v) : 0.f);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 16) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      int last_n = -1;
      const int withheld = g_withhold_k_tile;            // -1 except under the failure-path test hook
      const size_t sf_qk_tile = static_cast<size_t>(L::kSfQK);
      mbar_arrive_expect_tx(q_full, L::kQBytes + L::kSfQK);
      tma_load_3d(smem + L::kQ, &tm_q, q_full, 0, qt * kTile, bh);
      bulk_load(smem + L::kSfQ, args.sfq + (static_cast<size_t>(bh) * nkv_all + qt) * sf_qk_tile, L::kSfQK, q_full);
      for (int j = 0, n = 0; j < nkv; ++j) {
        if (!need(j)) continue;
        const int s = n % kKVStages;
        const uint32_t ph = (n / kKVStages) & 1;
        if (!mbar_wait(&k_empty[s], ph ^ 1, abort_flag)) break;
        if (n != withheld) {
          mbar_arrive_expect_tx(&k_full[s], L::kKBytes + L::kSfQK);
          tma_load_3d(smem + L::kK + s * L::kKBytes, &tm_k, &k_full[s], 0, j * kTile, bh);
          bulk_load(smem + L::kSfK + s * L::kSfQK, args.sfk + (static_cast<size_t>(bh) * nkv_all + j) * sf_qk_tile,
                    L::kSfQK, &k_full[s]);
        }
        if (!mbar_wait(&v_empty[s], ph ^ 1, abort_flag)) {
          if (n != withheld) drain_wait(&k_full[s], ph);
          break;
        }
        mbar_arrive_expect_tx(&v_full[s], L::kVBytes + L::kSfV);
        tma_load_3d(smem + L::kV + s * L::kVBytes, &tm_v, &v_full[s], j * (kTile / 2), 0, bh);
        bulk_load(smem + L::kSfVo + s * L::kSfV, args.sfv + (static_cast<size_t>(bh) * nkv_all + j) * L::kSfV,
                  L::kSfV, &v_full[s]);
        last_n = n++;
      }
      if (*abort_flag) {
        drain_wait(q_full, 0);
        for (int n = max(0, last_n - kKVStages + 1); n <= last_n; ++n) {
          const uint32_t ph = (n / kKVStages) & 1;
          if (n != withheld) drain_wait(&k_full[n % kKVStages], ph);
          drain_wait(&v_full[n % kKVStages], ph);
        }
      }
    }
    __syncwarp();
  } else if (warp == 17) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t kScaleE8M0 = MX ? (1u << 23) : 0u;   // scale format bit: UE8M0
      constexpr uint32_t kIdQK = idesc_nvfp4(kTile, kTile) | kScaleE8M0;
      constexpr uint32_t kIdPV = idesc_nvfp4(kTile, D) | kScaleE8M0;
      const uint32_t sQ = smem_u32(smem + L::kQ);
      bool ok = mbar_wait(q_full, 0, abort_flag);
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kNK; ++kk)
          tmem_cp_sf(tmem + kSfQc + 4 * kk, sdesc_sf_block(smem_u32(smem + L::kSfQ + 512 * kk)));
      }
      for (int j = 0, n = 0; ok && j <= nkv; ++j) {
        if (j < nkv && !need(j)) continue;
        if (j < nkv) {                                    // S_b = Q K_j^T, the n-th needed tile
          const int s = n % kKVStages;
          const int b = n & 1;
          ok = mbar_wait(&k_full[s], (n / kKVStages) & 1, abort_flag) &&
               mbar_wait(&s_free[b], ((n >> 1) & 1) ^ 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint32_t sK = smem_u32(smem + L::kK + s * L::kKBytes);
          const uint32_t sfk = tmem + kSfKc + b * 4 * kNK;
#pragma unroll
          for (int kk = 0; kk < kNK; ++kk)
            tmem_cp_sf(sfk + 4 * kk, sdesc_sf_block(smem_u32(smem + L::kSfK + s * L::kSfQK + 512 * kk)));
#pragma unroll
          for (int kk = 0; kk < kNK; ++kk)
            mma_nvfp4(tmem + b * kTile, sdesc_f4<L::kRowB>(sQ + 32 * kk), sdesc_f4<L::kRowB>(sK + 32 * kk), kIdQK,
                      tmem + kSfQc + 4 * kk, sfk + 4 * kk, kk > 0 ? 1u : 0u);
          mma_commit(&s_full[b]);
          mma_commit(&k_empty[s]);
        }
        if (n > 0) {                                      // O_in = P V of the (n-1)-th needed tile
          const int t = n - 1;
          const int s = t % kKVStages;
          const int b = t & 1;
          ok = mbar_wait(&v_full[s], (t / kKVStages) & 1, abort_flag) &&
               mbar_wait(&p_full[b], (t >> 1) & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint32_t sV = smem_u32(smem + L::kV + s * L::kVBytes);
          const uint32_t sP = smem_u32(smem + L::kP + b * L::kPBytes);
          const uint32_t sfv = tmem + kSfVc + b * 8;
          const uint32_t sfp = tmem + kSfPc + b * 8;
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            tmem_cp_sf(sfv + 4 * kk, sdesc_sf_block(smem_u32(smem + L::kSfVo + s * L::kSfV + 512 * kk)));
            tmem_cp_sf(sfp + 4 * kk, sdesc_sf_block(smem_u32(smem + L::kSfPo + b * L::kSfP + 512 * kk)));
          }
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            mma_nvfp4(tmem + kOin, sdesc_f4<64>(sP + 32 * kk), sdesc_f4<64>(sV + 32 * kk), kIdPV, sfp + 4 * kk,
                      sfv + 4 * kk, kk > 0 ? 1u : 0u);
          mma_commit(&pv_done[b]);
          mma_commit(&v_empty[s]);
        }
        ++n;
      }
      if (!ok) {
        mma_commit(drain_bar);
        drain_wait(drain_bar, 0);
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- softmax warps
    constexpr int kQD = D / 4;                        // output columns per warp
    const int kq = warp >> 2;                         // key quarter of the row
    const int wq = warp & 3;                          // TMEM lane quarter
    const int r = wq * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
    const int row_g = qt * kTile + r;
    const float cl = args.sm_log2;                    // S is already dequantised by the MMA
    float o_out[kQD];
#pragma unroll
    for (int i = 0; i < kQD; ++i) o_out[i] = 0.f;
    float m_ref = -INFINITY, l = 0.f;                 // l: this quarter's share of the row sum
    float a_pend = 0.f, s1_pend = 0.f;                // factors of the tile whose P V is pending
    bool ok = true;
    // this warp's output columns of O_in, read as one or two 16-column loads
    auto load_oin = [&](uint32_t (&o)[kQD]) {
      const uint32_t base = tmem + lane_base + kOin + kq * kQD;
      if constexpr (kQD == 32) {
        tmem_ld_32x32b_x32(base, o);
        tmem_ld_wait(o);
      } else {
        tmem_ld_32x32b_x16(base, o);
        tmem_ld_wait(o);
      }
    };

    int n = 0;                                        // key tiles processed
    for (int j = 0; j < nkv && ok; ++j) {
      if (!need(j)) continue;
      const int b = n & 1;
      if (!mbar_wait(&s_full[b], (n >> 1) & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      uint32_t sa[32];
      tmem_ld_32x32b_x32(tmem + lane_base + b * kTile + kq * 32, sa);
      tmem_ld_wait(sa);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[b]);          // S_b may take Q K_{j+2}^T
      const bool masked = ((j == nkv_all - 1) && (N & (kTile - 1))) || (CAUSAL && j == qt);
      if (masked) {
        const int kv0 = j * kTile + kq * 32;
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (kv0 + i >= N || (CAUSAL && kv0 + i > row_g)) sa[i] = __float_as_uint(-INFINITY);
      }
      // maxima of the two 16-key blocks of this quarter, then the row max via the other quarters
      float bmax[2];
#pragma unroll
      for (int hb = 0; hb < 2; ++hb) {
        const uint32_t *v = sa + hb * 16;
        float t[6];
#pragma unroll
        for (int i = 0; i < 5; ++i)
          t[i] = fmax3(__uint_as_float(v[3 * i]), __uint_as_float(v[3 * i + 1]), __uint_as_float(v[3 * i + 2]));
        t[5] = __uint_as_float(v[15]);
        bmax[hb] = fmaxf(fmax3(t[0], t[1], t[2]), fmax3(t[3], t[4], t[5]));
      }
      float *xm = xmax + (n & 1) * 4 * 128;
      xm[kq * 128 + r] = fmaxf(bmax[0], bmax[1]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&quad[wq]);
      if (!mbar_wait(&quad[wq], n & 1, abort_flag)) { ok = false; break; }
      const float tmax = fmaxf(fmax3(xm[r], xm[128 + r], xm[256 + r]), xm[384 + r]);
      const float m_tile = tmax * cl;                   // finite: every processed tile has a valid key
      const float m_new = fmaxf(m_ref, m_tile);
      const float alpha = ex2_approx(m_ref - m_new);
      const float s1 = ex2_approx(m_tile - m_new) * (1.f / 2688.f);
      const float moff = m_tile - kLog2_2688;           // P2 = 2^(S2 - moff) <= 2688
      const float moff6 = moff + kLog2_6;

      // two-stage NVFP4 quantisation of this quarter of P into buffer b
      if (!mbar_wait(&pv_done[b], ((n >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
      uint8_t *prow = smem + L::kP + b * L::kPBytes + r * 64;
      uint8_t *psf = smem + L::kSfPo + b * L::kSfP + (kq >> 1) * 512;   // 64-key slice of the quarter
      float psum = 0.f;
      const float2 cl2 = make_float2(cl, cl);
      uint32_t w[4];
      if constexpr (MX) {
        // MXFP4: the quarter's 32 keys are one block; scale = 2^(floor(log2 max P2) - 2),
        // its E8M0 code the biased exponent of max P2 minus 2 (0 below 2^-124),
        // stored in both 16-key slots the MMA reads.  P2 / scale = 2^(S2 - moff
        // - log2 scale) with an integer log2 scale.
        const float p2max = ex2_approx(fmaf(fmaxf(bmax[0], bmax[1]), cl, -moff));
        const uint32_t e = (__float_as_uint(p2max) >> 23) & 0xFFu;
        const uint32_t sc_code = e > 2u ? e - 2u : 0u;
        *reinterpret_cast<uint16_t *>(psf + sf_offset(r, (kq & 1) * 2)) = static_cast<uint16_t>(sc_code * 0x101u);
        const float lsc = static_cast<float>(static_cast<int>(sc_code) - 127);
        const float sc = sc_code != 0u ? __uint_as_float(sc_code << 23) : __uint_as_float(1u << 22);
        const float2 nb2 = make_float2(-(moff + lsc), -(moff + lsc));
        float2 bsum = make_float2(0.f, 0.f);
#pragma unroll
        for (int hb = 0; hb < 2; ++hb) {
          float2 y[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float2 x = ffma2(
                make_float2(__uint_as_float(sa[hb * 16 + 2 * i]), __uint_as_float(sa[hb * 16 + 2 * i + 1])), cl2, nb2);
            y[i] = make_float2(ex2_approx(x.x), ex2_approx(x.y));
            bsum = fadd2(bsum, y[i]);
          }
          w[2 * hb] = cvt_e2m1x8(y[0], y[1], y[2], y[3]);
          w[2 * hb + 1] = cvt_e2m1x8(y[4], y[5], y[6], y[7]);
        }
        psum = sc * (bsum.x + bsum.y);
      } else {
#pragma unroll
      for (int hb = 0; hb < 2; ++hb) {
        const int blk = (kq & 1) * 2 + hb;                // 16-key block within the 64-key slice
        // scale = E4M3(block max of P2 / 6): the division by 6 folds into the exponent
        const float amax6 = ex2_approx(fmaf(bmax[hb], cl, -moff6));
        const uint32_t sc_code = cvt_e4m3x2(amax6, 0.f) & 0x7Fu;   // amax6 >= 0: sign bit clear
        const float2 scl = reinterpret_cast<const float2 *>(smem + L::kLsc)[sc_code];   // scale, log2 scale
        const float sc = scl.x;
        psf[sf_offset(r, blk)] = static_cast<uint8_t>(sc_code);
        // P2 / scale = 2^(S2 - moff - log2 scale): the division folds into the
        // exponent's constant; the block's P2 sum is scale * sum(P2 / scale).
        const bool live = sc > 0.f;
        const float lsc = scl.y;
        const float2 nb2 = make_float2(-(moff + lsc), -(moff + lsc));
        float2 bsum = make_float2(0.f, 0.f);
        float2 y[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float2 x = ffma2(
              make_float2(__uint_as_float(sa[hb * 16 + 2 * i]), __uint_as_float(sa[hb * 16 + 2 * i + 1])), cl2, nb2);
          y[i] = make_float2(ex2_approx(x.x), ex2_approx(x.y));
          bsum = fadd2(bsum, y[i]);
        }
        w[2 * hb] = cvt_e2m1x8(y[0], y[1], y[2], y[3]);
        w[2 * hb + 1] = cvt_e2m1x8(y[4], y[5], y[6], y[7]);
        if (live) psum = fmaf(sc, bsum.x + bsum.y, psum);
        else {
          // a block whose scale rounds to 0 has all-zero codes; its P2 values
          // (below 6 * 2^-10 of 2688) still count towards the row sum
          w[2 * hb] = w[2 * hb + 1] = 0u;
          psum += (bsum.x + bsum.y);
        }
      }
      }
      // 16 bytes = keys 32 kq .. 32 kq + 31; 64-byte swizzled K-major row
      *reinterpret_cast<uint4 *>(prow + ((kq ^ ((r >> 1) & 3)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);

      // flush the previous tile: O_out = a O_out + s1 O_in (this quarter of the columns)
      if (n > 0) {
        const int t = n - 1;
        if (!mbar_wait(&pv_done[t & 1], (t >> 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        uint32_t o[kQD];
        load_oin(o);
        const float2 a2 = make_float2(a_pend, a_pend), s2 = make_float2(s1_pend, s1_pend);
        if (__all_sync(0xffffffffu, a_pend == 1.f)) {
          // the usual case (no row's reference max moved): O_out += s1 O_in, one packed FMA per two columns
#pragma unroll
          for (int i = 0; i < kQD; i += 2) {
            const float2 rr = ffma2(s2, make_float2(__uint_as_float(o[i]), __uint_as_float(o[i + 1])),
                                    make_float2(o_out[i], o_out[i + 1]));
            o_out[i] = rr.x;
            o_out[i + 1] = rr.y;
          }
        } else {
#pragma unroll
          for (int i = 0; i < kQD; i += 2) {
            const float2 tt = fmul2(s2, make_float2(__uint_as_float(o[i]), __uint_as_float(o[i + 1])));
            const float2 rr = ffma2(a2, make_float2(o_out[i], o_out[i + 1]), tt);
            o_out[i] = rr.x;
            o_out[i + 1] = rr.y;
          }
        }
      }
      l = fmaf(alpha, l, s1 * psum);
      a_pend = alpha;
      s1_pend = s1;
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[b]);
      m_ref = m_new;
      ++n;
    }

    // ---------------------------------------------------------- epilogue
    if (ok && n > 0) {
      xl[kq * 128 + r] = l;
      __syncwarp();
      if (lane == 0) mbar_arrive(&quad[wq]);
      const int t = n - 1;
      if (mbar_wait(&quad[wq], n & 1, abort_flag) && mbar_wait(&pv_done[t & 1], (t >> 1) & 1, abort_flag)) {
        tc_fence_after();
        const float inv_l = 1.f / ((xl[r] + xl[128 + r]) + (xl[256 + r] + xl[384 + r]));
        OutT *orow = reinterpret_cast<OutT *>(args.out) + (static_cast<size_t>(bh) * N + row_g) * D + kq * kQD;
        uint32_t o[kQD];
        load_oin(o);
        uint32_t packed[kQD / 2];
#pragma unroll
        for (int i = 0; i < kQD; i += 2) {
          const float o0 = fmaf(a_pend, o_out[i], s1_pend * __uint_as_float(o[i])) * inv_l;
          const float o1 = fmaf(a_pend, o_out[i + 1], s1_pend * __uint_as_float(o[i + 1])) * inv_l;
          packed[i >> 1] = pack2_out<OutT>(o0, o1);
        }
        if (row_g < N) {
          uint4 *dst = reinterpret_cast<uint4 *>(orow);
#pragma unroll
          for (int u = 0; u < kQD / 8; ++u)
            dst[u] = make_uint4(packed[4 * u], packed[4 * u + 1], packed[4 * u + 2], packed[4 * u + 3]);
        }
      }
    } else if (ok && row_g < N) {
      // every key block of this query tile is skipped: the rows are zeros
      uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<OutT *>(args.out) + (static_cast<size_t>(bh) * N + row_g) * D +
                                             kq * kQD);
#pragma unroll
      for (int u = 0; u < kQD / 8; ++u) dst[u] = make_uint4(0u, 0u, 0u, 0u);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 17) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace sattn
