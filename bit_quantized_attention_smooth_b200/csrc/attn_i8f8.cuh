// Fused attention of the INT8-QK / FP8-PV mode on sm_100a tensor cores.
//
// Method (TurboDiffusion explainer, wxsanhe.com post 64219, section 1 "hybrid
// attention"): S = Q K^T in INT8, P V in FP8, with a two-level accumulator for
// P V.  Per query tile of 128 rows and key tile j of 128 keys:
//   S_int  = q8 . k8^T                       tcgen05.mma kind::i8 -> int32 TMEM
//   S2     = S_int * s_q * s_k[j] * sm_scale * log2(e)
//   m      = running row max of S2 (online softmax)
//   P~     = 2^(S2 - m);  l += rowsum(P~)    FP32, one row per thread
//   p8     = E4M3(448 P~)                    written to shared memory
//   O_in  (+)= p8 . v8                       tcgen05.mma kind::f8f6f4 -> fp32 TMEM
//   every G tiles, or before a tile that raises some row's max:
//   O_out  = (O_out + O_in) * 2^(m_old - m_new)   (outer FP32 accumulator, TMEM)
//   O      = O_out * s_v[c] / (448 l)
//
// CTA = one 128-row query tile of one (b, h); 6 warps:
//   warps 0-3  softmax / flush / epilogue (thread t owns row t = TMEM lane t)
//   warp 4     TMA producer (Q once, then K_j and V_j through 3-stage rings)
//   warp 5     TMEM allocator and single-thread MMA issuer
// TMEM columns: S double buffer [0,128) [128,256), O_in [256,256+D),
// O_out [384,384+D).  S_{j+1} = Q K_{j+1}^T runs on the tensor cores while the
// softmax warps work on S_j; P V_j runs while they work on S_{j+1}.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ptx.cuh"

namespace sattn {

constexpr int kTile = 128;          // query rows and keys per tile
constexpr int kKVStages = 3;
constexpr int kFlushEvery = 4;      // G: key tiles per inner accumulation group
constexpr int kAttnThreads = 192;
constexpr float kLog2_448 = 8.807354922057604f;   // log2(448)

struct AttnArgs {
  const float *sq;   // [BH, nblk]
  const float *sk;   // [BH, nblk]
  const float *sv;   // [BH, D]
  void *out;         // [BH, N, D] bf16 / fp16
  int N;
  int nblk;          // ceil(N / 128)
  float sm_log2;     // sm_scale * log2(e)
};

template <int D>
struct AttnSmem {
  static constexpr int kQBytes = kTile * D;
  static constexpr int kKBytes = kTile * D;
  static constexpr int kVBytes = D * kTile;
  static constexpr int kPBytes = kTile * kTile;
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kQBytes;
  static constexpr int kV = kK + kKVStages * kKBytes;
  static constexpr int kP = kV + kKVStages * kVBytes;
  static constexpr int kBar = kP + 2 * kPBytes;
  // barriers: q_full, k_full[S], k_empty[S], v_full[S], v_empty[S], s_full[2],
  // s_free[2], p_full[2], p_free[2], vote, drain
  static constexpr int kNumBars = 1 + 4 * kKVStages + 8 + 2;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kBytes = kMisc + 64;
  static constexpr int kAlloc = kBytes + 1024;   // slack for 1024-byte alignment
};

template <typename OutT>
__device__ __forceinline__ uint32_t pack2_out(float a, float b);
template <>
__device__ __forceinline__ uint32_t pack2_out<__nv_bfloat16>(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}
template <>
__device__ __forceinline__ uint32_t pack2_out<__half>(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}

// Bounded wait used only while draining in-flight copies on an abort path.
__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity) {
  const unsigned long long t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      atomicOr(&g_error_word, kErrWaitTimeout);
      return;
    }
  }
}

// Sentinel for a masked score; |q8 . k8| <= 127 * 127 * 128 < 2^21, so no
// real INT8 score takes this value.
constexpr uint32_t kMaskedScore = 0x80000000u;

// One row of 448 * P~ = 2^(S2 - m + log2 448) -> E4M3 codes into the row's
// 128-byte line of the P tile, in the 128-byte-swizzled K-major layout the
// MMA reads (16-byte chunk c of row r stored at chunk c ^ (r mod 8)).
// Accumulates the unquantised values into l448.
template <bool MASKED>
__device__ __forceinline__ void write_p_row(const uint32_t (&S)[4][32], float c, float moff, uint8_t *prow, int r,
                                            float &l448) {
#pragma unroll
  for (int c16 = 0; c16 < 8; ++c16) {
    uint32_t w4[4];
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
      float p[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int idx = c16 * 16 + q4 * 4 + e;
        const uint32_t sv = S[idx >> 5][idx & 31];
        float x = fmaf(static_cast<float>(static_cast<int>(sv)), c, -moff);
        if (MASKED) x = (sv == kMaskedScore) ? -INFINITY : x;
        p[e] = ex2_approx(x);
        l448 += p[e];
      }
      w4[q4] = cvt_e4m3x2(p[0], p[1]) | (cvt_e4m3x2(p[2], p[3]) << 16);
    }
    *reinterpret_cast<uint4 *>(prow + ((c16 ^ (r & 7)) << 4)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
  }
}

template <int D, bool CAUSAL, typename OutT>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_i8f8_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const AttnArgs args) {
  using L = AttnSmem<D>;
  static_assert(D == 64 || D == 128, "head dim");
  constexpr int S_COL0 = 0, S_COL1 = 128, O_IN = 256, O_OUT = 384;
  constexpr uint32_t kTmemCols = 512;

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = smem + L::kQ;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kBar);
  uint64_t *q_full = bars;
  uint64_t *k_full = bars + 1;
  uint64_t *k_empty = k_full + kKVStages;
  uint64_t *v_full = k_empty + kKVStages;
  uint64_t *v_empty = v_full + kKVStages;
  uint64_t *s_full = v_empty + kKVStages;
  uint64_t *s_free = s_full + 2;
  uint64_t *p_full = s_free + 2;
  uint64_t *p_free = p_full + 2;
  uint64_t *vote_bar = p_free + 2;
  uint64_t *drain_bar = vote_bar + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMisc + 4);
  volatile int *pv_acc = reinterpret_cast<volatile int *>(smem + L::kMisc + 8);     // [2]
  volatile int *votes = reinterpret_cast<volatile int *>(smem + L::kMisc + 16);     // [2][4]

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int bh = blockIdx.y;
  const int N = args.N;
  const int nkv_all = args.nblk;
  const int qt = CAUSAL ? (static_cast<int>(gridDim.x) - 1 - static_cast<int>(blockIdx.x))
                        : static_cast<int>(blockIdx.x);
  const int nkv = CAUSAL ? min(qt + 1, nkv_all) : nkv_all;

  // ------------------------------------------------------------ set-up
  if (warp == 5) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (tid == 128) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kKVStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_free[b], 4);   // one arrival per softmax warp
      mbar_init(&p_full[b], 4);
      mbar_init(&p_free[b], 1);
    }
    mbar_init(vote_bar, 4);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (tid == 160) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      int last_j = -1;
      mbar_arrive_expect_tx(q_full, L::kQBytes);
      tma_load_3d(sQ, &tm_q, q_full, 0, qt * kTile, bh);
      for (int j = 0; j < nkv; ++j) {
        const int s = j % kKVStages;
        const uint32_t ph = (j / kKVStages) & 1;
        if (!mbar_wait(&k_empty[s], ph ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(&k_full[s], L::kKBytes);
        tma_load_3d(smem + L::kK + s * L::kKBytes, &tm_k, &k_full[s], 0, j * kTile, bh);
        if (!mbar_wait(&v_empty[s], ph ^ 1, abort_flag)) {
          // K_j is in flight without its V_j: drain it before leaving.
          drain_wait(&k_full[s], ph);
          break;
        }
        mbar_arrive_expect_tx(&v_full[s], L::kVBytes);
        tma_load_3d(smem + L::kV + s * L::kVBytes, &tm_v, &v_full[s], j * kTile, 0, bh);
        last_j = j;
      }
      if (*abort_flag) {
        // Wait for every copy this thread issued before the CTA releases its smem.
        drain_wait(q_full, 0);
        for (int j = max(0, last_j - kKVStages + 1); j <= last_j; ++j) {
          const uint32_t ph = (j / kKVStages) & 1;
          drain_wait(&k_full[j % kKVStages], ph);
          drain_wait(&v_full[j % kKVStages], ph);
        }
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdescQK = idesc_i8_s32(kTile, kTile);
      constexpr uint32_t kIdescPV = idesc_e4m3_f32(kTile, D);
      const uint32_t sQ_addr = smem_u32(sQ);
      bool ok = mbar_wait(q_full, 0, abort_flag);
      for (int j = 0; ok && j <= nkv; ++j) {
        if (j < nkv) {
          const int s = j % kKVStages;
          const int b = j & 1;
          ok = mbar_wait(&k_full[s], (j / kKVStages) & 1, abort_flag) &&
               mbar_wait(&s_free[b], ((j >> 1) & 1) ^ 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint32_t sK_addr = smem_u32(smem + L::kK + s * L::kKBytes);
          const uint32_t d_tmem = tmem + (b ? S_COL1 : S_COL0);
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk)
            mma_i8(d_tmem, sdesc_kmajor<D>(sQ_addr + kk * 32), sdesc_kmajor<D>(sK_addr + kk * 32), kIdescQK,
                   kk > 0 ? 1u : 0u);
          mma_commit(&s_full[b]);
          mma_commit(&k_empty[s]);
        }
        if (j > 0) {
          const int t = j - 1;
          const int s = t % kKVStages;
          const int b = t & 1;
          ok = mbar_wait(&v_full[s], (t / kKVStages) & 1, abort_flag) &&
               mbar_wait(&p_full[b], (t >> 1) & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint32_t acc = static_cast<uint32_t>(pv_acc[b]);
          const uint32_t sP_addr = smem_u32(smem + L::kP + b * L::kPBytes);
          const uint32_t sV_addr = smem_u32(smem + L::kV + s * L::kVBytes);
#pragma unroll
          for (int kk = 0; kk < kTile / 32; ++kk)
            mma_f8f6f4(tmem + O_IN, sdesc_kmajor<128>(sP_addr + kk * 32), sdesc_kmajor<128>(sV_addr + kk * 32),
                       kIdescPV, (acc | (kk > 0 ? 1u : 0u)));
          mma_commit(&p_free[b]);
          mma_commit(&v_empty[s]);
        }
      }
      if (!ok) {
        // Let every MMA issued so far finish before TMEM is released.
        mma_commit(drain_bar);
        drain_wait(drain_bar, 0);
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- softmax warps
    const int r = tid;                                  // row in tile == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const int row_g = qt * kTile + r;
    const float cq = args.sq[static_cast<size_t>(bh) * args.nblk + qt] * args.sm_log2;
    const float *sk = args.sk + static_cast<size_t>(bh) * args.nblk;
    float m_ref = -INFINITY;
    float l448 = 0.f;          // sum of 448 * P~ (the static FP8 scale folded in)
    int glen = 0;              // key tiles in the current inner group
    bool have_out = false;
    bool ok = true;

    for (int j = 0; j < nkv && ok; ++j) {
      const int b = j & 1;
      if (!mbar_wait(&s_full[b], (j >> 1) & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      uint32_t S[4][32];
      const uint32_t s_tmem = tmem + lane_base + (b ? S_COL1 : S_COL0);
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) tmem_ld_32x32b_x32(s_tmem + ch * 32, S[ch]);
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) tmem_ld_wait(S[ch]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[b]);

      // Mask keys beyond N and, for causal, keys after the query.
      const bool tail_tile = (j == nkv_all - 1) && (N & (kTile - 1));
      const bool masked_tile = tail_tile || (CAUSAL && j == qt);
      if (masked_tile) {
#pragma unroll
        for (int ch = 0; ch < 4; ++ch)
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int kv = j * kTile + ch * 32 + i;
            if (kv >= N || (CAUSAL && kv > row_g)) S[ch][i] = kMaskedScore;
          }
      }
      int smax = INT_MIN;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch)
#pragma unroll
        for (int i = 0; i < 32; ++i) smax = max(smax, static_cast<int>(S[ch][i]));
      const float c = cq * sk[j];
      const float mt = static_cast<float>(smax) * c;

      // CTA-wide vote: does any row's max grow?  Votes go through shared
      // memory and a bounded mbarrier round (no unbounded bar.sync).
      const bool grow = __any_sync(0xffffffffu, mt > m_ref);
      if (lane == 0) votes[(j & 1) * 4 + warp] = grow ? 1 : 0;
      __syncwarp();
      if (lane == 0) mbar_arrive(vote_bar);
      if (!mbar_wait(vote_bar, j & 1, abort_flag)) { ok = false; break; }
      const bool any_grow = (votes[(j & 1) * 4 + 0] | votes[(j & 1) * 4 + 1] | votes[(j & 1) * 4 + 2] |
                             votes[(j & 1) * 4 + 3]) != 0;

      if (any_grow || glen == kFlushEvery) {
        const float m_new = fmaxf(m_ref, mt);
        const float alpha = ex2_approx(m_ref - m_new);   // 0 when m_ref = -inf
        if (glen > 0) {
          // The group's last P V (tile j-1) must be complete before O_in is read.
          const int t = j - 1;
          if (!mbar_wait(&p_free[t & 1], (t >> 1) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int ch = 0; ch < D / 32; ++ch) {
            uint32_t oi[32], oo[32];
            tmem_ld_32x32b_x32(tmem + lane_base + O_IN + ch * 32, oi);
            if (have_out) {
              tmem_ld_32x32b_x32(tmem + lane_base + O_OUT + ch * 32, oo);
              tmem_ld_wait(oo);
            }
            tmem_ld_wait(oi);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float prev = have_out ? __uint_as_float(oo[i]) : 0.f;
              oo[i] = __float_as_uint((prev + __uint_as_float(oi[i])) * alpha);
            }
            tmem_st_32x32b_x32(tmem + lane_base + O_OUT + ch * 32, oo);
          }
          tmem_st_wait();
          have_out = true;
        }
        l448 *= alpha;
        m_ref = m_new;
        glen = 0;
      }

      // P~ * 448 = 2^(S2 - m + log2 448), quantised to E4M3 into P buffer b
      // (after P V of tile j-2 has finished reading it).
      if (!mbar_wait(&p_free[b], ((j >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
      const float moff = m_ref - kLog2_448;
      uint8_t *prow = smem + L::kP + b * L::kPBytes + r * 128;
      if (masked_tile)
        write_p_row<true>(S, c, moff, prow, r, l448);
      else
        write_p_row<false>(S, c, moff, prow, r, l448);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        if (warp == 0) pv_acc[b] = glen > 0 ? 1 : 0;
        mbar_arrive(&p_full[b]);
      }
      ++glen;
    }

    // ---------------------------------------------------------- epilogue
    if (ok) {
      const int t = nkv - 1;
      if (mbar_wait(&p_free[t & 1], (t >> 1) & 1, abort_flag)) {
        tc_fence_after();
        const float inv_l = 1.f / l448;
        const float *sv = args.sv + static_cast<size_t>(bh) * D;
        OutT *orow = reinterpret_cast<OutT *>(args.out) + (static_cast<size_t>(bh) * N + row_g) * D;
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t oi[32], oo[32];
          tmem_ld_32x32b_x32(tmem + lane_base + O_IN + ch * 32, oi);
          if (have_out) {
            tmem_ld_32x32b_x32(tmem + lane_base + O_OUT + ch * 32, oo);
            tmem_ld_wait(oo);
          }
          tmem_ld_wait(oi);
          uint32_t packed[16];
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float o0 = (have_out ? __uint_as_float(oo[i]) : 0.f) + __uint_as_float(oi[i]);
            const float o1 = (have_out ? __uint_as_float(oo[i + 1]) : 0.f) + __uint_as_float(oi[i + 1]);
            packed[i >> 1] = pack2_out<OutT>(o0 * sv[ch * 32 + i] * inv_l, o1 * sv[ch * 32 + i + 1] * inv_l);
          }
          if (row_g < N) {
            uint4 *dst = reinterpret_cast<uint4 *>(orow + ch * 32);
#pragma unroll
            for (int u = 0; u < 4; ++u)
              dst[u] = make_uint4(packed[4 * u], packed[4 * u + 1], packed[4 * u + 2], packed[4 * u + 3]);
          }
        }
      }
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace sattn
