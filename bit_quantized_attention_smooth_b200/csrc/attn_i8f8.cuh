// Fused attention of the INT8-QK / FP8-PV mode on sm_100a tensor cores.
//
// Method (TurboDiffusion explainer, wxsanhe.com post 64219, section 1 "hybrid
// attention"): S = Q K^T in INT8, P V in FP8, with a two-level accumulator for
// P V.  Per query tile of 128 rows and key tile j of 128 keys:
//   S_int  = q8 . k8^T                         tcgen05.mma kind::i8 -> int32 TMEM
//   S2     = S_int * s_q * s_k[j] * sm_scale * log2(e)
//   m      = reference max of the row (lazy: see below)
//   P~     = 2^(S2 - m);  l = alpha l + rowsum(P~)   FP32, one row per thread
//   p8     = E4M3(c_P P~),  c_P = 448 * 2^-tau   -> shared memory
//   O_in  (+)= p8 . v8                         tcgen05.mma kind::f8f6f4 -> fp32 TMEM
// Lazy reference max: m moves to a tile's row max only when that max exceeds
// m by more than tau = kLazyTau, so P~ <= 2^tau and c_P maps 2^tau onto 448.
// Each tile is processed in ONE speculative pass over S with the current m,
// which also tracks the row's largest exponent argument; only when some row
// of the warp went more than tau above its m (rare after the first tile) does
// the warp take the tile's row max from that argument and redo its P rows.
// The first tile is a pass against m = 0 (only its maximum is used) and a redo.
// Two-level accumulation: the tensor cores accumulate O_in over a group of
// kFlushEvery key tiles; at the start of every group the softmax threads add
// O_in into the outer FP32 accumulator O_out (registers) and the next P V
// overwrites O_in.  When a row's reference max moves, O_out is rescaled by
// alpha = 2^(m_old - m_new) through a per-row factor (O_out = beta * o_out,
// beta *= alpha), and inside a group that row's O_in in TMEM is multiplied by
// alpha (per warp, only when some lane of the warp needs it).  Both happen
// after P of the tile has been written, when the previous P V has long
// completed.  Finally
//   O = (O_out + O_in) * s_v[c] / (c_P l).
// Q scales: one per 128-token tile, or one per token (the row's thread holds
// its own scale, so the finer granularity costs nothing here).
// Per-token P (PTOK, the 8-bit bullet [17] of the SageAttention tag page): P
// is quantised against each row's maximum within the key tile, p8 =
// E4M3(448 2^(S2 - m_tile)), and the tile's P V is added into O_out with the
// factor 2^(m_tile - m) (m = the exact running max); each tile takes a max
// pass and a P pass over S, and O_in is flushed after every tile.
//
// CTA = two 128-row query tiles (A, B) of one (b, h) sharing every K/V tile;
// 12 warps in 3 warpgroups:
//   warps 0-3  softmax of tile A (thread t owns row t = TMEM lane t)
//   warps 4-7  softmax of tile B (same lanes, other TMEM columns)
//   warp 8     TMA producer (Q tiles once, then K_j and V_j through 3-stage rings)
//   warp 9     TMEM allocator and single-thread MMA issuer
//   warps 10-11 idle (they complete warpgroup 2, which gives its registers to
//              the softmax warpgroups through setmaxnreg)
// Two softmax warps per SM sub-partition hide each other's latency.  TMEM
// columns: S_A [0,128), S_B [128,256), O_in_A [256,256+D), O_in_B
// [256+D, 256+2D).  Each softmax warp reads its S once per tile (twice at
// the first tile and when it redoes one), 64 columns at a time (two 32-column loads behind one
// wait), so that the 128 outer-accumulator registers and the 64 score
// registers fit in the softmax warps' 232.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "../../include/sattn.h"
#include "ptx.cuh"

namespace sattn {

constexpr int kTile = 128;          // query rows and keys per tile
constexpr int kQTiles = 2;          // query tiles per CTA
constexpr int kKVStages = 3;
constexpr int kFlushEvery = 8;      // G: key tiles per inner accumulation group
constexpr int kAttnThreads = 384;       // 3 warpgroups
constexpr int kSoftmaxRegs = 232;       // per thread, softmax warpgroups 0 and 1
constexpr int kControlRegs = 40;        // per thread, warpgroup 2 (TMA, MMA, 2 idle warps)
// setmaxnreg moves registers between warpgroups of the block; the split must
// fit in what the block was launched with (threads x launch registers).
constexpr int kRegsNeeded = 256 * kSoftmaxRegs + 128 * kControlRegs;
constexpr float kLog2_448 = 8.807354922057604f;   // log2(448)
// Lazy reference max threshold (log2 units) and the static FP8 scale of P it
// implies: c_P = 448 * 2^-tau, log2(c_P) = log2(448) - tau.
constexpr float kLazyTau = SATTN_I8F8_LAZY_TAU;
constexpr float kLog2_CP = kLog2_448 - kLazyTau;

struct AttnArgs {
  const float *sq;   // [BH, sq_stride]: per 128-token tile (nblk) or per token (N)
  const float *sk;   // [BH, nblk]
  const float *sv;   // [BH, D]
  void *out;         // [BH, N, D] bf16 / fp16
  int N;
  int nblk;          // ceil(N / 128)
  int sq_stride;     // nblk, or N when q_per_token
  int q_per_token;   // 1: one Q scale per token
  float sm_log2;     // sm_scale * log2(e)
  const uint8_t *block_mask;   // [BH, nblk, nblk], nonzero = keep the 128x128 block; nullptr = dense
};

// Largest key-tile count of a block-sparse call: the CTA keeps its query
// tiles' rows of the block mask in shared memory.
constexpr int kMaxMaskTiles = 2048;

template <int D>
struct AttnSmem {
  static constexpr int kQBytes = kTile * D;
  static constexpr int kKBytes = kTile * D;
  static constexpr int kVBytes = D * kTile;
  static constexpr int kPBytes = kTile * kTile;
  static constexpr int kQ = 0;                                   // [2] query tiles
  static constexpr int kK = kQ + kQTiles * kQBytes;              // [stages]
  static constexpr int kV = kK + kKVStages * kKBytes;            // [stages]
  static constexpr int kP = kV + kKVStages * kVBytes;            // [2 tiles][2 buffers]
  static constexpr int kMask = kP + kQTiles * 2 * kPBytes;       // [2 tiles][kMaxMaskTiles] bytes (block-sparse calls)
  static constexpr int kBar = kMask + kQTiles * kMaxMaskTiles;
  // q_full, k_full[S], k_empty[S], v_full[S], v_empty[S], s_full[2], s_free[2],
  // p_full[2][2], pv_done[2][2], drain
  static constexpr int kNumBars = 1 + 4 * kKVStages + 2 + 2 + 4 + 4 + 1;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kBytes = kMisc + 16;
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

// Sentinel for a masked score; |q8 . k8| <= 127 * 127 * 128 < 2^22, so no
// real INT8 score takes this value.
constexpr uint32_t kMaskedScore = 0x80000000u;

__device__ __forceinline__ void mask_chunk(uint32_t (&s)[32], int kv0, int N, bool causal, int row_g) {
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int kv = kv0 + i;
    if (kv >= N || (causal && kv > row_g)) s[i] = kMaskedScore;
  }
}

// Maximum of 32 signed integer scores as a balanced tree (depth 5), so that
// the comparisons of one chunk are independent instead of one serial chain.
__device__ __forceinline__ int tree_max32(const uint32_t (&s)[32]) {
  int m[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) m[i] = max(static_cast<int>(s[i]), static_cast<int>(s[i + 16]));
#pragma unroll
  for (int w = 8; w > 0; w >>= 1)
#pragma unroll
    for (int i = 0; i < w; ++i) m[i] = max(m[i], m[i + w]);
  return m[0];
}

// 32 scores -> 32 E4M3 codes of c_P P~ (two 16-byte chunks of the row's
// 128-byte line in the 128-byte-swizzled K-major layout the MMA reads:
// 16-byte chunk c of row r lives at chunk c ^ (r mod 8)); accumulates the
// unquantised c_P P~ into sum2 (two partial sums) and, with TRACK, the
// largest exponent argument x = S2 - m + log2 c_P into xmax2.
// x = float(s) c - b with b = m - log2 c_P: the int32 -> float conversion is
// exact (|s| < 2^22) and x is one FMA, so it is within half an ulp; E4M3
// codes of P then agree with an exact computation except at rounding ties.
template <bool MASKED, bool TRACK>
__device__ __forceinline__ void p_chunk(const uint32_t (&s)[32], float c, float b, uint8_t *prow, int c16, int r,
                                        float2 &sum2, float2 &xmax2) {
  const float2 c2 = make_float2(c, c);
  const float2 nb2 = make_float2(-b, -b);
  uint32_t w[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    float2 x01 = ffma2(make_float2(static_cast<float>(static_cast<int>(s[4 * q])),
                                   static_cast<float>(static_cast<int>(s[4 * q + 1]))),
                       c2, nb2);
    float2 x23 = ffma2(make_float2(static_cast<float>(static_cast<int>(s[4 * q + 2])),
                                   static_cast<float>(static_cast<int>(s[4 * q + 3]))),
                       c2, nb2);
    if (MASKED) {
      if (s[4 * q] == kMaskedScore) x01.x = -INFINITY;
      if (s[4 * q + 1] == kMaskedScore) x01.y = -INFINITY;
      if (s[4 * q + 2] == kMaskedScore) x23.x = -INFINITY;
      if (s[4 * q + 3] == kMaskedScore) x23.y = -INFINITY;
    }
    if (TRACK) {
      xmax2.x = fmax3(xmax2.x, x01.x, x01.y);
      xmax2.y = fmax3(xmax2.y, x23.x, x23.y);
    }
    const float2 p01 = make_float2(ex2_approx(x01.x), ex2_approx(x01.y));
    const float2 p23 = make_float2(ex2_approx(x23.x), ex2_approx(x23.y));
    sum2 = fadd2(sum2, fadd2(p01, p23));
    w[q] = cvt_e4m3x4(p01, p23);
  }
  *reinterpret_cast<uint4 *>(prow + ((c16 ^ (r & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
  *reinterpret_cast<uint4 *>(prow + (((c16 + 1) ^ (r & 7)) << 4)) = make_uint4(w[4], w[5], w[6], w[7]);
}

// One pass over an S tile: P~ codes of the row into its P line in shared
// memory; returns the row's sum of c_P P~ and (into xmax2) its largest
// exponent argument x = S2 - m + log2 c_P.  S is read W columns per TMEM
// round trip (W = 64: fewer waits, more live registers; the causal kernels
// run faster with W = 32, the others with W = 64, measured).
template <int W>
__device__ __forceinline__ float p_pass(uint32_t s_tmem, float c, float b, uint8_t *prow, int r, bool masked, int kv0,
                                        int N, bool causal, int row_g, float2 &xmax2) {
  static_assert(W == 32 || W == 64, "columns per TMEM round trip");
  float2 tsum2 = make_float2(0.f, 0.f);
  if constexpr (W == 64) {
#pragma unroll 1
    for (int hh = 0; hh < 2; ++hh) {
      uint32_t s0[32], s1[32];
      tmem_ld_32x32b_x32(s_tmem + hh * 64, s0);
      tmem_ld_32x32b_x32(s_tmem + hh * 64 + 32, s1);
      tmem_ld_wait(s0);
      tmem_ld_wait(s1);
      if (masked) {
        mask_chunk(s0, kv0 + hh * 64, N, causal, row_g);
        mask_chunk(s1, kv0 + hh * 64 + 32, N, causal, row_g);
        p_chunk<true, true>(s0, c, b, prow, hh * 4, r, tsum2, xmax2);
        p_chunk<true, true>(s1, c, b, prow, hh * 4 + 2, r, tsum2, xmax2);
      } else {
        p_chunk<false, true>(s0, c, b, prow, hh * 4, r, tsum2, xmax2);
        p_chunk<false, true>(s1, c, b, prow, hh * 4 + 2, r, tsum2, xmax2);
      }
    }
  } else {
#pragma unroll 1
    for (int hh = 0; hh < 4; ++hh) {
      uint32_t s0[32];
      tmem_ld_32x32b_x32(s_tmem + hh * 32, s0);
      tmem_ld_wait(s0);
      if (masked) {
        mask_chunk(s0, kv0 + hh * 32, N, causal, row_g);
        p_chunk<true, true>(s0, c, b, prow, hh * 2, r, tsum2, xmax2);
      } else {
        p_chunk<false, true>(s0, c, b, prow, hh * 2, r, tsum2, xmax2);
      }
    }
  }
  return tsum2.x + tsum2.y;
}

// Largest valid INT8 score of the row in an S tile (masked keys read as
// kMaskedScore = INT_MIN, so a row without a valid key returns INT_MIN).
template <int W>
__device__ __forceinline__ int s_max_pass(uint32_t s_tmem, bool masked, int kv0, int N, bool causal, int row_g) {
  static_assert(W == 32 || W == 64, "columns per TMEM round trip");
  int mx = static_cast<int>(kMaskedScore);
#pragma unroll 1
  for (int hh = 0; hh < kTile / W; ++hh) {
    uint32_t s0[32], s1[32];
    tmem_ld_32x32b_x32(s_tmem + hh * W, s0);
    if constexpr (W == 64) tmem_ld_32x32b_x32(s_tmem + hh * W + 32, s1);
    tmem_ld_wait(s0);
    if constexpr (W == 64) tmem_ld_wait(s1);
    if (masked) {
      mask_chunk(s0, kv0 + hh * W, N, causal, row_g);
      if constexpr (W == 64) mask_chunk(s1, kv0 + hh * W + 32, N, causal, row_g);
    }
    mx = max(mx, tree_max32(s0));
    if constexpr (W == 64) mx = max(mx, tree_max32(s1));
  }
  return mx;
}

// PTOK = true: per-token P (see the file comment).
template <int D, bool CAUSAL, typename OutT, bool SPARSE, bool PTOK = false>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_i8f8_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const AttnArgs args) {
  using L = AttnSmem<D>;
  static_assert(D == 64 || D == 128, "head dim");
  constexpr uint32_t kTmemCols = 512;
  constexpr int kOin0 = 256;

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kBar);
  uint64_t *q_full = bars;
  uint64_t *k_full = bars + 1;
  uint64_t *k_empty = k_full + kKVStages;
  uint64_t *v_full = k_empty + kKVStages;
  uint64_t *v_empty = v_full + kKVStages;
  uint64_t *s_full = v_empty + kKVStages;   // [tile]
  uint64_t *s_free = s_full + 2;            // [tile]
  uint64_t *p_full = s_free + 2;            // [tile * 2 + buffer]
  uint64_t *pv_done = p_full + 4;           // [tile * 2 + buffer]
  uint64_t *drain_bar = pv_done + 4;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMisc + 4);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int bh = blockIdx.y;
  const int N = args.N;
  const int nkv_all = args.nblk;
  const int pair = CAUSAL ? (static_cast<int>(gridDim.x) - 1 - static_cast<int>(blockIdx.x))
                          : static_cast<int>(blockIdx.x);
  int qt_of[kQTiles], nkv_of[kQTiles];
#pragma unroll
  for (int x = 0; x < kQTiles; ++x) {
    qt_of[x] = pair * kQTiles + x;
    nkv_of[x] = qt_of[x] >= nkv_all ? 0 : (CAUSAL ? min(qt_of[x] + 1, nkv_all) : nkv_all);
  }
  const int nkv_max = max(nkv_of[0], nkv_of[1]);
  // Block-sparse skipping: key tile j of query tile x is processed iff
  // need(x, j).  The three roles walk the same sequences: the producer and the
  // MMA issuer the tiles that either query tile needs (the K/V ring advances
  // per such tile), each softmax warpgroup the tiles its query tile needs (its
  // S, P and O_in barriers advance per such tile).  Dense calls need every
  // tile below nkv_of[x], and the sequences are the tile indices.
  const uint8_t *smask = smem + L::kMask;
  auto need = [&](int x, int j) -> bool { return j < nkv_of[x] && (!SPARSE || smask[x * kMaxMaskTiles + j] != 0); };

  // ------------------------------------------------------------ set-up
  if (SPARSE) {
    uint8_t *sm = smem + L::kMask;
    for (int i = tid; i < kQTiles * nkv_all; i += kAttnThreads) {
      const int x = i / nkv_all, j = i - x * nkv_all;
      sm[x * kMaxMaskTiles + j] = qt_of[x] < nkv_all
          ? args.block_mask[(static_cast<size_t>(bh) * nkv_all + qt_of[x]) * nkv_all + j] : uint8_t(0);
    }
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (tid == 256) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kKVStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&s_full[x], 1);
      mbar_init(&s_free[x], 4);   // one arrival per softmax warp of the tile
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&p_full[i], 4);
      mbar_init(&pv_done[i], 1);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (tid == 288) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 8) {
    regs_decrease<kControlRegs>();
    if (warp == 8) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      int last_u = -1;
      const int withheld = g_withhold_k_tile;            // -1 except under the failure-path test hook
      const int nq = nkv_of[1] > 0 ? 2 : 1;             // tile B may lie past the last token
      mbar_arrive_expect_tx(q_full, nq * L::kQBytes);
      for (int x = 0; x < nq; ++x)
        tma_load_3d(smem + L::kQ + x * L::kQBytes, &tm_q, q_full, 0, qt_of[x] * kTile, bh);
      for (int j = 0, un = 0; j < nkv_max; ++j) {       // un: position in the sequence of loaded tiles
        if (SPARSE && !need(0, j) && !need(1, j)) continue;
        const int u = SPARSE ? un : j;                     // dense: every tile below nkv_max is loaded
        const int s = u % kKVStages;
        const uint32_t ph = (u / kKVStages) & 1;
        if (!mbar_wait(&k_empty[s], ph ^ 1, abort_flag)) break;
        if (u != withheld) {
          mbar_arrive_expect_tx(&k_full[s], L::kKBytes);
          tma_load_3d(smem + L::kK + s * L::kKBytes, &tm_k, &k_full[s], 0, j * kTile, bh);
        }
        if (!mbar_wait(&v_empty[s], ph ^ 1, abort_flag)) {
          if (u != withheld) drain_wait(&k_full[s], ph);   // K_j is in flight without its V_j
          break;
        }
        mbar_arrive_expect_tx(&v_full[s], L::kVBytes);
        tma_load_3d(smem + L::kV + s * L::kVBytes, &tm_v, &v_full[s], j * kTile, 0, bh);
        last_u = u;
        ++un;
      }
      if (*abort_flag) {
        // Wait for every copy this thread issued before the CTA releases its smem.
        drain_wait(q_full, 0);
        for (int u = max(0, last_u - kKVStages + 1); u <= last_u; ++u) {
          const uint32_t ph = (u / kKVStages) & 1;
          if (u != withheld) drain_wait(&k_full[u % kKVStages], ph);
          drain_wait(&v_full[u % kKVStages], ph);
        }
      }
    }
    __syncwarp();
    } else if (warp == 9) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdescQK = idesc_i8_s32(kTile, kTile);
      constexpr uint32_t kIdescPV = idesc_e4m3_f32(kTile, D);
      bool ok = mbar_wait(q_full, 0, abort_flag);
      int u = 0, prev_u = -1, prev_j = -1;               // loaded-tile sequence: this and the previous tile
      int nqk[kQTiles] = {0, 0}, npv[kQTiles] = {0, 0};  // per query tile: QK and PV products issued
      for (int j = 0; ok && j <= nkv_max; ++j) {
        const bool tail = j == nkv_max;                   // one step past the last tile: its P V only
        if (SPARSE && !tail && !need(0, j) && !need(1, j)) continue;
        if (!SPARSE) {                                     // dense: the sequences are the tile indices
          u = j;
          prev_u = prev_j = j - 1;
          nqk[0] = nqk[1] = j;
          npv[0] = npv[1] = j - 1;
        }
        bool k_ready = false, v_ready = false;
#pragma unroll
        for (int x = 0; x < kQTiles && ok; ++x) {
          if (!tail && need(x, j)) {                        // S_x = Q_x K_j^T
            const int s = u % kKVStages;
            if (!k_ready) {
              ok = mbar_wait(&k_full[s], (u / kKVStages) & 1, abort_flag);
              k_ready = true;
            }
            ok = ok && mbar_wait(&s_free[x], (nqk[x] & 1) ^ 1, abort_flag);
            if (!ok) break;
            tc_fence_after();
            const uint32_t sQ = smem_u32(smem + L::kQ + x * L::kQBytes);
            const uint32_t sK = smem_u32(smem + L::kK + s * L::kKBytes);
#pragma unroll
            for (int kk = 0; kk < D / 32; ++kk)
              mma_i8(tmem + x * kTile, sdesc_kmajor<D>(sQ + kk * 32), sdesc_kmajor<D>(sK + kk * 32), kIdescQK,
                     kk > 0 ? 1u : 0u);
            mma_commit(&s_full[x]);
            ++nqk[x];
          }
          if (prev_u >= 0 && need(x, prev_j)) {             // O_in_x (+)= P_x V of the previous loaded tile
            if (!SPARSE) npv[x] = prev_j;
            const int t = npv[x];
            const int s = prev_u % kKVStages;
            const int pb = x * 2 + (t & 1);
            if (!v_ready) {
              ok = mbar_wait(&v_full[s], (prev_u / kKVStages) & 1, abort_flag);
              v_ready = true;
            }
            ok = ok && mbar_wait(&p_full[pb], (t >> 1) & 1, abort_flag);
            if (!ok) break;
            tc_fence_after();
            const uint32_t acc = (!PTOK && (t % kFlushEvery) != 0) ? 1u : 0u;   // PTOK: one tile per O_in
            const uint32_t sP = smem_u32(smem + L::kP + pb * L::kPBytes);
            const uint32_t sV = smem_u32(smem + L::kV + s * L::kVBytes);
#pragma unroll
            for (int kk = 0; kk < kTile / 32; ++kk)
              mma_f8f6f4(tmem + kOin0 + x * D, sdesc_kmajor<128>(sP + kk * 32), sdesc_kmajor<128>(sV + kk * 32),
                         kIdescPV, acc | (kk > 0 ? 1u : 0u));
            mma_commit(&pv_done[pb]);
            ++npv[x];
          }
        }
        if (!ok) break;
        if (k_ready) mma_commit(&k_empty[u % kKVStages]);
        if (v_ready) mma_commit(&v_empty[prev_u % kKVStages]);
        if (SPARSE && !tail) {
          prev_u = u++;
          prev_j = j;
        }
      }
      if (!ok) {
        // Let every MMA issued so far finish before TMEM is released.
        mma_commit(drain_bar);
        drain_wait(drain_bar, 0);
      }
    }
    __syncwarp();
    }
  } else {
    regs_increase<kSoftmaxRegs>();
    // ---------------------------------------------------------- softmax warps
    const int x = warp >> 2;                            // query tile of this warp
    const int wq = warp & 3;                            // TMEM lane quarter
    const int r = wq * 32 + lane;                       // row in tile == TMEM lane
    const int qt = qt_of[x];
    const int nkv = nkv_of[x];
    const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t s_tmem = tmem + lane_base + x * kTile;
    const uint32_t o_tmem = tmem + lane_base + kOin0 + x * D;
    const int row_g = qt * kTile + r;
    const int sq_idx = args.q_per_token ? min(row_g, N - 1) : qt;
    const float cq = nkv > 0 ? args.sq[static_cast<size_t>(bh) * args.sq_stride + sq_idx] * args.sm_log2 : 0.f;
    const float *sk = args.sk + static_cast<size_t>(bh) * args.nblk;
    uint8_t *p_base = smem + L::kP + (x * 2) * L::kPBytes + r * 128;

    float o_out[D];
#pragma unroll
    for (int i = 0; i < D; ++i) o_out[i] = 0.f;
    float m_ref = -INFINITY;   // reference max of the row (lazy)
    float lsum = 0.f;          // sum of c_P * P~ (the static FP8 scale folded in)
    float beta = 1.f;          // the outer accumulator is beta * o_out (rescaled lazily)
    float f_pend = 1.f;        // PTOK: factor of the tile whose P V is pending, 2^(m_tile - m)
    bool ok = true;

    int n = 0;                 // key tiles processed (the S, P and O_in barriers advance per tile)
    for (int j = 0; j < nkv; ++j) {
      if (SPARSE && !smask[x * kMaxMaskTiles + j]) continue;
      if (!SPARSE) n = j;                                  // dense: the tile index
      if (!mbar_wait(&s_full[x], n & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const bool masked = ((j == nkv_all - 1) && (N & (kTile - 1))) || (CAUSAL && j == qt);
      const int kv0 = j * kTile;
      const float c = cq * sk[j];

      // P~ -> E4M3 into P buffer (n & 1), once P V of the tile two before has read it
      const int pb = x * 2 + (n & 1);
      if (!mbar_wait(&pv_done[pb], ((n >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
      uint8_t *prow = p_base + (n & 1) * L::kPBytes;
      float2 xm2 = make_float2(-INFINITY, -INFINITY);
      float tsum, m_new = m_ref, alpha = 1.f, f_tile = 1.f;
      bool moved = false;
      if constexpr (PTOK) {
        // per-token P: the tile's row max first, then the codes of 448 2^(S2 - m_tile)
        const int smax = s_max_pass<CAUSAL ? 32 : 64>(s_tmem, masked, kv0, N, CAUSAL, row_g);
        const float m_tile = smax != static_cast<int>(kMaskedScore) ? static_cast<float>(smax) * c : -INFINITY;
        // a row without a valid key in the tile (all masked) writes zero codes
        tsum = p_pass<CAUSAL ? 32 : 64>(s_tmem, c, m_tile != -INFINITY ? m_tile - kLog2_448 : 0.f, prow, r, masked,
                                        kv0, N, CAUSAL, row_g, xm2);
        m_new = fmaxf(m_ref, m_tile);
        if (m_new == -INFINITY) {                     // no valid key in the row so far
          alpha = 1.f;
          f_tile = 0.f;
        } else {
          alpha = n > 0 ? ex2_approx(m_ref - m_new) : 0.f;
          f_tile = ex2_approx(m_tile - m_new);
        }
        tsum *= f_tile;
      } else {
        // speculative pass with the current reference max (0 at the first tile,
        // which only serves to find the tile's row max)
        const float m_try = n > 0 ? m_ref : 0.f;
        tsum = p_pass<CAUSAL ? 32 : 64>(s_tmem, c, m_try - kLog2_CP, prow, r, masked, kv0, N, CAUSAL, row_g, xm2);
        // x = S2 - m + log2 c_P;  the row max moves when S2max - m > tau  <=>  xmax > log2 448
        const float xmax = fmaxf(xm2.x, xm2.y);
        const bool up = n == 0 || xmax > kLog2_448;
        moved = __any_sync(0xffffffffu, up);   // warp-uniform
        if (moved) {
          if (up) m_new = fmaxf(m_ref, xmax + (m_try - kLog2_CP));   // the tile's row max
          alpha = n > 0 ? ex2_approx(m_ref - m_new) : 0.f;
          tsum = p_pass<CAUSAL ? 32 : 64>(s_tmem, c, m_new - kLog2_CP, prow, r, masked, kv0, N, CAUSAL, row_g, xm2);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[x]);
      lsum = fmaf(alpha, lsum, tsum);

      // two-level accumulation: flush O_in at a group start (PTOK: after every
      // tile, with its factor), or rescale when the reference max moved
      const bool boundary = n > 0 && (PTOK || (n % kFlushEvery) == 0);
      const bool grow = !PTOK && n > 0 && moved;
      if (boundary || grow) {
        const int t = n - 1;
        if (!mbar_wait(&pv_done[x * 2 + (t & 1)], (t >> 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        if (boundary) {
          // O_out += O_in (both relative to m_ref; PTOK: O_in times its tile's
          // factor); o_out holds O_out / beta
          const float inv_beta = PTOK ? f_pend / beta : 1.f / beta;
#pragma unroll
          for (int ch = 0; ch < D / 32; ch += 2) {
            uint32_t o0[32], o1[32];
            tmem_ld_32x32b_x32(o_tmem + ch * 32, o0);
            tmem_ld_32x32b_x32(o_tmem + ch * 32 + 32, o1);
            tmem_ld_wait(o0);
            tmem_ld_wait(o1);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              o_out[ch * 32 + i] = fmaf(__uint_as_float(o0[i]), inv_beta, o_out[ch * 32 + i]);
              o_out[ch * 32 + 32 + i] = fmaf(__uint_as_float(o1[i]), inv_beta, o_out[ch * 32 + 32 + i]);
            }
          }
        } else {
          // the group's partial sum in TMEM must follow the new reference max
#pragma unroll 1
          for (int ch = 0; ch < D / 32; ch += 2) {
            uint32_t o0[32], o1[32];
            tmem_ld_32x32b_x32(o_tmem + ch * 32, o0);
            tmem_ld_32x32b_x32(o_tmem + ch * 32 + 32, o1);
            tmem_ld_wait(o0);
            tmem_ld_wait(o1);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              o0[i] = __float_as_uint(__uint_as_float(o0[i]) * alpha);
              o1[i] = __float_as_uint(__uint_as_float(o1[i]) * alpha);
            }
            tmem_st_32x32b_x32(o_tmem + ch * 32, o0);
            tmem_st_32x32b_x32(o_tmem + ch * 32 + 32, o1);
          }
          tmem_st_wait();
        }
      }
      beta *= alpha;
      if (__any_sync(0xffffffffu, beta < 0x1p-64f)) {
        // keep beta away from the float32 underflow range (rare)
#pragma unroll
        for (int i = 0; i < D; ++i) o_out[i] *= beta;
        beta = 1.f;
      }
      fence_proxy_async_smem();                          // P writes -> async proxy (MMA)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[pb]);
      m_ref = m_new;
      f_pend = f_tile;
      ++n;
    }

    // ---------------------------------------------------------- epilogue
    if (ok && n > 0) {
      const int t = n - 1;
      if (mbar_wait(&pv_done[x * 2 + (t & 1)], (t >> 1) & 1, abort_flag)) {
        tc_fence_after();
        const float inv_l = 1.f / lsum;
        const float *sv = args.sv + static_cast<size_t>(bh) * D;
        OutT *orow = reinterpret_cast<OutT *>(args.out) + (static_cast<size_t>(bh) * N + row_g) * D;
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t o[32];
          tmem_ld_32x32b_x32(o_tmem + ch * 32, o);
          tmem_ld_wait(o);
          uint32_t packed[16];
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float i0 = PTOK ? f_pend * __uint_as_float(o[i]) : __uint_as_float(o[i]);
            const float i1 = PTOK ? f_pend * __uint_as_float(o[i + 1]) : __uint_as_float(o[i + 1]);
            const float o0 = fmaf(beta, o_out[ch * 32 + i], i0) * sv[ch * 32 + i] * inv_l;
            const float o1 = fmaf(beta, o_out[ch * 32 + i + 1], i1) * sv[ch * 32 + i + 1] * inv_l;
            packed[i >> 1] = pack2_out<OutT>(o0, o1);
          }
          if (row_g < N) {
            uint4 *dst = reinterpret_cast<uint4 *>(orow + ch * 32);
#pragma unroll
            for (int u = 0; u < 4; ++u)
              dst[u] = make_uint4(packed[4 * u], packed[4 * u + 1], packed[4 * u + 2], packed[4 * u + 3]);
          }
        }
      }
    } else if (ok && qt < nkv_all && row_g < N) {
      // every key block of this query tile is skipped: the rows are zeros
      uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<OutT *>(args.out) + (static_cast<size_t>(bh) * N + row_g) * D);
#pragma unroll
      for (int u = 0; u < D / 8; ++u) dst[u] = make_uint4(0u, 0u, 0u, 0u);
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace sattn
