// The quantiser: one persistent kernel for every tile of Q, K and V of both
// modes.
//
// K smoothing needs the column mean of all of K before any K code, and the
// per-channel V scale the column maximum of all of V before any V code, so K
// and V are read twice: once for the statistics, once for the codes.  The
// work is one queue of items, taken in ticket order by all CTAs; per head h:
//   A(h) = statistics items of K (then, I8QK_F8PV, of V) of h, then Q tiles of h
//   B(h) = K tiles of h, then V tiles of h
// A tile is 128 tokens x d of one tensor of one (b,h); a statistics item is
// kStatBlocks consecutive tiles, reduced over the CTA and published once.
// The order is A(0) .. A(L-1), then A(h+L) B(h) for h = 0, 1, ..: a head's K
// and V are quantised L heads after their statistics were read, so that
// their second read comes from L2 (the host picks L so that L + 1 heads' K
// and V stay well inside the 126 MB L2, and so that the items taken but not
// yet finished by all CTAs -- about four per CTA -- fit between a head's last
// statistics item and its first K tile; the statistics reads carry an
// evict-last hint and every other read evict-first).  HBM then sees each
// input byte once.
//
// A K (V) tile waits for its head's K (V) statistics: at the end of every
// statistics item, each of the d/32 warps that add into the head's
// accumulators fences its atomics and bumps the tensor's done counter of the
// head once; before the K/V tile is handed to the compute warps, the producer
// spins (bounded) until that counter reaches d/32 times the tensor's number
// of statistics items.  The queue order
// makes the wait finite: an item waits only for items with smaller tickets,
// each already taken by a running CTA that processes its items in ticket
// order (the tiles of one item in consecutive stages); the unfinished item
// with the smallest ticket never waits.
//
// CTA: 8 compute warps + 1 producer warp.  The producer warp takes tickets,
// bulk-copies (cp.async.bulk, no multicast) each tile into a ring of
// kQuantStages shared-memory stages and, for a K or V tile, waits for the
// head's statistics and puts the per-channel mu or s_v beside the stage; the
// compute warps process the stages in order and release each with one arrive
// per warp.  Two CTAs per SM.
#pragma once

#include "quant_i8f8.cuh"
#include "quant_nvfp4.cuh"

namespace sattn {

constexpr int kQuantStages = 3;
constexpr int kQuantThreads = kQuantConsumers + 32;
constexpr int kStatBlocks = 8;         // 128-token blocks per statistics item
constexpr int kChanRows = 3;           // per-channel values a stage carries

enum QuantScheme : int { kSchemeI8Block = 0, kSchemeI8Token = 1, kSchemeNvfp4 = 2, kSchemeMxfp4 = 3 };

// The FP4 schemes (NVFP4 and its MXFP4 ablation) share the tiles, the layout
// and the queue: K statistics only (V needs no per-channel scale).
__host__ __device__ constexpr bool fp4_scheme(int scheme) {
  return scheme == kSchemeNvfp4 || scheme == kSchemeMxfp4;
}
enum QuantItemKind : int { kItemKStat = 0, kItemVStat = 1, kItemQ = 2, kItemK = 3, kItemV = 4, kItemEnd = 5 };

// A queue item, or (in a stage slot) one tile of it: blocks blk .. blk +
// nsub - 1 of one tensor of head bh; a slot holds block blk, its `rows`, and
// its index `sub` within the item.
struct QuantItem {
  int kind, bh, blk, rows, sub, nsub;
};

// Failure-path test hook: when non-zero, no head's statistics ever count as
// ready (the producers' waits for them run out).
__device__ int g_withhold_statistics = 0;

struct QuantArgs {
  const void *q, *k, *v;
  uint8_t *q8, *k8, *vt8;      // codes
  uint8_t *sq, *sk, *sv;       // scales: float32 (I8QK_F8PV) or E4M3 blocks (NVFP4)
  float *mu;
  double *ksum;
  unsigned *vmax;
  unsigned *done;              // [2][BH] statistics publications per head: K, then V
  unsigned *ticket;            // next ticket
  int BH, N, nblk, nv;
  int lag;                     // heads whose statistics are read before B(0)
};

// Statistics items per head: K (and, I8QK_F8PV, V) in groups of kStatBlocks blocks.
__host__ __device__ __forceinline__ int quant_stat_items(int scheme, int nblk) {
  const int groups = (nblk + kStatBlocks - 1) / kStatBlocks;
  return fp4_scheme(scheme) ? groups : 2 * groups;
}

// Number of items in the queue.
__host__ __device__ __forceinline__ long long quant_items(int scheme, int BH, int nblk) {
  return static_cast<long long>(BH) * (quant_stat_items(scheme, nblk) + 3 * nblk);
}

// Ticket -> item, in the order given in the file comment, with lag L =
// min(lag, BH): A(0) .. A(L-1), then for h = 0 .. BH-1: A(h+L) (while h+L <
// BH) followed by B(h).
__host__ __device__ __forceinline__ QuantItem quant_item(int scheme, unsigned t, int BH, int nblk, int N, int lag) {
  const int nstat = quant_stat_items(scheme, nblk);
  const unsigned a = static_cast<unsigned>(nstat + nblk);   // |A(h)|
  const unsigned b = static_cast<unsigned>(2 * nblk);       // |B(h)|
  const unsigned L = static_cast<unsigned>(lag < BH ? lag : BH);
  const unsigned paired = static_cast<unsigned>(BH) - L;    // B(h) preceded by A(h+L)
  QuantItem it;
  it.kind = kItemEnd;
  it.bh = it.blk = it.rows = it.sub = 0;
  it.nsub = 1;
  if (static_cast<long long>(t) >= quant_items(scheme, BH, nblk)) return it;
  int h;
  unsigned r;
  bool in_a;
  if (t < L * a) {
    h = static_cast<int>(t / a);
    r = t % a;
    in_a = true;
  } else if (t - L * a < paired * (a + b)) {
    const unsigned p = (t - L * a) / (a + b);
    const unsigned rr = (t - L * a) % (a + b);
    in_a = rr < a;
    h = static_cast<int>(in_a ? p + L : p);
    r = in_a ? rr : rr - a;
  } else {
    const unsigned t3 = t - L * a - paired * (a + b);
    h = static_cast<int>(paired + t3 / b);
    r = t3 % b;
    in_a = false;
  }
  if (in_a) {
    if (r < static_cast<unsigned>(nstat)) {
      const int groups = (nblk + kStatBlocks - 1) / kStatBlocks;   // K statistics first, then V
      const int g = static_cast<int>(r) % groups;
      it.kind = static_cast<int>(r) < groups ? kItemKStat : kItemVStat;
      it.blk = g * kStatBlocks;
      it.nsub = nblk - it.blk < kStatBlocks ? nblk - it.blk : kStatBlocks;
    } else {
      it.kind = kItemQ;
      it.blk = static_cast<int>(r) - nstat;
    }
  } else {
    it.kind = r < static_cast<unsigned>(nblk) ? kItemK : kItemV;
    it.blk = static_cast<int>(r % static_cast<unsigned>(nblk));
  }
  it.bh = h;
  it.rows = N - it.blk * kBlockTokens < kBlockTokens ? N - it.blk * kBlockTokens : kBlockTokens;
  return it;
}

template <int D>
struct QuantSmem {
  static constexpr int kTileBytes = kBlockTokens * D * 2;
  static constexpr int kTiles = 0;
  // per stage, kChanRows x D floats: mu (K tiles) or s_v, RN(r (1 - 2^-20)),
  // RN(r (1 + 2^-20)) with r = RN(1/s_v) (V tiles)
  static constexpr int kChan = kTiles + kQuantStages * kTileBytes;
  static constexpr int kScratch = kChan + kQuantStages * kChanRows * D * 4;
  static constexpr int kSlots = kScratch + ((static_cast<int>(sizeof(QuantScratch<D>)) + 15) / 16) * 16;
  static constexpr int kBars = kSlots + ((kQuantStages * static_cast<int>(sizeof(QuantItem)) + 7) / 8) * 8;
  static constexpr int kFlags = kBars + 2 * kQuantStages * 8;
  static constexpr int kBytes = kFlags + 16;
  static constexpr int kAlloc = kBytes + 128;      // room to align the base to 128 bytes
};

// Bounded spin of one thread until *count >= target (acquire at GPU scope).
__device__ __forceinline__ bool wait_count(const unsigned *count, unsigned target, volatile int *abort_flag) {
  if (ld_acquire_gpu(count) >= target) return true;
  const long long t0 = clock64();
  while (ld_acquire_gpu(count) < target) {
    if (*abort_flag) return false;
    if (clock64() - t0 > g_wait_limit) {
      atomicOr(&g_error_word, kErrWaitTimeout);
      *abort_flag = 1;
      return false;
    }
    __nanosleep(100);
  }
  return true;
}

// The compute warps' work on one tile.
template <typename T, int D, int SCHEME>
__device__ __forceinline__ void quant_tile(const QuantArgs &a, const QuantItem &it, const T *tile, const float *cs,
                                           QuantScratch<D> &sc, uint64_t *empty) {
  constexpr bool NV = fp4_scheme(SCHEME);
  constexpr bool MX = SCHEME == kSchemeMxfp4;
  const size_t hrow = static_cast<size_t>(it.bh) * a.N;   // first row of the head
  const int tok0 = it.blk * kBlockTokens;
  const size_t sblk = static_cast<size_t>(it.bh) * a.nblk + it.blk;
  switch (it.kind) {
    case kItemKStat:
      stat_tile<T, D, false>(tile, it.rows, it.sub == 0, sc, empty);
      if (it.sub == it.nsub - 1)
        stat_publish<D, false>(sc, a.ksum + static_cast<size_t>(it.bh) * D, nullptr, a.done + it.bh);   // K
      break;
    case kItemVStat:
      stat_tile<T, D, true>(tile, it.rows, it.sub == 0, sc, empty);
      if (it.sub == it.nsub - 1)
        stat_publish<D, true>(sc, nullptr, a.vmax + static_cast<size_t>(it.bh) * D, a.done + a.BH + it.bh);   // V
      break;
    case kItemQ:
      if (NV)
        nvfp4_rows_tile<T, D, false, MX>(tile, it.rows, cs, sc.e4m3_recip, a.q8 + (hrow + tok0) * (D / 2),
                                     a.sq + sblk * (D / 64) * 512, empty);
      else if (SCHEME == kSchemeI8Token)
        q_token_tile<T, D>(tile, it.rows, sc, reinterpret_cast<int8_t *>(a.q8) + (hrow + tok0) * D,
                           reinterpret_cast<float *>(a.sq) + hrow + tok0, empty);
      else
        qk_block_tile<T, D, false>(tile, it.rows, cs, sc, reinterpret_cast<int8_t *>(a.q8) + (hrow + tok0) * D,
                                   reinterpret_cast<float *>(a.sq) + sblk, empty);
      break;
    case kItemK:
      if (NV)
        nvfp4_rows_tile<T, D, true, MX>(tile, it.rows, cs, sc.e4m3_recip, a.k8 + (hrow + tok0) * (D / 2),
                                    a.sk + sblk * (D / 64) * 512, empty);
      else
        qk_block_tile<T, D, true>(tile, it.rows, cs, sc, reinterpret_cast<int8_t *>(a.k8) + (hrow + tok0) * D,
                                  reinterpret_cast<float *>(a.sk) + sblk, empty);
      break;
    default:   // kItemV
      if (NV)
        nvfp4_v_tile<T, D, MX>(tile, it.rows, tok0, a.nv, sc.e4m3_recip,
                           a.vt8 + static_cast<size_t>(it.bh) * D * (a.nv / 2), a.sv + sblk * 1024, empty);
      else
        v_tile<T, D>(tile, it.rows, tok0, a.nv, cs, a.vt8 + static_cast<size_t>(it.bh) * D * a.nv, empty);
      break;
  }
}

template <typename T, int D, int SCHEME>
__global__ void __launch_bounds__(kQuantThreads, 2) quant_kernel(const QuantArgs a) {
  using L = QuantSmem<D>;
  constexpr bool NV = fp4_scheme(SCHEME);
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  QuantScratch<D> &sc = *reinterpret_cast<QuantScratch<D> *>(smem + L::kScratch);
  float *chan = reinterpret_cast<float *>(smem + L::kChan);
  QuantItem *slot = reinterpret_cast<QuantItem *>(smem + L::kSlots);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::kBars);
  uint64_t *empty = full + kQuantStages;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kFlags);
  volatile int *go = abort_flag + 1;               // go[0], go[1]: per-tile decision of thread 0

  if (threadIdx.x == 0) {
    for (int s = 0; s < kQuantStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kQuantWarps);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (NV) fill_e4m3_recip(sc.e4m3_recip);
  __syncthreads();

  if (threadIdx.x >= kQuantConsumers) {
    // ------------------------------------------------------------ producer warp
    // Lane 0 takes tickets (one ahead, so that the atomic's latency overlaps
    // the item's copies) and issues one copy per tile of the item; for a K or
    // V tile the whole warp then waits for the head's statistics and writes
    // the stage's per-channel mu (K) or s_v (V), before the stage's `full`
    // barrier is arrived on: the compute warps find everything in shared
    // memory.
    const int lane = threadIdx.x & 31;
    // every statistics item of a tensor is published once per warp that issued accumulator atomics
    const unsigned stats_target = static_cast<unsigned>((a.nblk + kStatBlocks - 1) / kStatBlocks) * (D / 32) +
                                  (g_withhold_statistics ? 1u : 0u);
    uint64_t keep = 0, stream = 0;
    unsigned next = 0;
    if (lane == 0) {
      keep = make_l2_policy_evict_last();
      stream = make_l2_policy_evict_first();
      next = atomicAdd(a.ticket, 1u);
    }
    int i = 0;                                     // stage uses issued
    bool stop = false;
    while (!stop) {
      const QuantItem item = quant_item(SCHEME, __shfl_sync(0xffffffffu, next, 0), a.BH, a.nblk, a.N, a.lag);
      if (lane == 0 && item.kind != kItemEnd) next = atomicAdd(a.ticket, 1u);
      for (int sub = 0; sub < item.nsub; ++sub) {
        const int s = i % kQuantStages;
        bool ok = true;
        if (lane == 0 && i >= kQuantStages) ok = mbar_wait(&empty[s], ((i / kQuantStages) - 1) & 1, abort_flag);
        if (!__shfl_sync(0xffffffffu, ok, 0)) {
          stop = true;
          break;
        }
        QuantItem it = item;
        it.blk = item.blk + sub;
        it.sub = sub;
        it.rows = a.N - it.blk * kBlockTokens < kBlockTokens ? a.N - it.blk * kBlockTokens : kBlockTokens;
        if (it.kind == kItemEnd) {
          if (lane == 0) {
            slot[s] = it;
            mbar_arrive(&full[s]);
          }
          ++i;
          stop = true;
          break;
        }
        if (lane == 0) {
          slot[s] = it;
          const void *base = (it.kind == kItemQ) ? a.q : (it.kind == kItemK || it.kind == kItemKStat) ? a.k : a.v;
          const T *src = static_cast<const T *>(base) +
                         (static_cast<size_t>(it.bh) * a.N + static_cast<size_t>(it.blk) * kBlockTokens) * D;
          const uint32_t bytes = static_cast<uint32_t>(it.rows) * D * sizeof(T);
          mbar_expect_tx(&full[s], bytes);
          bulk_load(smem + L::kTiles + s * L::kTileBytes, src, bytes, &full[s],
                    (it.kind == kItemKStat || it.kind == kItemVStat) ? keep : stream);
        }
        if (it.kind == kItemK || (!NV && it.kind == kItemV)) {
          bool ready = true;
          if (lane == 0)
            ready = wait_count(a.done + (it.kind == kItemV ? a.BH : 0) + it.bh, stats_target, abort_flag);
          if (__shfl_sync(0xffffffffu, ready, 0)) {
            float *cs = chan + s * kChanRows * D;
#pragma unroll
            for (int c = lane; c < D; c += 32) {
              const size_t hc = static_cast<size_t>(it.bh) * D + c;
              if (it.kind == kItemK) {
                const float mu = static_cast<float>(__ldcg(a.ksum + hc) / static_cast<double>(a.N));
                cs[c] = mu;
                if (it.blk == 0) a.mu[hc] = mu;
              } else {
                const float m = __uint_as_float(__ldcg(a.vmax + hc));
                const float sv = m == 0.f ? 1.f : __fdiv_rn(m, 448.f);
                float rlo, rhi;
                const bool fast = bracket(sv, rlo, rhi);
                cs[c] = sv;
                cs[D + c] = fast ? rlo : 0.f;       // 0: no safe bracket, take the quotient
                cs[2 * D + c] = fast ? rhi : 0.f;
                if (it.blk == 0) reinterpret_cast<float *>(a.sv)[hc] = sv;
              }
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&full[s]);      // release: the slot and the stage's channel values
        ++i;
        if (__shfl_sync(0xffffffffu, *abort_flag, 0)) {
          stop = true;
          break;
        }
      }
    }
    // every copy this warp issued lands before the CTA can exit
    if (lane == 0)
      for (int u = i > kQuantStages ? i - kQuantStages : 0; u < i; ++u)
        drain_wait(&full[u % kQuantStages], (u / kQuantStages) & 1);
    return;
  }

  // -------------------------------------------------------------- compute warps
  const int ct = threadIdx.x;
  for (int i = 0;; ++i) {
    const int s = i % kQuantStages;
    const uint32_t par = (i / kQuantStages) & 1;
    if (ct == 0) {
      bool ok = mbar_wait(&full[s], par, abort_flag) && !*abort_flag;
      if (ok && slot[s].kind == kItemEnd) ok = false;
      go[i & 1] = ok ? 1 : 0;
    }
    __syncwarp();
    named_bar_sync(kQuantBar, kQuantConsumers);
    if (!go[i & 1]) break;
    mbar_try_wait(&full[s], par);                  // completed: orders this thread after the copy
    const QuantItem it = slot[s];
    quant_tile<T, D, SCHEME>(a, it, reinterpret_cast<const T *>(smem + L::kTiles + s * L::kTileBytes),
                             chan + s * kChanRows * D,
                             sc, &empty[s]);
  }
}

}  // namespace sattn
