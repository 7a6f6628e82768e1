// C-ABI of libsattn.so: argument validation, workspace layout, TMA tensor
// maps and kernel launches.  Declarations and contracts: include/sattn.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <climits>
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/sattn.h"
#include "attn_i8f8.cuh"
#include "attn_nvfp4.cuh"
#include "debug_scores.cuh"
#include "quant_fused.cuh"

namespace sattn {
namespace {

constexpr size_t kSectionAlign = 1024;
constexpr int kMaxDevices = 64;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Kernels this library has launched since load (or the last reset).
std::atomic<unsigned long long> g_launches{0};

constexpr int kFlagBits = SATTN_FP16_IO | SATTN_Q_PER_TOKEN | SATTN_P_PER_TOKEN;

int base_mode(int mode) { return mode & ~kFlagBits; }

bool valid_mode(int mode) {
  const int base = base_mode(mode);
  return (mode & ~(kFlagBits | 0xFF)) == 0 && (base == SATTN_I8QK_F8PV || base == SATTN_NVFP4 || base == SATTN_MXFP4);
}

bool q_per_token(int mode) { return (mode & SATTN_Q_PER_TOKEN) != 0; }
bool p_per_token(int mode) { return (mode & SATTN_P_PER_TOKEN) != 0; }

int check_shape(int B, int H, int N, int d, int mode) {
  if (B < 1 || H < 1 || N < 1) return SATTN_ERR_INVALID_ARG;
  if (!valid_mode(mode)) return SATTN_ERR_INVALID_ARG;
  if ((q_per_token(mode) || p_per_token(mode)) && base_mode(mode) != SATTN_I8QK_F8PV) return SATTN_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return SATTN_ERR_UNSUPPORTED;
  const long long total = static_cast<long long>(B) * H * N * d;
  if (total >= (1LL << 31) || static_cast<long long>(B) * H >= 65536) return SATTN_ERR_UNSUPPORTED;
  return SATTN_OK;
}

bool aligned16(const void *p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The FP4 modes (NVFP4 and MXFP4) share the workspace layout and the kernels.
bool is_nvfp4(int mode) { return base_mode(mode) == SATTN_NVFP4 || base_mode(mode) == SATTN_MXFP4; }
bool is_mxfp4(int mode) { return base_mode(mode) == SATTN_MXFP4; }

// The vmax section holds vmax[BH][d] and then the quantiser's work counters:
// done[2][BH] (K, V statistics) and the ticket counter.  Offset of done from
// the section start.
size_t counters_offset(size_t BH, int d) { return BH * d * sizeof(unsigned); }

// NVFP4 workspace: q8/k8/vt8 hold the packed E2M1 codes of Q, K - mean and
// V^T (N rounded up to 32 tokens), sq/sk/sv the E4M3 scale blocks of Q, K, V.
sattn_ws_layout_t make_layout_nvfp4(int B, int H, int N, int d) {
  sattn_ws_layout_t L;
  std::memset(&L, 0xFF, sizeof(L));
  const size_t BH = static_cast<size_t>(B) * H;
  L.nblk = (N + kBlockTokens - 1) / kBlockTokens;
  L.nv = (N + 31) / 32 * 32;
  size_t off = 0;
  L.q8 = off;   off = align_up(off + BH * N * d / 2, kSectionAlign);
  L.k8 = off;   off = align_up(off + BH * N * d / 2, kSectionAlign);
  L.vt8 = off;  off = align_up(off + BH * d * L.nv / 2, kSectionAlign);
  L.sq = off;   off = align_up(off + BH * L.nblk * (d / 64) * 512, kSectionAlign);
  L.sk = off;   off = align_up(off + BH * L.nblk * (d / 64) * 512, kSectionAlign);
  L.sv = off;   off = align_up(off + BH * L.nblk * 1024, kSectionAlign);
  L.mu = off;   off = align_up(off + BH * d * sizeof(float), kSectionAlign);
  L.ksum = off; off += BH * d * sizeof(double);
  L.vmax = off; off = align_up(off + counters_offset(BH, d) + (2 * BH + 1) * sizeof(unsigned), kSectionAlign);
  L.total = off;
  return L;
}

// I8F8 workspace; with per-token Q scales, sq holds N floats per head instead
// of one per 128-token block.
sattn_ws_layout_t make_layout_i8f8(int B, int H, int N, int d, bool per_token) {
  sattn_ws_layout_t L;
  std::memset(&L, 0xFF, sizeof(L));
  const size_t BH = static_cast<size_t>(B) * H;
  L.nblk = (N + kBlockTokens - 1) / kBlockTokens;
  L.nv = (N + 15) / 16 * 16;
  size_t off = 0;
  L.q8 = off;   off = align_up(off + BH * N * d, kSectionAlign);
  L.k8 = off;   off = align_up(off + BH * N * d, kSectionAlign);
  L.vt8 = off;  off = align_up(off + BH * d * L.nv, kSectionAlign);
  L.sq = off;   off = align_up(off + BH * (per_token ? N : L.nblk) * sizeof(float), kSectionAlign);
  L.sk = off;   off = align_up(off + BH * L.nblk * sizeof(float), kSectionAlign);
  L.sv = off;   off = align_up(off + BH * d * sizeof(float), kSectionAlign);
  L.mu = off;   off = align_up(off + BH * d * sizeof(float), kSectionAlign);
  L.ksum = off; off += BH * d * sizeof(double);
  L.vmax = off; off = align_up(off + counters_offset(BH, d) + (2 * BH + 1) * sizeof(unsigned), kSectionAlign);
  L.total = off;
  return L;
}

sattn_ws_layout_t make_layout(int B, int H, int N, int d, int mode) {
  return is_nvfp4(mode) ? make_layout_nvfp4(B, H, N, d) : make_layout_i8f8(B, H, N, d, q_per_token(mode));
}

// ---------------------------------------------------------------- tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// The current CUDA context (driver handle), looked up like the encoder above.
// The library's per-device caches (owned workspace, host pipeline, address of
// the no-alloc array) remember the context they were made in: after
// cudaDeviceReset, or under another context, they are rebuilt instead of
// reused (the old pointers died with their context and are not freed).
using CtxGetCurrentFn = CUresult (*)(CUcontext *);
CUcontext current_context() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  CUcontext c = nullptr;
  if (fn == nullptr || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// 3-D uint8 tensor [dim2][dim1][dim0] (dim0 contiguous), box {box0, box1, 1}.
bool make_map_u8(CUtensorMap *map, const void *base, uint64_t dim0, uint64_t dim1, uint64_t dim2, uint64_t stride1,
                 uint64_t stride2, uint32_t box0, uint32_t box1, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {dim0, dim1, dim2};
  const cuuint64_t strides[2] = {stride1, stride2};
  const cuuint32_t box[3] = {box0, box1, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// SMs of the current device (persistent grids).
int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  return n;
}

// The quantiser (quant_fused.cuh): zeroes the statistics accumulators and
// work counters (and, NVFP4, the V scale blocks, whose rows past d are never
// written), then one persistent launch of two CTAs per SM.
template <typename T, int D, int SCHEME>
int launch_quant(const void *q, const void *k, const void *v, int BH, int N, uint8_t *ws, const sattn_ws_layout_t &L,
                 cudaStream_t st) {
  if (cudaMemsetAsync(ws + L.ksum, 0, L.total - L.ksum, st) != cudaSuccess) return SATTN_ERR_CUDA;
  if (fp4_scheme(SCHEME) &&
      cudaMemsetAsync(ws + L.sv, 0, static_cast<size_t>(BH) * L.nblk * 1024, st) != cudaSuccess)
    return SATTN_ERR_CUDA;
  const int sms = sm_count();
  if (sms <= 0) return SATTN_ERR_CUDA;
  auto kern = quant_kernel<T, D, SCHEME>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, QuantSmem<D>::kAlloc) != cudaSuccess)
    return SATTN_ERR_CUDA;
  QuantArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.q8 = ws + L.q8;
  a.k8 = ws + L.k8;
  a.vt8 = ws + L.vt8;
  a.sq = ws + L.sq;
  a.sk = ws + L.sk;
  a.sv = ws + L.sv;
  a.mu = reinterpret_cast<float *>(ws + L.mu);
  a.ksum = reinterpret_cast<double *>(ws + L.ksum);
  a.vmax = reinterpret_cast<unsigned *>(ws + L.vmax);
  a.done = reinterpret_cast<unsigned *>(ws + L.vmax + counters_offset(BH, D));
  a.ticket = a.done + 2 * BH;
  a.BH = BH;
  a.N = N;
  a.nblk = L.nblk;
  a.nv = L.nv;
  const long long items = quant_items(SCHEME, BH, L.nblk);
  const int grid = static_cast<int>(std::min<long long>(2LL * sms, items));
  // Lag (in heads) between a head's statistics and its K/V codes: enough for
  // the items in flight (about four per CTA) to fit in between, capped so that
  // the K and V of the lagged heads (read once, re-read from L2) stay within
  // 64 MB of the 126 MB L2.
  const long long per_head = quant_stat_items(SCHEME, L.nblk) + L.nblk;   // |A(h)|
  const long long kv_head = 2LL * N * D * static_cast<long long>(sizeof(T));
  const long long want = (4LL * grid + per_head - 1) / per_head;
  const long long cap = std::max<long long>(1, (64LL << 20) / kv_head);
  a.lag = static_cast<int>(std::max<long long>(1, std::min(want, cap)));
  kern<<<grid, kQuantThreads, QuantSmem<D>::kAlloc, st>>>(a);
  g_launches += 1;
  return cudaGetLastError() == cudaSuccess ? SATTN_OK : SATTN_ERR_CUDA;
}

template <int D, bool CAUSAL, typename OutT, bool SPARSE, bool MX>
int launch_attn_nvfp4(const uint8_t *ws, const sattn_ws_layout_t &L, void *out, int BH, int N, float sm_scale,
                      const uint8_t *block_mask, cudaStream_t st) {
  using SL = AttnF4Smem<D>;
  CUtensorMap tq, tk, tv;
  const CUtensorMapSwizzle swqk = D == 128 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
  const uint64_t rowb = D / 2;
  if (!make_map_u8(&tq, ws + L.q8, rowb, N, BH, rowb, static_cast<uint64_t>(N) * rowb, rowb, kTile, swqk) ||
      !make_map_u8(&tk, ws + L.k8, rowb, N, BH, rowb, static_cast<uint64_t>(N) * rowb, rowb, kTile, swqk) ||
      !make_map_u8(&tv, ws + L.vt8, (N + 1) / 2, D, BH, L.nv / 2, static_cast<uint64_t>(L.nv / 2) * D, kTile / 2, D,
                   CU_TENSOR_MAP_SWIZZLE_64B))
    return SATTN_ERR_CUDA;
  // More than half of the SM's shared memory: one CTA (and its 512 TMEM
  // columns) per SM.
  const int smem = SL::kAlloc > 118 * 1024 ? SL::kAlloc : 118 * 1024;
  auto kern = attn_nvfp4_kernel<D, CAUSAL, OutT, SPARSE, MX>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return SATTN_ERR_CUDA;
  AttnF4Args a;
  a.sfq = ws + L.sq;
  a.sfk = ws + L.sk;
  a.sfv = ws + L.sv;
  a.out = out;
  a.N = N;
  a.nblk = L.nblk;
  a.sm_log2 = static_cast<float>(static_cast<double>(sm_scale) * 1.4426950408889634);
  a.block_mask = block_mask;
  kern<<<dim3(L.nblk, BH), kF4Threads, smem, st>>>(tq, tk, tv, a);
  g_launches += 1;
  return cudaGetLastError() == cudaSuccess ? SATTN_OK : SATTN_ERR_CUDA;
}

template <int D, bool CAUSAL, typename OutT, bool SPARSE, bool PTOK>
int launch_attn_i8f8(const uint8_t *ws, const sattn_ws_layout_t &L, void *out, int BH, int N, float sm_scale,
                     bool per_token, const uint8_t *block_mask, cudaStream_t st) {
  using SL = AttnSmem<D>;
  CUtensorMap tq, tk, tv;
  const CUtensorMapSwizzle swqk = D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  if (!make_map_u8(&tq, ws + L.q8, D, N, BH, D, static_cast<uint64_t>(N) * D, D, kTile, swqk) ||
      !make_map_u8(&tk, ws + L.k8, D, N, BH, D, static_cast<uint64_t>(N) * D, D, kTile, swqk) ||
      !make_map_u8(&tv, ws + L.vt8, N, D, BH, L.nv, static_cast<uint64_t>(L.nv) * D, kTile, D,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return SATTN_ERR_CUDA;
  // More than half of the SM's shared memory: one CTA (and its 512 TMEM
  // columns) per SM.
  const int smem = SL::kAlloc > 118 * 1024 ? SL::kAlloc : 118 * 1024;
  auto kern = attn_i8f8_kernel<D, CAUSAL, OutT, SPARSE, PTOK>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return SATTN_ERR_CUDA;
  // The kernel's setmaxnreg split must fit in its launch registers, or its
  // register increase would never be granted.
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return SATTN_ERR_CUDA;
  if (static_cast<long long>(fa.numRegs) * kAttnThreads < kRegsNeeded) return SATTN_ERR_CUDA;
  AttnArgs a;
  a.sq = reinterpret_cast<const float *>(ws + L.sq);
  a.sk = reinterpret_cast<const float *>(ws + L.sk);
  a.sv = reinterpret_cast<const float *>(ws + L.sv);
  a.out = out;
  a.N = N;
  a.nblk = L.nblk;
  a.sq_stride = per_token ? N : L.nblk;
  a.q_per_token = per_token ? 1 : 0;
  a.sm_log2 = static_cast<float>(static_cast<double>(sm_scale) * 1.4426950408889634);
  a.block_mask = block_mask;
  kern<<<dim3((L.nblk + kQTiles - 1) / kQTiles, BH), kAttnThreads, smem, st>>>(tq, tk, tv, a);
  g_launches += 1;
  return cudaGetLastError() == cudaSuccess ? SATTN_OK : SATTN_ERR_CUDA;
}

template <int D, typename OutT>
int dispatch_attn(const uint8_t *ws, const sattn_ws_layout_t &L, void *out, int BH, int N, int causal, float sm,
                  int mode, const uint8_t *mask, cudaStream_t st) {
  if (is_mxfp4(mode)) {
    if (mask != nullptr)
      return causal ? launch_attn_nvfp4<D, true, OutT, true, true>(ws, L, out, BH, N, sm, mask, st)
                    : launch_attn_nvfp4<D, false, OutT, true, true>(ws, L, out, BH, N, sm, mask, st);
    return causal ? launch_attn_nvfp4<D, true, OutT, false, true>(ws, L, out, BH, N, sm, nullptr, st)
                  : launch_attn_nvfp4<D, false, OutT, false, true>(ws, L, out, BH, N, sm, nullptr, st);
  }
  if (is_nvfp4(mode)) {
    if (mask != nullptr)
      return causal ? launch_attn_nvfp4<D, true, OutT, true, false>(ws, L, out, BH, N, sm, mask, st)
                    : launch_attn_nvfp4<D, false, OutT, true, false>(ws, L, out, BH, N, sm, mask, st);
    return causal ? launch_attn_nvfp4<D, true, OutT, false, false>(ws, L, out, BH, N, sm, nullptr, st)
                  : launch_attn_nvfp4<D, false, OutT, false, false>(ws, L, out, BH, N, sm, nullptr, st);
  }
  const bool pt = q_per_token(mode);
  if (p_per_token(mode)) {
    if (mask != nullptr) return SATTN_ERR_UNSUPPORTED;   // per-token P: dense calls only
    return causal ? launch_attn_i8f8<D, true, OutT, false, true>(ws, L, out, BH, N, sm, pt, nullptr, st)
                  : launch_attn_i8f8<D, false, OutT, false, true>(ws, L, out, BH, N, sm, pt, nullptr, st);
  }
  if (mask != nullptr)
    return causal ? launch_attn_i8f8<D, true, OutT, true, false>(ws, L, out, BH, N, sm, pt, mask, st)
                  : launch_attn_i8f8<D, false, OutT, true, false>(ws, L, out, BH, N, sm, pt, mask, st);
  return causal ? launch_attn_i8f8<D, true, OutT, false, false>(ws, L, out, BH, N, sm, pt, nullptr, st)
                : launch_attn_i8f8<D, false, OutT, false, false>(ws, L, out, BH, N, sm, pt, nullptr, st);
}

// Checks of a block-sparse call beyond those of the dense one.
int check_block_mask(int N, const void *block_mask) {
  if (block_mask == nullptr) return SATTN_ERR_INVALID_ARG;
  if ((N + kTile - 1) / kTile > kMaxMaskTiles) return SATTN_ERR_UNSUPPORTED;
  return SATTN_OK;
}

int fwd_quantized_impl(const void *workspace, size_t ws_bytes, void *out, int B, int H, int N, int d, int causal,
                       float sm_scale, int mode, const uint8_t *mask, sattn_stream_t stream) {
  const int st = check_shape(B, H, N, d, mode);
  if (st != SATTN_OK) return st;
  if (!aligned16(out)) return SATTN_ERR_INVALID_ARG;
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return SATTN_ERR_WORKSPACE;
  const sattn_ws_layout_t L = make_layout(B, H, N, d, mode);
  if (ws_bytes < L.total) return SATTN_ERR_WORKSPACE;
  const uint8_t *ws = static_cast<const uint8_t *>(workspace);
  if (static_cast<const uint8_t *>(out) < ws + L.total &&
      ws < static_cast<const uint8_t *>(out) + static_cast<size_t>(B) * H * N * d * 2)
    return SATTN_ERR_INVALID_ARG;
  if (!(sm_scale > 0.f) || !std::isfinite(sm_scale)) sm_scale = 1.0f / std::sqrt(static_cast<float>(d));
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  const int BH = B * H;
  const bool fp16 = (mode & SATTN_FP16_IO) != 0;
  if (d == 128)
    return fp16 ? dispatch_attn<128, __half>(ws, L, out, BH, N, causal, sm_scale, mode, mask, cs)
                : dispatch_attn<128, __nv_bfloat16>(ws, L, out, BH, N, causal, sm_scale, mode, mask, cs);
  return fp16 ? dispatch_attn<64, __half>(ws, L, out, BH, N, causal, sm_scale, mode, mask, cs)
              : dispatch_attn<64, __nv_bfloat16>(ws, L, out, BH, N, causal, sm_scale, mode, mask, cs);
}

// Library-owned workspace of sattn_fwd, one per device.
struct OwnedWorkspace {
  void *ptr = nullptr;
  size_t bytes = 0;
  CUcontext ctx = nullptr;   // context the pointer belongs to
};
std::mutex g_ws_mutex;
OwnedWorkspace g_ws[kMaxDevices];

}  // namespace
}  // namespace sattn

using namespace sattn;

extern "C" {

size_t sattn_workspace_bytes(int B, int H, int N, int d, int mode) {
  if (check_shape(B, H, N, d, mode) != SATTN_OK) return 0;
  return make_layout(B, H, N, d, mode).total;
}

int sattn_workspace_layout(int B, int H, int N, int d, int mode, sattn_ws_layout_t *out) {
  if (out == nullptr) return SATTN_ERR_INVALID_ARG;
  const int st = check_shape(B, H, N, d, mode);
  if (st != SATTN_OK) return st;
  *out = make_layout(B, H, N, d, mode);
  return SATTN_OK;
}

int sattn_quantize(const void *q, const void *k, const void *v, int B, int H, int N, int d, int mode,
                   void *workspace, size_t ws_bytes, sattn_stream_t stream) {
  const int st = check_shape(B, H, N, d, mode);
  if (st != SATTN_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return SATTN_ERR_INVALID_ARG;
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return SATTN_ERR_WORKSPACE;
  const sattn_ws_layout_t L = make_layout(B, H, N, d, mode);
  if (ws_bytes < L.total) return SATTN_ERR_WORKSPACE;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  const int BH = B * H;
  const bool fp16 = (mode & SATTN_FP16_IO) != 0;
  if (is_mxfp4(mode)) {
    if (d == 128)
      return fp16 ? launch_quant<__half, 128, kSchemeMxfp4>(q, k, v, BH, N, ws, L, cs)
                  : launch_quant<__nv_bfloat16, 128, kSchemeMxfp4>(q, k, v, BH, N, ws, L, cs);
    return fp16 ? launch_quant<__half, 64, kSchemeMxfp4>(q, k, v, BH, N, ws, L, cs)
                : launch_quant<__nv_bfloat16, 64, kSchemeMxfp4>(q, k, v, BH, N, ws, L, cs);
  }
  if (is_nvfp4(mode)) {
    if (d == 128)
      return fp16 ? launch_quant<__half, 128, kSchemeNvfp4>(q, k, v, BH, N, ws, L, cs)
                  : launch_quant<__nv_bfloat16, 128, kSchemeNvfp4>(q, k, v, BH, N, ws, L, cs);
    return fp16 ? launch_quant<__half, 64, kSchemeNvfp4>(q, k, v, BH, N, ws, L, cs)
                : launch_quant<__nv_bfloat16, 64, kSchemeNvfp4>(q, k, v, BH, N, ws, L, cs);
  }
  if (q_per_token(mode)) {
    if (d == 128)
      return fp16 ? launch_quant<__half, 128, kSchemeI8Token>(q, k, v, BH, N, ws, L, cs)
                  : launch_quant<__nv_bfloat16, 128, kSchemeI8Token>(q, k, v, BH, N, ws, L, cs);
    return fp16 ? launch_quant<__half, 64, kSchemeI8Token>(q, k, v, BH, N, ws, L, cs)
                : launch_quant<__nv_bfloat16, 64, kSchemeI8Token>(q, k, v, BH, N, ws, L, cs);
  }
  if (d == 128)
    return fp16 ? launch_quant<__half, 128, kSchemeI8Block>(q, k, v, BH, N, ws, L, cs)
                : launch_quant<__nv_bfloat16, 128, kSchemeI8Block>(q, k, v, BH, N, ws, L, cs);
  return fp16 ? launch_quant<__half, 64, kSchemeI8Block>(q, k, v, BH, N, ws, L, cs)
              : launch_quant<__nv_bfloat16, 64, kSchemeI8Block>(q, k, v, BH, N, ws, L, cs);
}

int sattn_fwd_quantized(const void *workspace, size_t ws_bytes, void *out, int B, int H, int N, int d, int causal,
                        float sm_scale, int mode, sattn_stream_t stream) {
  return fwd_quantized_impl(workspace, ws_bytes, out, B, H, N, d, causal, sm_scale, mode, nullptr, stream);
}

int sattn_fwd_quantized_sparse(const void *workspace, size_t ws_bytes, void *out, int B, int H, int N, int d,
                               int causal, float sm_scale, int mode, const uint8_t *block_mask,
                               sattn_stream_t stream) {
  const int st = check_shape(B, H, N, d, mode);
  if (st != SATTN_OK) return st;
  const int sm = check_block_mask(N, block_mask);
  if (sm != SATTN_OK) return sm;
  return fwd_quantized_impl(workspace, ws_bytes, out, B, H, N, d, causal, sm_scale, mode, block_mask, stream);
}

static int fwd_impl(const void *q, const void *k, const void *v, void *out, int B, int H, int N, int d, int causal,
                    float sm_scale, int mode, const uint8_t *mask, sattn_stream_t stream) {
  const int st = check_shape(B, H, N, d, mode);
  if (st != SATTN_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return SATTN_ERR_INVALID_ARG;
  const size_t io_bytes = static_cast<size_t>(B) * H * N * d * 2;
  const uint8_t *o = static_cast<const uint8_t *>(out);
  for (const void *in : {q, k, v}) {
    const uint8_t *p = static_cast<const uint8_t *>(in);
    if (o < p + io_bytes && p < o + io_bytes) return SATTN_ERR_INVALID_ARG;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SATTN_ERR_CUDA;
  const size_t need = make_layout(B, H, N, d, mode).total;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  void *ws = nullptr;
  size_t ws_bytes = 0;
  {
    std::lock_guard<std::mutex> lock(g_ws_mutex);
    OwnedWorkspace &w = g_ws[dev];
    const CUcontext ctx = current_context();
    if (w.ctx != ctx) w = OwnedWorkspace{nullptr, 0, ctx};   // a reset or another context: start afresh
    if (w.bytes < need) {
      if (w.ptr != nullptr && cudaFreeAsync(w.ptr, cs) != cudaSuccess) return SATTN_ERR_CUDA;
      w.ptr = nullptr;
      w.bytes = 0;
      if (cudaMallocAsync(&w.ptr, need, cs) != cudaSuccess) return SATTN_ERR_CUDA;
      w.bytes = need;
    }
    ws = w.ptr;
    ws_bytes = w.bytes;
  }
  const int s1 = sattn_quantize(q, k, v, B, H, N, d, mode, ws, ws_bytes, stream);
  if (s1 != SATTN_OK) return s1;
  return fwd_quantized_impl(ws, ws_bytes, out, B, H, N, d, causal, sm_scale, mode, mask, stream);
}

int sattn_fwd(const void *q, const void *k, const void *v, void *out, int B, int H, int N, int d, int causal,
              float sm_scale, int mode, sattn_stream_t stream) {
  return fwd_impl(q, k, v, out, B, H, N, d, causal, sm_scale, mode, nullptr, stream);
}

int sattn_fwd_sparse(const void *q, const void *k, const void *v, void *out, int B, int H, int N, int d, int causal,
                     float sm_scale, int mode, const uint8_t *block_mask, sattn_stream_t stream) {
  const int st = check_shape(B, H, N, d, mode);
  if (st != SATTN_OK) return st;
  const int sm = check_block_mask(N, block_mask);
  if (sm != SATTN_OK) return sm;
  return fwd_impl(q, k, v, out, B, H, N, d, causal, sm_scale, mode, block_mask, stream);
}

// Pipelined forward over host buffers: chunks of heads are copied in on one
// stream, quantized and attended on two compute streams in turn, and copied
// out on a fourth, so that the PCIe transfers of one chunk overlap the
// compute of its neighbours.  Heads are independent, so every chunk runs the
// same kernels as sattn_fwd on a B = 1, H = heads-in-chunk problem and the
// result is bit-identical to sattn_fwd.
namespace {
struct HostPipe {
  bool ready = false;
  CUcontext ctx = nullptr;   // context the streams, events and buffers belong to
  cudaStream_t s_in = nullptr, s_out = nullptr, s_comp[2] = {nullptr, nullptr};
  cudaEvent_t ev_start = nullptr, ev_in[2] = {nullptr, nullptr}, ev_comp[2] = {nullptr, nullptr},
              ev_out[2] = {nullptr, nullptr};
  uint8_t *slot[2] = {nullptr, nullptr};   // device q, k, v, out of one chunk
  size_t slot_bytes = 0;
  uint8_t *ws[2] = {nullptr, nullptr};     // workspace of one chunk
  size_t ws_bytes = 0;
};
std::mutex g_host_mutex;
HostPipe g_host[kMaxDevices];

// Chunks per call: enough that the first copy in and the last copy out (the
// pipeline's fill and drain) are short; a chunk smaller than the GPU is fine,
// since the two compute streams let neighbouring chunks share the SMs.
constexpr int kHostChunks = 12;
constexpr size_t kHostSlotCap = size_t(1) << 30;   // device bytes of one slot at most

bool host_pipe_init(HostPipe &p) {
  if (p.ready) return true;
  cudaStream_t *ss[4] = {&p.s_in, &p.s_out, &p.s_comp[0], &p.s_comp[1]};
  for (cudaStream_t *s : ss)
    if (cudaStreamCreateWithFlags(s, cudaStreamNonBlocking) != cudaSuccess) return false;
  cudaEvent_t *es[7] = {&p.ev_start, &p.ev_in[0], &p.ev_in[1], &p.ev_comp[0], &p.ev_comp[1], &p.ev_out[0], &p.ev_out[1]};
  for (cudaEvent_t *e : es)
    if (cudaEventCreateWithFlags(e, cudaEventDisableTiming) != cudaSuccess) return false;
  p.ready = true;
  return true;
}

// Grows the slot and workspace buffers; waits for the pipe's streams first,
// since the old buffers may still be in use by the previous call.
bool host_pipe_reserve(HostPipe &p, size_t slot_bytes, size_t ws_bytes) {
  if (p.slot_bytes >= slot_bytes && p.ws_bytes >= ws_bytes) return true;
  for (cudaStream_t s : {p.s_in, p.s_out, p.s_comp[0], p.s_comp[1]})
    if (cudaStreamSynchronize(s) != cudaSuccess) return false;
  if (p.slot_bytes < slot_bytes) {
    for (uint8_t *&b : p.slot) {
      if (b != nullptr && cudaFree(b) != cudaSuccess) return false;
      b = nullptr;
    }
    p.slot_bytes = 0;
    for (uint8_t *&b : p.slot)
      if (cudaMalloc(reinterpret_cast<void **>(&b), slot_bytes) != cudaSuccess) return false;
    p.slot_bytes = slot_bytes;
  }
  if (p.ws_bytes < ws_bytes) {
    for (uint8_t *&b : p.ws) {
      if (b != nullptr && cudaFree(b) != cudaSuccess) return false;
      b = nullptr;
    }
    p.ws_bytes = 0;
    for (uint8_t *&b : p.ws)
      if (cudaMalloc(reinterpret_cast<void **>(&b), ws_bytes) != cudaSuccess) return false;
    p.ws_bytes = ws_bytes;
  }
  return true;
}
}  // namespace

int sattn_fwd_host(const void *q, const void *k, const void *v, void *out, int B, int H, int N, int d, int causal,
                   float sm_scale, int mode, sattn_stream_t stream) {
  const int st = check_shape(B, H, N, d, mode);
  if (st != SATTN_OK) return st;
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr) return SATTN_ERR_INVALID_ARG;
  const int BH = B * H;
  const size_t head_bytes = static_cast<size_t>(N) * d * 2;
  const size_t io_bytes = head_bytes * BH;
  const uint8_t *o = static_cast<const uint8_t *>(out);
  for (const void *in : {q, k, v}) {
    const uint8_t *pi = static_cast<const uint8_t *>(in);
    if (o < pi + io_bytes && pi < o + io_bytes) return SATTN_ERR_INVALID_ARG;
  }
  int hc = (BH + kHostChunks - 1) / kHostChunks;                       // heads per chunk
  const int hc_cap = static_cast<int>(std::max<size_t>(1, kHostSlotCap / (4 * head_bytes)));
  hc = std::max(1, std::min(hc, hc_cap));
  const int nchunks = (BH + hc - 1) / hc;
  const size_t part = align_up(head_bytes * hc, kSectionAlign);       // one of q, k, v, out in a slot
  const size_t ws_need = make_layout(1, hc, N, d, mode).total;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SATTN_ERR_CUDA;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lock(g_host_mutex);
  HostPipe &p = g_host[dev];
  const CUcontext ctx = current_context();
  if (p.ctx != ctx) {                     // a reset or another context: the old handles are gone
    p = HostPipe{};
    p.ctx = ctx;
  }
  if (!host_pipe_init(p) || !host_pipe_reserve(p, 4 * part, ws_need)) return SATTN_ERR_CUDA;
  // everything this call does follows the caller's earlier work on its stream
  if (cudaEventRecord(p.ev_start, cs) != cudaSuccess) return SATTN_ERR_CUDA;
  for (cudaStream_t s : {p.s_in, p.s_out, p.s_comp[0], p.s_comp[1]})
    if (cudaStreamWaitEvent(s, p.ev_start, 0) != cudaSuccess) return SATTN_ERR_CUDA;
  const uint8_t *hq = static_cast<const uint8_t *>(q), *hk = static_cast<const uint8_t *>(k),
                *hv = static_cast<const uint8_t *>(v);
  uint8_t *hout = static_cast<uint8_t *>(out);
  int last = 0;
  for (int c = 0; c < nchunks; ++c) {
    const int sl = c & 1;
    const int h0 = c * hc, hn = std::min(hc, BH - h0);
    const size_t off = head_bytes * h0, len = head_bytes * hn;
    uint8_t *dq = p.slot[sl], *dk = dq + part, *dv = dk + part, *dout = dv + part;
    // copy in, once compute of the chunk that last used this slot is done
    if (cudaStreamWaitEvent(p.s_in, p.ev_comp[sl], 0) != cudaSuccess ||
        cudaMemcpyAsync(dq, hq + off, len, cudaMemcpyHostToDevice, p.s_in) != cudaSuccess ||
        cudaMemcpyAsync(dk, hk + off, len, cudaMemcpyHostToDevice, p.s_in) != cudaSuccess ||
        cudaMemcpyAsync(dv, hv + off, len, cudaMemcpyHostToDevice, p.s_in) != cudaSuccess ||
        cudaEventRecord(p.ev_in[sl], p.s_in) != cudaSuccess)
      return SATTN_ERR_CUDA;
    // compute, once the inputs are in and the slot's last output has been copied out
    cudaStream_t sc = p.s_comp[sl];
    if (cudaStreamWaitEvent(sc, p.ev_in[sl], 0) != cudaSuccess || cudaStreamWaitEvent(sc, p.ev_out[sl], 0) != cudaSuccess)
      return SATTN_ERR_CUDA;
    const sattn_stream_t ss = reinterpret_cast<sattn_stream_t>(sc);
    int r = sattn_quantize(dq, dk, dv, 1, hn, N, d, mode, p.ws[sl], p.ws_bytes, ss);
    if (r != SATTN_OK) return r;
    r = sattn_fwd_quantized(p.ws[sl], p.ws_bytes, dout, 1, hn, N, d, causal, sm_scale, mode, ss);
    if (r != SATTN_OK) return r;
    // copy out
    if (cudaEventRecord(p.ev_comp[sl], sc) != cudaSuccess || cudaStreamWaitEvent(p.s_out, p.ev_comp[sl], 0) != cudaSuccess ||
        cudaMemcpyAsync(hout + off, dout, len, cudaMemcpyDeviceToHost, p.s_out) != cudaSuccess ||
        cudaEventRecord(p.ev_out[sl], p.s_out) != cudaSuccess)
      return SATTN_ERR_CUDA;
    last = sl;
  }
  // the copies out run in order on one stream: the last one ends the call
  return cudaStreamWaitEvent(cs, p.ev_out[last], 0) == cudaSuccess ? SATTN_OK : SATTN_ERR_CUDA;
}

const char *sattn_status_string(int status) {
  switch (status) {
    case SATTN_OK: return "SATTN_OK";
    case SATTN_ERR_INVALID_ARG: return "SATTN_ERR_INVALID_ARG: invalid argument";
    case SATTN_ERR_UNSUPPORTED: return "SATTN_ERR_UNSUPPORTED: unsupported shape or mode";
    case SATTN_ERR_WORKSPACE: return "SATTN_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case SATTN_ERR_CUDA: return "SATTN_ERR_CUDA: CUDA runtime error";
    default: return "unknown sattn status";
  }
}

int sattn_debug_set_wait_limit(long long cycles, int withhold_k_tile) {
  const long long limit = cycles <= 0 ? kWaitLimitCycles : std::max<long long>(cycles, 1000);
  if (withhold_k_tile < -1) return SATTN_ERR_INVALID_ARG;
  if (cudaMemcpyToSymbol(g_wait_limit, &limit, sizeof(limit)) != cudaSuccess ||
      cudaMemcpyToSymbol(g_withhold_k_tile, &withhold_k_tile, sizeof(withhold_k_tile)) != cudaSuccess)
    return SATTN_ERR_CUDA;
  return SATTN_OK;
}

int sattn_debug_scores(const void *workspace, size_t ws_bytes, int B, int H, int N, int d, int mode, void *out,
                       sattn_stream_t stream) {
  const int st = check_shape(B, H, N, d, mode);
  if (st != SATTN_OK) return st;
  if (out == nullptr || (reinterpret_cast<uintptr_t>(out) & 15u)) return SATTN_ERR_INVALID_ARG;
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return SATTN_ERR_WORKSPACE;
  const sattn_ws_layout_t L = make_layout(B, H, N, d, mode);
  if (ws_bytes < L.total) return SATTN_ERR_WORKSPACE;
  const uint8_t *ws = static_cast<const uint8_t *>(workspace);
  const int BH = B * H;
  const int np = L.nblk * kTile;
  const dim3 grid(L.nblk, L.nblk, BH);
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (is_nvfp4(mode)) {                           // NVFP4 and MXFP4: float32 products of the dequantised codes
    CUtensorMap tq, tk;
    const CUtensorMapSwizzle swqk = d == 128 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
    const uint64_t rowb = d / 2;
    if (!make_map_u8(&tq, ws + L.q8, rowb, N, BH, rowb, static_cast<uint64_t>(N) * rowb, rowb, kTile, swqk) ||
        !make_map_u8(&tk, ws + L.k8, rowb, N, BH, rowb, static_cast<uint64_t>(N) * rowb, rowb, kTile, swqk))
      return SATTN_ERR_CUDA;
    float *o = static_cast<float *>(out);
    const uint8_t *sfq = ws + L.sq, *sfk = ws + L.sk;
    const bool mx = is_mxfp4(mode);
    if (d == 128) {
      if (mx)
        debug_scores_fp4_kernel<128, true><<<grid, kDebugThreads, DebugScoresF4Smem<128>::kAlloc, cs>>>(
            tq, tk, sfq, sfk, L.nblk, o, np);
      else
        debug_scores_fp4_kernel<128, false><<<grid, kDebugThreads, DebugScoresF4Smem<128>::kAlloc, cs>>>(
            tq, tk, sfq, sfk, L.nblk, o, np);
    } else {
      if (mx)
        debug_scores_fp4_kernel<64, true><<<grid, kDebugThreads, DebugScoresF4Smem<64>::kAlloc, cs>>>(
            tq, tk, sfq, sfk, L.nblk, o, np);
      else
        debug_scores_fp4_kernel<64, false><<<grid, kDebugThreads, DebugScoresF4Smem<64>::kAlloc, cs>>>(
            tq, tk, sfq, sfk, L.nblk, o, np);
    }
    g_launches += 1;
    return cudaGetLastError() == cudaSuccess ? SATTN_OK : SATTN_ERR_CUDA;
  }
  CUtensorMap tq, tk;
  const CUtensorMapSwizzle sw = d == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  if (!make_map_u8(&tq, ws + L.q8, d, N, BH, d, static_cast<uint64_t>(N) * d, d, kTile, sw) ||
      !make_map_u8(&tk, ws + L.k8, d, N, BH, d, static_cast<uint64_t>(N) * d, d, kTile, sw))
    return SATTN_ERR_CUDA;
  int32_t *o = static_cast<int32_t *>(out);
  if (d == 128)
    debug_scores_kernel<128><<<grid, kDebugThreads, DebugScoresSmem<128>::kAlloc, cs>>>(tq, tk, o, np);
  else
    debug_scores_kernel<64><<<grid, kDebugThreads, DebugScoresSmem<64>::kAlloc, cs>>>(tq, tk, o, np);
  g_launches += 1;
  return cudaGetLastError() == cudaSuccess ? SATTN_OK : SATTN_ERR_CUDA;
}

int sattn_debug_withhold_statistics(int on) {
  const int v = on ? 1 : 0;
  return cudaMemcpyToSymbol(g_withhold_statistics, &v, sizeof(v)) == cudaSuccess ? SATTN_OK : SATTN_ERR_CUDA;
}

unsigned long long sattn_kernel_launches(int reset) {
  return reset ? g_launches.exchange(0) : g_launches.load();
}

int sattn_device_error(int clear) {
  unsigned int word = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return -1;
  if (cudaMemcpyFromSymbol(&word, g_error_word, sizeof(word)) != cudaSuccess) return -1;
  if (clear) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero)) != cudaSuccess) return -1;
  }
  return static_cast<int>(word);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// sattn_fwd_noalloc: sattn_fwd for callers that cannot allocate device memory.
//
// Its workspace is a fixed static device array of SATTN_NOALLOC_MAX_BYTES
// (declared below), which every GPU that loads this library holds until the
// process exits.  Host code cannot pass the array's name to a kernel (on the
// host it names a stand-in object, not device memory), so the first call on a
// device, with that device current, looks the array's device address up with
// cudaGetSymbolAddress and caches it; make that first call before any stream
// capture.  No call allocates or frees memory.  All calls on a device share
// the array and it keeps the last call's contents: the quantisation step
// clears the two reduction buffers it accumulates into on every call, and
// calls that overlap on the GPU (other streams, other host threads) race.
namespace sattn {

__device__ __align__(256) uint8_t g_noalloc_workspace[SATTN_NOALLOC_MAX_BYTES];

namespace {
std::mutex g_noalloc_mutex;
void *g_noalloc_addr[kMaxDevices];   // device address of the array per device, once looked up
CUcontext g_noalloc_ctx[kMaxDevices];  // context it was looked up in
}  // namespace
}  // namespace sattn

extern "C" int sattn_fwd_noalloc(const void *q, const void *k, const void *v, void *out, int B, int H, int N,
                                 int d, int causal, float sm_scale, int mode, sattn_stream_t stream) {
  const int st = check_shape(B, H, N, d, mode);
  if (st != SATTN_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return SATTN_ERR_INVALID_ARG;
  const size_t io_bytes = static_cast<size_t>(B) * H * N * d * 2;
  const uint8_t *o = static_cast<const uint8_t *>(out);
  for (const void *in : {q, k, v}) {
    const uint8_t *p = static_cast<const uint8_t *>(in);
    if (o < p + io_bytes && p < o + io_bytes) return SATTN_ERR_INVALID_ARG;
  }
  const size_t need = make_layout(B, H, N, d, mode).total;
  if (need > SATTN_NOALLOC_MAX_BYTES) return SATTN_ERR_WORKSPACE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SATTN_ERR_CUDA;
  void *ws = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    const CUcontext ctx = current_context();
    if (g_noalloc_addr[dev] == nullptr || g_noalloc_ctx[dev] != ctx) {
      void *addr = nullptr;
      if (cudaGetSymbolAddress(&addr, g_noalloc_workspace) != cudaSuccess || addr == nullptr)
        return SATTN_ERR_CUDA;
      g_noalloc_addr[dev] = addr;
      g_noalloc_ctx[dev] = ctx;
    }
    ws = g_noalloc_addr[dev];
  }
  const int s1 = sattn_quantize(q, k, v, B, H, N, d, mode, ws, SATTN_NOALLOC_MAX_BYTES, stream);
  if (s1 != SATTN_OK) return s1;
  return sattn_fwd_quantized(ws, SATTN_NOALLOC_MAX_BYTES, out, B, H, N, d, causal, sm_scale, mode, stream);
}
