/*
 * sattn -- SageAttention-style quantized attention forward for NVIDIA B200 (sm_100a).
 *
 * C ABI of libsattn.so.  All entry points are plain C: device pointers (host
 * pointers for sattn_fwd_host), sizes, a CUDA stream.  No entry point throws or aborts; each returns a status code
 * (sattn_status_t) and never synchronizes the stream unless stated.
 *
 * The operation (TurboDiffusion explainer, wxsanhe.com post 64219, section 1
 * "hybrid attention": QK in INT8, PV in FP8, outlier smoothing, two-level
 * accumulation; SageAttention tag page, reportify.cn, SageAttention3 summary,
 * bullets [15][16][17]: NVFP4 microscaling, two-stage P scale, per-block INT8):
 *
 *     O = softmax(Q K^T * sm_scale [+ causal mask]) V
 *
 * computed with quantized operands:
 *   SATTN_I8QK_F8PV : K smoothed by its per-channel token mean; Q and K INT8
 *                     with one float32 scale per 128-token block (Q: or per
 *                     token, SATTN_Q_PER_TOKEN); V FP8 E4M3 with one scale per
 *                     channel; P FP8 E4M3 with the static scale 448 * 2^-tau
 *                     of a lazy reference max (SATTN_I8F8_LAZY_TAU);
 *                     P.V accumulated in an inner FP32 accumulator that is
 *                     flushed into an outer FP32 accumulator every few key
 *                     blocks (two-level accumulation).
 *   SATTN_NVFP4     : FP4 E2M1 values with one E4M3 scale per 16 values for
 *                     Q, K (along channels) and V (along tokens); P quantized
 *                     in two stages (a per-row, per-key-block float32 scale,
 *                     then NVFP4).  P.V is flushed into the outer
 *                     accumulator every key block, since the stage-1 scale
 *                     changes per block.
 *   SATTN_MXFP4     : the MXFP4 ablation of SATTN_NVFP4 (same tag page, FP4
 *                     bullet [15], which reports NVFP4 more accurate than
 *                     MXFP4): every FP4 operand (Q, K, V, and P's second
 *                     stage) in blocks of 32 values with one E8M0 scale
 *                     2^(floor(log2 max|x|) - 2) (OCP Microscaling); the
 *                     same kernels, tensor layout and workspace layout as
 *                     SATTN_NVFP4, the E8M0 scale stored for each 16-value
 *                     half of its block.
 *
 * Tensor layout (all modes): q, k, v, out are contiguous [B, H, N, d] ("BHND"),
 * element type bf16 (default) or fp16 (mode | SATTN_FP16_IO); out has the
 * input's element type.  Device pointers must be 16-byte aligned (the host
 * pointers of sattn_fwd_host may have any alignment).
 * Supported: d in {64, 128}; N >= 1; B*H >= 1; B*H*N*d < 2^31.
 * sm_scale <= 0 selects 1/sqrt(d).  causal masks key j > query i.
 *
 * Errors: invalid arguments are rejected before any launch with
 * SATTN_ERR_INVALID_ARG / SATTN_ERR_UNSUPPORTED / SATTN_ERR_WORKSPACE.  A
 * failed launch returns SATTN_ERR_CUDA.  Faults during execution surface at the
 * caller's next synchronization, as with any CUDA kernel.  Every wait inside
 * the kernels is bounded; a wait that runs out sets a device-side error word
 * (read with sattn_device_error) and the kernel returns early with partial
 * output.
 */
#ifndef SATTN_H
#define SATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; 0 is the legacy default stream. */
typedef struct CUstream_st *sattn_stream_t;

typedef enum {
  SATTN_I8QK_F8PV = 0,
  SATTN_NVFP4 = 1,
  SATTN_MXFP4 = 2,          /* the MXFP4 ablation of SATTN_NVFP4 (above) */
  SATTN_FP16_IO = 0x100,    /* flag: q, k, v, out are fp16 instead of bf16 */
  SATTN_Q_PER_TOKEN = 0x200, /* flag, I8QK_F8PV only: one INT8 scale per query
                               token instead of per 128-token block (the
                               "thread-level quantization" of the QbitAI
                               reprint, txrjy.com, SageAttention paragraph);
                               NVFP4 or MXFP4 with it is SATTN_ERR_UNSUPPORTED */
  SATTN_P_PER_TOKEN = 0x400  /* flag, I8QK_F8PV only, dense calls only: P
                               quantized per token (tag page, SageAttention3
                               summary, 8-bit bullet [17]): each query row's
                               P of a key block is stored as
                               E4M3(448 * P~ / rowmax of the block) and the
                               block's P V is scaled back by that max; the
                               inner accumulator is then flushed after every
                               key block.  The quantized operands (and the
                               workspace) are those of the mode without it.
                               With another mode, or in a block-sparse call:
                               SATTN_ERR_UNSUPPORTED */
} sattn_mode_t;

/* Lazy reference-max threshold of the I8QK_F8PV softmax (powers of two): a
 * row's reference max m moves to a key tile's row max only when that max
 * exceeds m by more than this, so P~ = 2^(S*log2e - m) <= 2^tau and P is
 * stored as E4M3(448 * 2^-tau * P~).  The pages do not say when the running
 * max of the streaming softmax moves; 0 would be the exact running max. */
#define SATTN_I8F8_LAZY_TAU 4.0f

typedef enum {
  SATTN_OK = 0,
  SATTN_ERR_INVALID_ARG = 1,
  SATTN_ERR_UNSUPPORTED = 2,
  SATTN_ERR_WORKSPACE = 3,
  SATTN_ERR_CUDA = 4
} sattn_status_t;

/* Bytes of workspace that sattn_quantize fills for this problem and mode
 * (0 for invalid arguments).  Depends only on (B, H, N, d, mode).  Bookkeeping
 * of this library; no passage of the pages defines it. */
size_t sattn_workspace_bytes(int B, int H, int N, int d, int mode);

/* Quantize q, k, v into `workspace` (device memory of at least
 * sattn_workspace_bytes(...) bytes, 256-byte aligned, owned by the caller).
 * I8QK_F8PV: per-channel K mean (float64 sum of the stored values / N, rounded
 * once to float32: the "outlier smoothing" of the TurboDiffusion explainer,
 * section 1), INT8 codes and scales of Q (per 128-token block, or per token
 * with SATTN_Q_PER_TOKEN) and of K - mean per block (tag page, SageAttention3
 * summary, bullet [17]: per-block INT8), per-channel FP8 codes and scales of V
 * (explainer, section 1: PV in FP8; V stored transposed, tokens contiguous).
 * NVFP4: E2M1 codes with one E4M3 scale per 16 values of Q, K - mean (along
 * channels) and V (along tokens) (tag page, bullet [15]).  MXFP4: E2M1 codes
 * with one E8M0 scale per 32 values, along the same axes (the ablation of the
 * same bullet).  A NaN input makes
 * the scale it feeds NaN.  Asynchronous on `stream`: one memset of the
 * workspace's scratch section and one kernel launch, whose tiles of K and V
 * wait (bounded; on time-out the device error word records it, see
 * sattn_device_error) for their head's statistics.  The workspace stays
 * valid for any number of sattn_fwd_quantized calls with the same
 * (B, H, N, d, mode).  Errors: see the header overview; nothing is written
 * when an argument is rejected. */
int sattn_quantize(const void *q, const void *k, const void *v,
                   int B, int H, int N, int d, int mode,
                   void *workspace, size_t ws_bytes, sattn_stream_t stream);

/* Fused attention over a workspace filled by sattn_quantize with the same
 * (B, H, N, d, mode).  Writes out [B, H, N, d].  I8QK_F8PV: S = Q K^T on the
 * INT8 tensor cores, online softmax in FP32, P in FP8, P V on the FP8 tensor
 * cores into an inner accumulator flushed into an outer FP32 one every few key
 * blocks (TurboDiffusion explainer, section 1: INT8 QK, FP8 PV, two-level
 * accumulation).  NVFP4: block-scaled FP4 tensor cores for both products, P
 * quantized in two stages (tag page, SageAttention3 summary, bullets
 * [15][16]); MXFP4 the same with E8M0 scales per 32 values, P's second
 * stage included.  `out` must not alias the workspace (SATTN_ERR_INVALID_ARG).
 * Asynchronous on `stream`. */
int sattn_fwd_quantized(const void *workspace, size_t ws_bytes, void *out,
                        int B, int H, int N, int d, int causal, float sm_scale,
                        int mode, sattn_stream_t stream);

/* Block-sparse sattn_fwd_quantized: the 128 x 128 blocks of (query, key)
 * that `block_mask` marks 0 are skipped -- their keys are left out of the
 * softmax of that block's queries, and their K/V tiles are neither loaded nor
 * multiplied -- on top of the causal mask (the "skip" part of Sparse-Linear
 * Attention, TurboDiffusion explainer, SLA section, with the mask given by
 * the caller).  block_mask: device memory, uint8 [B*H][nblk][nblk], nblk =
 * ceil(N / 128), entry [bh][i][j] nonzero = query block i keeps key block j.
 * A query block that keeps no key block gets zero output rows.  Every mode
 * (not with SATTN_P_PER_TOKEN: SATTN_ERR_UNSUPPORTED);
 * nblk <= 2048 (N <= 262144), else SATTN_ERR_UNSUPPORTED; block_mask == NULL
 * is SATTN_ERR_INVALID_ARG.  The
 * mask is read by the kernel, so it must stay unchanged until `stream` has
 * passed the call.  Otherwise as sattn_fwd_quantized. */
int sattn_fwd_quantized_sparse(const void *workspace, size_t ws_bytes, void *out,
                               int B, int H, int N, int d, int causal, float sm_scale,
                               int mode, const uint8_t *block_mask, sattn_stream_t stream);

/* sattn_quantize followed by sattn_fwd_quantized, with a workspace that the
 * library owns: the one-call, drop-in form of the attention (tag page,
 * SageAttention3 summary, bullet [5]: plug-and-play; explainer, section 1:
 * usable in place of FlashAttention).  One workspace per device, allocated on
 * first use with cudaMallocAsync on `stream` and grown (never shrunk) when a
 * larger problem arrives.  Calls that share a device must be ordered (same
 * stream, or synchronized), because they share this workspace, which belongs
 * to the context current at its allocation (after cudaDeviceReset, or under
 * another context, the next call allocates a new one).  `out` must
 * not alias q, k or v (SATTN_ERR_INVALID_ARG). */
int sattn_fwd(const void *q, const void *k, const void *v, void *out,
              int B, int H, int N, int d, int causal, float sm_scale, int mode,
              sattn_stream_t stream);

/* sattn_fwd with block-sparse key skipping (block_mask as in
 * sattn_fwd_quantized_sparse).  The quantization is the dense one: the K
 * mean and the V channel scales still cover every token. */
int sattn_fwd_sparse(const void *q, const void *k, const void *v, void *out,
                     int B, int H, int N, int d, int causal, float sm_scale, int mode,
                     const uint8_t *block_mask, sattn_stream_t stream);

/* sattn_fwd on HOST buffers (a deployment variant; the pages have no
 * counterpart): q, k, v and out are host pointers ([B, H, N, d],
 * same element type and layout as sattn_fwd); pinned (page-locked) memory lets
 * the copies run asynchronously, pageable memory works but serializes them.
 * The call splits the B*H heads into up to 12 chunks and pipelines them: chunk c
 * is copied to the device on one stream, quantized and attended on one of two
 * compute streams, and copied back on a fourth stream, so that the PCIe
 * transfers of one chunk overlap the compute of the others.  Attention heads
 * are independent and every quantization scale is per head, so the output is
 * bit-identical to sattn_fwd on the same inputs.  The device buffers (two
 * chunks of q, k, v, out and two workspaces) and the streams are owned by the
 * library, one set per device, created on first use with cudaMalloc and grown
 * when a larger problem arrives (growing waits for the previous call's work).
 * The call is ordered on `stream` like a kernel launch: its work starts after
 * the work already queued on `stream`, and `out` holds the result once
 * `stream` has passed the call (e.g. after cudaStreamSynchronize(stream)).
 * q, k, v must stay unchanged and out untouched until then.  Calls on one
 * device are serialized by the library.  `out` must not alias q, k or v. */
int sattn_fwd_host(const void *q, const void *k, const void *v, void *out,
                   int B, int H, int N, int d, int causal, float sm_scale, int mode,
                   sattn_stream_t stream);

/* Size of the static device workspace of sattn_fwd_noalloc: 64 MiB, enough
 * for B*H*N*d up to about 22 million elements (e.g. B=1, H=12, N=4096, d=128). */
#define SATTN_NOALLOC_MAX_BYTES (64ull << 20)

/* sattn_fwd for callers that cannot allocate device memory.  The method has
 * no counterpart on the pages; this is a deployment variant.  Some hosts own
 * every byte of device memory and do not let a library allocate on its own
 * (an inference engine that reserves its memory budget up front and loads
 * this code as a plugin, or a process whose allocator is locked after
 * start-up); for them this entry point takes its workspace from one static
 * device array of SATTN_NOALLOC_MAX_BYTES that the library defines, so it
 * never calls cudaMalloc, cudaMallocAsync, cudaFree or any allocating routine.
 * Every GPU that loads libsattn.so holds that array until the process exits.
 * Arguments, layout and semantics are those of sattn_fwd.  Returns
 * SATTN_ERR_WORKSPACE, before any launch, when the problem needs more than
 * SATTN_NOALLOC_MAX_BYTES (sattn_workspace_bytes tells).  The first call on a
 * device looks up the array's device address (cudaGetSymbolAddress) with that
 * device current, and so does the first call after the device's context
 * changed (cudaDeviceReset, or the caller's own context); make such a call
 * before any stream capture.  All calls
 * on one device share the array, which keeps the previous call's contents
 * (each call re-clears what must start at zero): calls that overlap on the GPU,
 * from other streams or host threads, race and must be ordered by the caller. */
int sattn_fwd_noalloc(const void *q, const void *k, const void *v, void *out,
                      int B, int H, int N, int d, int causal, float sm_scale, int mode,
                      sattn_stream_t stream);

/* Human-readable name of a status code (static string). */
const char *sattn_status_string(int status);

/* Failure-path test hook; not for production use.  Sets, on the current
 * device, the bound of the kernels' waits between their roles (cycles <= 0:
 * the default of about 2-4 s; otherwise at least 1000 cycles) and, when
 * withhold_k_tile >= 0, makes every attention kernel skip loading that key
 * tile, so that the waits for it run out: the kernel then sets bit 0 of the
 * device error word (sattn_device_error), lets the copies and MMAs already in
 * flight complete, releases its tensor memory and returns with partial
 * output.  Waits that only drain work in flight keep the default bound.
 * Call with (0, -1) to restore normal operation.  Synchronous (it writes two
 * device variables).  Returns SATTN_ERR_INVALID_ARG for withhold_k_tile < -1. */
int sattn_debug_set_wait_limit(long long cycles, int withhold_k_tile);

/* Failure-path test hook; not for production use.  With on != 0, the
 * quantiser (sattn_quantize and every call that quantises) never sees a
 * head's K/V statistics as complete: the waits for them run out after the
 * bound set by sattn_debug_set_wait_limit, bit 0 of the device error word is
 * set, the copies in flight complete and the kernel returns with the
 * workspace partly written.  on == 0 restores normal operation.  Synchronous
 * (it writes one device variable).  Returns SATTN_OK or SATTN_ERR_CUDA. */
int sattn_debug_withhold_statistics(int on);

/* Test accessor; not for production use.  Writes the scores S = Q K^T of
 * the quantized operands of a workspace filled by sattn_quantize with the
 * same (B, H, N, d, mode), computed on the tensor cores the way the attention
 * kernels do (their tensor maps, descriptors and MMA kinds), one 128 x 128
 * tile per CTA:
 *   I8QK_F8PV: int32 S_int[b, h, i, j] = sum_c q8[b, h, i, c] k8[b, h, j, c]
 *              (TurboDiffusion explainer, section 1: QK^T in INT8), exact;
 *   NVFP4 / MXFP4: float32 sum_c Q^[i, c] K'^[j, c] of the dequantized E2M1
 *              codes with their block scales applied by the block-scaled MMA
 *              (tag page, SageAttention3 summary, FP4 bullet [15]).
 * out: device memory [B*H, Np, Np], Np = ceil(N/128) * 128, of int32 or
 * float32 as above, 16-byte aligned, owned by the caller; rows and columns at
 * and past N hold products of zero codes (0).  Asynchronous on `stream`, one
 * launch.  Errors as sattn_fwd_quantized. */
int sattn_debug_scores(const void *workspace, size_t ws_bytes, int B, int H, int N, int d, int mode,
                       void *out, sattn_stream_t stream);

/* Number of CUDA kernels this library has launched, in this process, since it
 * was loaded or since the last call with reset != 0 (which returns the count
 * and sets it to 0).  Counts launches (of every entry point, all devices), not
 * completions; memset nodes are not counted.  Never touches the GPU. */
unsigned long long sattn_kernel_launches(int reset);

/* Device-side error word of the current device: 0 when no kernel wait has run
 * out of time since the last clear.  Synchronizes the device.  clear != 0
 * resets the word to 0 after reading. */
int sattn_device_error(int clear);

/* Byte offsets of the workspace sections, for tests and tools that read the
 * quantized operands.  Offsets not used by a mode are set to SIZE_MAX.
 *   I8QK_F8PV: q8  int8   [B*H, N, d]        k8 int8 [B*H, N, d]
 *              vt8 e4m3   [B*H, d, Nv]  (Nv = N rounded up to 16)
 *              sq float32 [B*H, ceil(N/128)], or [B*H, N] with SATTN_Q_PER_TOKEN
 *              sk float32 [B*H, ceil(N/128)]   sv, mu float32 [B*H, d]
 *              ksum float64 [B*H, d], vmax uint32 [B*H, d] followed by
 *              the quantiser's work counters uint32 [2*B*H + 1] (scratch)
 *   NVFP4 (same fields, other contents):
 *              q8, k8 E2M1 codes, two per byte (low nibble = even channel)
 *                        [B*H, N, d/2]
 *              vt8 E2M1 codes of V transposed [B*H, d, Nv/2] (Nv = N
 *                        rounded up to 32; low nibble = even token)
 *              sq, sk E4M3 block scales [B*H, ceil(N/128), d/64, 512]; row m
 *                        (token within the 128-token block) and 16-channel
 *                        block b at byte 16*(m%32) + 4*(m/32) + b
 *              sv E4M3 block scales of V [B*H, ceil(N/128), 2, 512]; same
 *                        byte order with m = channel and b = 16-token block
 *              mu float32 [B*H, d]; ksum, vmax scratch as above
 *   MXFP4: as NVFP4, with E8M0 scale codes (scale 2^(code - 127)) of blocks
 *              of 32 values, each written at both of its 16-value positions
 *              b = 2c, 2c + 1 of block c */
typedef struct {
  size_t q8, k8, vt8, sq, sk, sv, mu, ksum, vmax, total;
  int nv, nblk;
} sattn_ws_layout_t;

int sattn_workspace_layout(int B, int H, int N, int d, int mode, sattn_ws_layout_t *out);

#ifdef __cplusplus
}
#endif

#endif /* SATTN_H */
