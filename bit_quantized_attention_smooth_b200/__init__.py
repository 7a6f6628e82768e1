"""sattn: SageAttention-style quantized attention forward for B200 (sm_100a).

Python binding of the C ABI in ``include/sattn.h`` (``libsattn.so``, built
in-tree by ``build.py``).  This module only marshals arguments: every step of
the computation runs in the library's CUDA kernels.  It raises when the
library is missing or a tensor is not on a CUDA device; there is no fallback.

    import bit_quantized_attention_smooth_b200 as sattn
    out = sattn.fwd(q, k, v, causal=False, mode="i8f8")     # q, k, v [B, H, N, d]
"""

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsattn.so")

MODES = {"i8f8": 0, "nvfp4": 1, "mxfp4": 2}
FP16_IO = 0x100
Q_PER_TOKEN = 0x200
P_PER_TOKEN = 0x400
# Lazy reference-max threshold of the I8QK_F8PV kernel (SATTN_I8F8_LAZY_TAU in
# include/sattn.h): the row max moves only when a key tile exceeds it by more
# than this many powers of two, and P's static FP8 scale is 448 * 2^-tau.
I8F8_LAZY_TAU = 4.0
STATUS = {0: "SATTN_OK", 1: "SATTN_ERR_INVALID_ARG", 2: "SATTN_ERR_UNSUPPORTED",
          3: "SATTN_ERR_WORKSPACE", 4: "SATTN_ERR_CUDA"}

# Every entry point declared in include/sattn.h.
EXPORTS = ("sattn_workspace_bytes", "sattn_quantize", "sattn_fwd_quantized", "sattn_fwd",
           "sattn_status_string", "sattn_device_error", "sattn_workspace_layout", "sattn_fwd_noalloc",
           "sattn_fwd_host", "sattn_kernel_launches", "sattn_debug_set_wait_limit", "sattn_debug_withhold_statistics",
           "sattn_fwd_quantized_sparse", "sattn_fwd_sparse", "sattn_debug_scores")


class SattnError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)}")


class WsLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in
                ("q8", "k8", "vt8", "sq", "sk", "sv", "mu", "ksum", "vmax", "total")] + \
               [("nv", ctypes.c_int), ("nblk", ctypes.c_int)]


_lib = None


def lib():
    """The loaded libsattn.so (raises OSError when it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise OSError(f"libsattn.so not built at {LIB_PATH}; run bit_quantized_attention_smooth_b200/build.py")
        L = ctypes.CDLL(LIB_PATH)
        i, sz, vp, f = ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_float
        L.sattn_workspace_bytes.restype = sz
        L.sattn_workspace_bytes.argtypes = [i, i, i, i, i]
        L.sattn_quantize.restype = i
        L.sattn_quantize.argtypes = [vp, vp, vp, i, i, i, i, i, vp, sz, vp]
        L.sattn_fwd_quantized.restype = i
        L.sattn_fwd_quantized.argtypes = [vp, sz, vp, i, i, i, i, i, f, i, vp]
        L.sattn_fwd.restype = i
        L.sattn_fwd.argtypes = [vp, vp, vp, vp, i, i, i, i, i, f, i, vp]
        L.sattn_status_string.restype = ctypes.c_char_p
        L.sattn_status_string.argtypes = [i]
        L.sattn_device_error.restype = i
        L.sattn_device_error.argtypes = [i]
        L.sattn_workspace_layout.restype = i
        L.sattn_workspace_layout.argtypes = [i, i, i, i, i, ctypes.POINTER(WsLayout)]
        L.sattn_fwd_noalloc.restype = i
        L.sattn_fwd_noalloc.argtypes = [vp, vp, vp, vp, i, i, i, i, i, f, i, vp]
        L.sattn_fwd_host.restype = i
        L.sattn_fwd_host.argtypes = [vp, vp, vp, vp, i, i, i, i, i, f, i, vp]
        L.sattn_kernel_launches.restype = ctypes.c_ulonglong
        L.sattn_kernel_launches.argtypes = [i]
        L.sattn_debug_set_wait_limit.restype = i
        L.sattn_debug_set_wait_limit.argtypes = [ctypes.c_longlong, i]
        L.sattn_debug_withhold_statistics.restype = i
        L.sattn_debug_withhold_statistics.argtypes = [i]
        L.sattn_fwd_quantized_sparse.restype = i
        L.sattn_fwd_quantized_sparse.argtypes = [vp, sz, vp, i, i, i, i, i, f, i, vp, vp]
        L.sattn_fwd_sparse.restype = i
        L.sattn_fwd_sparse.argtypes = [vp, vp, vp, vp, i, i, i, i, i, f, i, vp, vp]
        L.sattn_debug_scores.restype = i
        L.sattn_debug_scores.argtypes = [vp, sz, i, i, i, i, i, vp, vp]
        _lib = L
    return _lib


def mode_code(mode, dtype, q_per_token=False, p_per_token=False):
    if mode not in MODES:
        raise ValueError(f"mode must be one of {list(MODES)}")
    if dtype not in (torch.bfloat16, torch.float16):
        raise TypeError("q, k, v must be bfloat16 or float16")
    return (MODES[mode] | (FP16_IO if dtype == torch.float16 else 0) | (Q_PER_TOKEN if q_per_token else 0) |
            (P_PER_TOKEN if p_per_token else 0))


def _check(status, what):
    if status != 0:
        raise SattnError(status, what)


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check_qkv(q, k, v):
    for t in (q, k, v):
        if not t.is_cuda:
            raise ValueError("q, k, v must be CUDA tensors")
        if not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous [B, H, N, d]")
    if q.dim() != 4 or q.shape != k.shape or q.shape != v.shape:
        raise ValueError("q, k, v must share the shape [B, H, N, d]")
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("q, k, v must share one dtype")
    return tuple(q.shape)


def workspace_bytes(B, H, N, d, mode="i8f8", dtype=torch.bfloat16, q_per_token=False):
    return int(lib().sattn_workspace_bytes(B, H, N, d, mode_code(mode, dtype, q_per_token)))


def workspace_layout(B, H, N, d, mode="i8f8", dtype=torch.bfloat16, q_per_token=False):
    out = WsLayout()
    _check(lib().sattn_workspace_layout(B, H, N, d, mode_code(mode, dtype, q_per_token), ctypes.byref(out)),
           "sattn_workspace_layout")
    return {n: getattr(out, n) for n, _ in WsLayout._fields_}


def quantize(q, k, v, mode="i8f8", workspace=None, stream=None, q_per_token=False):
    """Quantise q, k, v into a uint8 workspace tensor (allocated when not given).
    ``q_per_token``: one INT8 scale per query token (I8QK_F8PV only)."""
    B, H, N, d = _check_qkv(q, k, v)
    m = mode_code(mode, q.dtype, q_per_token)
    nbytes = int(lib().sattn_workspace_bytes(B, H, N, d, m))
    if nbytes == 0:
        raise SattnError(2, "sattn_workspace_bytes")
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    _check(lib().sattn_quantize(q.data_ptr(), k.data_ptr(), v.data_ptr(), B, H, N, d, m,
                                workspace.data_ptr(), workspace.numel(), _stream(stream)),
           "sattn_quantize")
    return workspace


def fwd_quantized(workspace, shape, causal=False, sm_scale=None, mode="i8f8", dtype=torch.bfloat16,
                  out=None, stream=None, q_per_token=False, p_per_token=False):
    """Attention over a workspace filled by ``quantize``; returns out [B, H, N, d].
    ``p_per_token``: P quantised per query row and key block (I8QK_F8PV only)."""
    B, H, N, d = shape
    if out is None:
        out = torch.empty((B, H, N, d), dtype=dtype, device=workspace.device)
    _check(lib().sattn_fwd_quantized(workspace.data_ptr(), workspace.numel(), out.data_ptr(),
                                     B, H, N, d, int(bool(causal)), float(sm_scale or 0.0),
                                     mode_code(mode, dtype, q_per_token, p_per_token), _stream(stream)),
           "sattn_fwd_quantized")
    return out


def fwd(q, k, v, causal=False, sm_scale=None, mode="i8f8", out=None, stream=None, q_per_token=False,
        p_per_token=False):
    """O = softmax(Q K^T * sm_scale) V with quantised operands (library-owned workspace)."""
    B, H, N, d = _check_qkv(q, k, v)
    if out is None:
        out = torch.empty_like(q)
    _check(lib().sattn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, H, N, d,
                           int(bool(causal)), float(sm_scale or 0.0),
                           mode_code(mode, q.dtype, q_per_token, p_per_token), _stream(stream)),
           "sattn_fwd")
    return out


def _check_block_mask(block_mask, q):
    B, H, N, _ = q.shape
    nb = (N + 127) // 128
    if not block_mask.is_cuda or block_mask.dtype not in (torch.uint8, torch.bool):
        raise ValueError("block_mask must be a CUDA uint8/bool tensor")
    if tuple(block_mask.shape) != (B, H, nb, nb) or not block_mask.is_contiguous():
        raise ValueError(f"block_mask must be contiguous [B, H, {nb}, {nb}]")


def fwd_sparse(q, k, v, block_mask, causal=False, sm_scale=None, mode="i8f8", out=None, stream=None,
               q_per_token=False):
    """``fwd`` that skips the 128 x 128 (query, key) blocks where ``block_mask``
    [B, H, ceil(N/128), ceil(N/128)] (uint8 or bool, on the device) is 0."""
    B, H, N, d = _check_qkv(q, k, v)
    _check_block_mask(block_mask, q)
    if out is None:
        out = torch.empty_like(q)
    _check(lib().sattn_fwd_sparse(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, H, N, d,
                                  int(bool(causal)), float(sm_scale or 0.0), mode_code(mode, q.dtype, q_per_token),
                                  block_mask.data_ptr(), _stream(stream)),
           "sattn_fwd_sparse")
    return out


def fwd_quantized_sparse(workspace, shape, block_mask, causal=False, sm_scale=None, mode="i8f8",
                         dtype=torch.bfloat16, out=None, stream=None, q_per_token=False):
    """``fwd_quantized`` with block-sparse key skipping (see ``fwd_sparse``)."""
    B, H, N, d = shape
    if out is None:
        out = torch.empty((B, H, N, d), dtype=dtype, device=workspace.device)
    _check_block_mask(block_mask, out)
    _check(lib().sattn_fwd_quantized_sparse(workspace.data_ptr(), workspace.numel(), out.data_ptr(),
                                            B, H, N, d, int(bool(causal)), float(sm_scale or 0.0),
                                            mode_code(mode, dtype, q_per_token), block_mask.data_ptr(),
                                            _stream(stream)),
           "sattn_fwd_quantized_sparse")
    return out


def fwd_host(q, k, v, causal=False, sm_scale=None, mode="i8f8", out=None, stream=None, q_per_token=False):
    """``fwd`` on host (CPU) tensors: copies in, computes and copies out chunk by
    chunk, overlapping the transfers with the compute.  Pinned tensors
    (``tensor.pin_memory()``) let the copies run asynchronously.  The call is
    ordered on the current CUDA stream (or ``stream``); ``out`` holds the result
    once that stream has passed it, e.g. after ``torch.cuda.synchronize()``."""
    for t in (q, k, v):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous host tensors [B, H, N, d]")
    if q.dim() != 4 or q.shape != k.shape or q.shape != v.shape:
        raise ValueError("q, k, v must share the shape [B, H, N, d]")
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("q, k, v must share one dtype")
    B, H, N, d = q.shape
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    elif out.is_cuda or not out.is_contiguous() or out.shape != q.shape or out.dtype != q.dtype:
        raise ValueError("out must be a contiguous host tensor like q")
    _check(lib().sattn_fwd_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, H, N, d,
                                int(bool(causal)), float(sm_scale or 0.0), mode_code(mode, q.dtype, q_per_token),
                                _stream(stream)),
           "sattn_fwd_host")
    return out


def debug_scores(workspace, shape, mode="i8f8", dtype=torch.bfloat16, stream=None, q_per_token=False):
    """Test accessor: the scores Q K^T of a quantised workspace computed on the
    tensor cores, [B, H, Np, Np] (Np = N rounded up to 128): int32 q8 . k8^T
    (I8QK_F8PV) or float32 products of the dequantised FP4 operands."""
    B, H, N, d = shape
    np_ = (N + 127) // 128 * 128
    out = torch.empty((B, H, np_, np_), dtype=torch.int32 if mode == "i8f8" else torch.float32,
                      device=workspace.device)
    _check(lib().sattn_debug_scores(workspace.data_ptr(), workspace.numel(), B, H, N, d,
                                    mode_code(mode, dtype, q_per_token), out.data_ptr(), _stream(stream)),
           "sattn_debug_scores")
    return out


def device_error(clear=False):
    """Device-side error word (0 = no bounded wait ran out); synchronises the device."""
    return int(lib().sattn_device_error(int(bool(clear))))


def kernel_launches(reset=False):
    """CUDA kernels the library has launched since load or the last reset."""
    return int(lib().sattn_kernel_launches(int(bool(reset))))
