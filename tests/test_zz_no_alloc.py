"""sattn_fwd_noalloc: the entry point for callers that cannot allocate device memory.

Some callers own every byte of device memory (an inference engine that
reserves its budget up front and loads this library as a plugin, a process
whose allocator is locked after start-up) and cannot let the library call
cudaMalloc.  sattn_fwd_noalloc takes its workspace from a static device array
instead.  The GPU test calls it through the C ABI and compares it with
sattn_fwd, the entry point that allocates its own workspace.  Both run the same
kernels on the same inputs, so the outputs must be equal bit for bit.  The
calls come in pairs of the same shape with new inputs: the array keeps the
previous call's contents, and a second call of the same shape lays its
reduction buffers (K channel sums, V channel maxima) exactly over the first
call's, so anything stale that leaked through would change the second output.
The file is collected last on purpose: a failure here comes after every other
test has run.
"""

import ctypes

import pytest
import torch

import bit_quantized_attention_smooth_b200 as sattn
from bit_quantized_attention_smooth_b200 import build as sattn_build
import workloads as W

NOALLOC_MAX = 64 << 20
WORKSPACE_ERR = 3


def _lib():
    sattn_build.build()
    return sattn.lib()


def test_noalloc_rejects_problems_beyond_its_array():
    L = _lib()
    p = ctypes.c_void_p(1 << 20)
    o = ctypes.c_void_p(1 << 40)
    big = (1, 12, 32760, 128)                 # needs ~151 MB > 64 MiB
    assert L.sattn_workspace_bytes(*big, 0) > NOALLOC_MAX
    assert L.sattn_fwd_noalloc(p, p, p, o, *big, 0, 0.0, 0, None) == WORKSPACE_ERR


def _noalloc(L, q, k, v, causal, mode):
    B, H, N, d = q.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    out = torch.full_like(q, float("nan"))
    st = L.sattn_fwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                             B, H, N, d, int(causal), 0.0, sattn.mode_code(mode, q.dtype), stream)
    assert st == 0, sattn.STATUS.get(st, st)
    return out


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,N,d,dtype,causal,mode", [
    (1, 4, 1000, 128, "bf16", False, "i8f8"),
    (2, 3, 777, 64, "fp16", True, "i8f8"),
    (1, 3, 1000, 128, "bf16", False, "nvfp4"),
])
def test_noalloc_matches_allocating_entry_point_on_two_calls(B, H, N, d, dtype, causal, mode):
    assert torch.cuda.is_available(), "needs a CUDA device"
    L = _lib()
    assert L.sattn_workspace_bytes(B, H, N, d, sattn.mode_code(mode, torch.bfloat16)) <= NOALLOC_MAX
    for seed in (41, 42):                      # two calls in a row: same shape, new inputs
        w = W.custom(B, H, N, d, dtype, causal=causal, seed=seed)
        q, k, v = W.make_inputs(w, "cuda")
        k += 0.5 * seed                        # shift the K mean between the calls
        ref = sattn.fwd(q, k, v, causal=causal, mode=mode)   # allocates its workspace
        out = _noalloc(L, q, k, v, causal, mode)
        torch.cuda.synchronize()
        assert torch.isfinite(out).all()
        assert torch.equal(out, ref)
    assert sattn.device_error() == 0
