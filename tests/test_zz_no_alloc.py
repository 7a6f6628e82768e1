"""sattn_fwd_noalloc: the entry point for callers that cannot allocate device memory.

Some callers own every byte of device memory (an inference engine that
reserves its budget up front and loads this library as a plugin, a process
whose allocator is locked after start-up) and cannot let the library call
cudaMalloc.  sattn_fwd_noalloc takes its workspace from a static device array
instead.  These tests call it through the C ABI and compare it with sattn_fwd,
the entry point that allocates its own workspace, on two calls in a row with
different inputs (the array keeps the previous call's contents, so the second
call checks that nothing stale leaks through).  The file is collected last on
purpose: a failure here comes after every other test has run.
"""

import ctypes

import numpy as np
import pytest
import torch

import bit_quantized_attention_smooth_b200 as sattn
from bit_quantized_attention_smooth_b200 import build as sattn_build
import workloads as W

NOALLOC_MAX = 64 << 20
WORKSPACE_ERR = 3
MAX_ABS, MEAN_ABS = 2e-2, 2e-3      # the tolerance of the parity tests


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


@pytest.mark.gpu
def test_noalloc_matches_allocating_entry_point_on_two_calls():
    assert torch.cuda.is_available(), "needs a CUDA device"
    L = _lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    cases = [W.custom(1, 4, 1000, 128, seed=41), W.custom(2, 3, 777, 64, "fp16", seed=42)]
    for w in cases:                            # two calls in a row, different inputs
        assert L.sattn_workspace_bytes(w.B, w.H, w.N, w.d, 0) <= NOALLOC_MAX
        q, k, v = W.make_inputs(w, "cuda")
        ref = sattn.fwd(q, k, v)               # existing entry point (allocates its workspace)
        out = torch.full_like(q, float("nan"))
        mode = sattn.mode_code("i8f8", q.dtype)
        st = L.sattn_fwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                 w.B, w.H, w.N, w.d, 0, 0.0, mode, stream)
        assert st == 0, sattn.STATUS.get(st, st)
        torch.cuda.synchronize()
        a = out.float().cpu().numpy()
        b = ref.float().cpu().numpy()
        assert np.isfinite(a).all()
        err = np.abs(a - b)
        assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())
    assert sattn.device_error() == 0
