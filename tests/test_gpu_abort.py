"""The bounded-wait failure paths of the attention kernels and the quantiser,
made to run on purpose.

Every wait between the roles of an attention kernel (copy producer, MMA issuer,
softmax warps) gives up after a bound, records bit 0 of the device error word,
lets the copies and MMAs already in flight complete, frees the kernel's tensor
memory and returns.  These tests shorten that bound through the library's test
hook and make the copy producer skip one key tile, so that the barrier of that
tile never completes (a flag that nothing sets).  They check that the call
returns, the device still answers, the error word says what happened, and a
later call with the normal bound gives the normal result again.  No wait is
removed and nothing faults: the only change is which barrier never completes.
"""

import pytest
import torch

import bit_quantized_attention_smooth_b200 as sattn
from bit_quantized_attention_smooth_b200 import build as sattn_build
import workloads as W

OK, INVALID = 0, 1


def test_hook_rejects_bad_tile_index_without_a_gpu():
    sattn_build.build()
    assert sattn.lib().sattn_debug_set_wait_limit(0, -2) == INVALID


@pytest.mark.gpu
@pytest.mark.parametrize("mode,causal", [("i8f8", False), ("i8f8", True), ("nvfp4", False)])
def test_wait_that_runs_out_sets_error_word_and_the_next_call_is_clean(mode, causal):
    assert torch.cuda.is_available(), "needs a CUDA device"
    sattn_build.build()
    L = sattn.lib()
    w = W.custom(1, 2, 640, 128, seed=61)           # 5 key tiles, a few CTAs
    q, k, v = W.make_inputs(w, "cuda")
    sattn.device_error(clear=True)
    ref = sattn.fwd(q, k, v, causal=causal, mode=mode)
    torch.cuda.synchronize()
    assert sattn.device_error() == 0
    try:
        # ~0.1 ms bound; key tile 2 is never loaded, so the MMA issuer's wait for it runs out
        assert L.sattn_debug_set_wait_limit(200_000, 2) == OK
        out = sattn.fwd(q, k, v, causal=causal, mode=mode)   # launches fine; the kernel gives up inside
        torch.cuda.synchronize()                             # no fault: the kernel returned
        word = sattn.device_error(clear=True)
        assert word & 1, f"error word {word}: a wait should have run out"
        assert out.shape == q.shape
    finally:
        assert L.sattn_debug_set_wait_limit(0, -1) == OK
    again = sattn.fwd(q, k, v, causal=causal, mode=mode)
    torch.cuda.synchronize()
    assert sattn.device_error() == 0
    assert torch.equal(again, ref)


@pytest.mark.gpu
@pytest.mark.parametrize("mode", ["i8f8", "nvfp4"])
def test_quantiser_statistics_wait_that_runs_out_sets_error_word_and_the_next_call_is_clean(mode):
    """The quantiser's producers wait for a head's K/V statistics before they
    hand out its K and V tiles.  The hook makes that count unreachable (a flag
    that nothing sets); with a short bound every such wait runs out, the
    kernel returns, and the next call with the hook off writes the same
    workspace as before."""
    assert torch.cuda.is_available(), "needs a CUDA device"
    sattn_build.build()
    L = sattn.lib()
    w = W.custom(1, 2, 640, 128, seed=62)
    q, k, v = W.make_inputs(w, "cuda")
    lay = sattn.workspace_layout(w.B, w.H, w.N, w.d, mode=mode, dtype=q.dtype)
    data = lay["ksum"]                               # codes and scales; the scratch after them differs
    sattn.device_error(clear=True)
    ref = sattn.quantize(q, k, v, mode=mode)[:data].clone()
    torch.cuda.synchronize()
    assert sattn.device_error() == 0
    try:
        assert L.sattn_debug_set_wait_limit(200_000, -1) == OK
        assert L.sattn_debug_withhold_statistics(1) == OK
        sattn.quantize(q, k, v, mode=mode)          # launches fine; the kernel gives up inside
        torch.cuda.synchronize()                     # no fault: the kernel returned
        word = sattn.device_error(clear=True)
        assert word & 1, f"error word {word}: a statistics wait should have run out"
    finally:
        assert L.sattn_debug_withhold_statistics(0) == OK
        assert L.sattn_debug_set_wait_limit(0, -1) == OK
    again = sattn.quantize(q, k, v, mode=mode)[:data]
    torch.cuda.synchronize()
    assert sattn.device_error() == 0
    assert torch.equal(again, ref)
