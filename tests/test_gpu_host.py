"""sattn_fwd_host: the forward pass over host buffers, pipelined in chunks of heads.

The call splits the heads into chunks that are copied in, computed and copied
out on separate streams.  Heads are independent and every quantisation scale
is per head, so its output must equal sattn_fwd's bit for bit; these tests
check that on shapes with one chunk, several chunks and a short last chunk,
in both modes, both I/O types and with the causal mask, and on two calls in a
row with different inputs (the device slots are reused across calls).
"""

import pytest
import torch

import bit_quantized_attention_smooth_b200 as sattn
from bit_quantized_attention_smooth_b200 import build as sattn_build
import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def gpu_lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    sattn_build.build()
    sattn.lib()
    sattn.device_error(clear=True)
    yield
    assert sattn.device_error() == 0, "a kernel wait ran out of time"


def _host_vs_device(w, causal, mode):
    q, k, v = (t.pin_memory() for t in W.make_inputs(w, "cpu"))
    ref = sattn.fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, mode=mode).cpu()
    out = sattn.fwd_host(q, k, v, causal=causal, mode=mode)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)


@pytest.mark.parametrize("B,H,N,d,dtype,causal,mode", [
    (2, 3, 1000, 128, "bf16", False, "i8f8"),     # 6 heads: 3 chunks of 2
    (1, 5, 700, 128, "bf16", True, "i8f8"),       # 5 heads: chunks of 2, 2, 1
    (1, 1, 300, 64, "fp16", True, "i8f8"),        # one chunk
    (1, 5, 700, 128, "bf16", False, "nvfp4"),
    (2, 2, 520, 64, "fp16", True, "nvfp4"),
])
def test_fwd_host_is_bit_identical_to_fwd(B, H, N, d, dtype, causal, mode):
    _host_vs_device(W.custom(B, H, N, d, dtype, seed=31 + N), causal, mode)


def test_fwd_host_two_calls_in_a_row():
    shape = (1, 6, 900, 128)
    outs, refs = [], []
    for seed in (41, 42):
        w = W.custom(*shape, seed=seed)
        q, k, v = (t.pin_memory() for t in W.make_inputs(w, "cpu"))
        refs.append(sattn.fwd(q.cuda(), k.cuda(), v.cuda()).cpu())
        outs.append(sattn.fwd_host(q, k, v))
    torch.cuda.synchronize()
    for o, r in zip(outs, refs):
        assert torch.equal(o, r)


def test_fwd_host_is_ordered_on_the_callers_stream():
    w = W.custom(1, 4, 800, 64, seed=43)
    q, k, v = (t.pin_memory() for t in W.make_inputs(w, "cpu"))
    ref = sattn.fwd(q.cuda(), k.cuda(), v.cuda()).cpu()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        torch.cuda._sleep(20_000_000)          # queue work ahead of the call on the same stream
        out = sattn.fwd_host(q, k, v)
    s.synchronize()
    assert torch.equal(out, ref)
