"""GPU parity of block-sparse key skipping (both modes) against the oracle.

A mask over 128 x 128 (query, key) blocks drops whole blocks from the
softmax; the kernel neither loads nor multiplies their K/V tiles.  Compared
element by element with the oracle's emulation under the same mask (same
tolerance as the dense path); an all-ones mask must give the dense output bit
for bit; a query block that keeps no key block gives zeros.
"""

import numpy as np
import pytest
import torch

import bit_quantized_attention_smooth_b200 as sattn
from bit_quantized_attention_smooth_b200 import build as sattn_build
from oracle import attention as A
import workloads as W

pytestmark = pytest.mark.gpu
MAX_ABS, MEAN_ABS = 2e-2, 2e-3


@pytest.fixture(scope="module", autouse=True)
def gpu_lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    sattn_build.build()
    sattn.lib()
    sattn.device_error(clear=True)
    yield
    assert sattn.device_error() == 0, "a kernel wait ran out of time"


def _mask(B, H, N, seed, keep, empty_block=None):
    nb = (N + 127) // 128
    m = np.random.default_rng(seed).random((B, H, nb, nb)) < keep
    if empty_block is not None:
        b, h, i = empty_block
        m[b, h, i, :] = False
    return m


@pytest.mark.parametrize("B,H,N,d,dtype,causal,keep,qtok,empty", [
    (1, 2, 1000, 128, "bf16", False, 0.5, False, (0, 1, 3)),
    (1, 3, 900, 128, "bf16", True, 0.6, False, (0, 0, 5)),
    (2, 2, 700, 64, "fp16", False, 0.3, False, None),
    (1, 2, 1300, 64, "bf16", True, 0.7, True, (0, 1, 0)),
    (1, 1, 2560, 128, "bf16", False, 0.15, False, None),
])
def test_block_sparse_matches_oracle(B, H, N, d, dtype, causal, keep, qtok, empty):
    w = W.custom(B, H, N, d, dtype, causal=causal, seed=N + d)
    q, k, v = W.make_inputs(w, "cuda")
    m = _mask(B, H, N, N, keep, empty)
    out = sattn.fwd_sparse(q, k, v, torch.from_numpy(m.astype(np.uint8)).cuda(), causal=causal, q_per_token=qtok)
    torch.cuda.synchronize()
    got = out.float().cpu().numpy().reshape(B * H, N, d)
    qf, kf, vf = (t.float().cpu().numpy() for t in (q, k, v))
    emu = A.attn_quant_emul_i8f8(qf, kf, vf, causal=causal, block_q=1 if qtok else 128,
                                 tau=sattn.I8F8_LAZY_TAU, block_mask=m)
    err = np.abs(got - emu)
    print(f"block-sparse {w.name} causal={causal} keep={keep}: max|err|={err.max():.3e} mean|err|={err.mean():.3e}")
    assert np.isfinite(got).all()
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS
    if empty is not None:
        b, h, i = empty
        assert np.all(got[b * H + h, i * 128:(i + 1) * 128] == 0)


@pytest.mark.parametrize("causal", [False, True])
def test_all_ones_mask_is_bit_identical_to_dense(causal):
    w = W.custom(1, 2, 1100, 128, seed=93)
    q, k, v = W.make_inputs(w, "cuda")
    ones = torch.ones((1, 2, 9, 9), dtype=torch.uint8, device="cuda")
    a = sattn.fwd_sparse(q, k, v, ones, causal=causal)
    b = sattn.fwd(q, k, v, causal=causal)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_sparse_quantized_entry_point_and_launch_count():
    w = W.custom(1, 2, 600, 64, seed=94)
    q, k, v = W.make_inputs(w, "cuda")
    m = torch.from_numpy(_mask(1, 2, 600, 5, 0.5).astype(np.uint8)).cuda()
    ws = sattn.quantize(q, k, v)
    sattn.kernel_launches(reset=True)
    a = sattn.fwd_quantized_sparse(ws, q.shape, m, dtype=q.dtype)
    assert sattn.kernel_launches() == 1
    b = sattn.fwd_sparse(q, k, v, m)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


@pytest.mark.parametrize("B,H,N,d,causal,keep,empty", [
    (1, 2, 1000, 128, False, 0.5, (0, 1, 2)),
    (1, 2, 700, 64, True, 0.6, (0, 0, 4)),
])
def test_nvfp4_block_sparse_matches_oracle(B, H, N, d, causal, keep, empty):
    w = W.custom(B, H, N, d, causal=causal, seed=N + 2 * d)
    q, k, v = W.make_inputs(w, "cuda")
    m = _mask(B, H, N, N + 1, keep, empty)
    out = sattn.fwd_sparse(q, k, v, torch.from_numpy(m.astype(np.uint8)).cuda(), causal=causal, mode="nvfp4")
    torch.cuda.synchronize()
    got = out.float().cpu().numpy().reshape(B * H, N, d)
    qf, kf, vf = (t.float().cpu().numpy() for t in (q, k, v))
    emu = A.attn_quant_emul_nvfp4(qf, kf, vf, causal=causal, block_mask=m)
    err = np.abs(got - emu)
    print(f"nvfp4 block-sparse {w.name} causal={causal}: max|err|={err.max():.3e} mean|err|={err.mean():.3e}")
    assert np.isfinite(got).all()
    assert err.max() <= 6e-2 and err.mean() <= 6e-3
    b, h, i = empty
    assert np.all(got[b * H + h, i * 128:(i + 1) * 128] == 0)


def test_nvfp4_all_ones_mask_is_bit_identical_to_dense():
    w = W.custom(1, 2, 900, 128, seed=95)
    q, k, v = W.make_inputs(w, "cuda")
    ones = torch.ones((1, 2, 8, 8), dtype=torch.uint8, device="cuda")
    a = sattn.fwd_sparse(q, k, v, ones, mode="nvfp4")
    b = sattn.fwd(q, k, v, mode="nvfp4")
    torch.cuda.synchronize()
    assert torch.equal(a, b)
