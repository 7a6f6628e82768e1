"""Pins for the 8-bit attention backward in the oracle (no GPU).

With every quantiser replaced by the identity the emulation must equal the
exact attention backward, here computed by torch autograd in float64 on the
CPU (an independent library routine); the 8-bit version must stay close to
it; subtracting the K channel mean must not change dK.
"""

import numpy as np
import pytest
import torch

from oracle import backward as BW
import workloads as W


def _inputs(N, d, seed):
    w = W.custom(1, 1, N, d, seed=seed)
    q, k, v = (t.float().numpy()[0, 0] for t in W.make_inputs(w))
    do = np.random.default_rng(seed).standard_normal((N, d)).astype(np.float32)
    return q, k, v, do


def _autograd(q, k, v, do, s):
    qt, kt, vt = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    o = torch.softmax(qt @ kt.T * s, dim=1) @ vt
    o.backward(torch.tensor(do, dtype=torch.float64))
    return o.detach().numpy(), qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy()


@pytest.mark.parametrize("N,d", [(200, 32), (300, 64)])
def test_unquantised_emulation_is_the_exact_backward(N, d):
    q, k, v, do = _inputs(N, d, N + d)
    s = 1 / np.sqrt(d)
    got = BW.attn_fwd_bwd_8bit(q, k, v, do, quantise=False)
    ref = _autograd(q, k, v, do, s)
    for g, r in zip(got, ref):
        assert np.abs(g - r).max() < 1e-10 * max(1.0, np.abs(r).max())


def test_k_smoothing_leaves_dk_unchanged():
    """The rows of dS sum to zero, so the gradient through the K mean vanishes:
    autograd of softmax(Q (K - mean K)^T) V gives the same dK as without the mean."""
    q, k, v, do = _inputs(150, 32, 7)
    s = 1 / np.sqrt(32)
    _, _, dk1, _ = _autograd(q, k, v, do, s)
    kt = torch.tensor(k, dtype=torch.float64, requires_grad=True)
    qt, vt = torch.tensor(q, dtype=torch.float64), torch.tensor(v, dtype=torch.float64)
    o = torch.softmax(qt @ (kt - kt.mean(dim=0, keepdim=True)).T * s, dim=1) @ vt
    o.backward(torch.tensor(do, dtype=torch.float64))
    assert np.abs(kt.grad.numpy() - dk1).max() < 1e-12


def test_8bit_backward_stays_close_to_exact():
    q, k, v, do = _inputs(512, 64, 11)
    s = 1 / np.sqrt(64)
    got = BW.attn_fwd_bwd_8bit(q, k, v, do)
    ref = _autograd(q, k, v, do, s)
    for name, g, r in zip(("O", "dQ", "dK", "dV"), got, ref):
        cos = float((g * r).sum() / (np.linalg.norm(g) * np.linalg.norm(r)))
        print(f"{name}: cosine to exact {cos:.5f}")
        assert cos > 0.99, (name, cos)
