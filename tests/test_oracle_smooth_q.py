"""Pins for the Q-smoothing and per-token-P variants of the I8F8 scheme (oracle only).

Q smoothing subtracts each query block's channel mean before the INT8
quantisation and adds the exact correction qbar . K'_j back to the scores, so
with exact arithmetic the softmax does not change; per-token P rescales each
row's P tile so that its maximum maps to 448 and multiplies the tile's
contribution back.
"""

import numpy as np
import pytest

from oracle import attention as A
from oracle import quant as Qz
from oracle.formats import e4m3_decode
import workloads as W


def _inputs(N=300, d=32, seed=101, bias=0.0):
    w = W.custom(1, 2, N, d, seed=seed)
    q, k, v = (t.float().numpy() for t in W.make_inputs(w))
    q = (q + np.float32(bias) * np.linspace(-1, 1, d, dtype=np.float32)[None, None, None, :]).astype(np.float32)
    return q, k, v


def test_smoothing_is_exact_in_float64():
    """softmax((Q - qbar) K^T + qbar K^T) == softmax(Q K^T): the correction term
    restores the scores exactly (float64, no quantisation)."""
    q, k, v, = _inputs(bias=3.0)
    e = A.attn_exact(q, k, v)
    q64 = q.astype(np.float64)
    for b0 in range(0, 300, 128):
        qbar = q64[:, :, b0:b0 + 128].mean(axis=2, keepdims=True)
        S = ((q64[:, :, b0:b0 + 128] - qbar) @ np.swapaxes(k.astype(np.float64), 2, 3)
             + qbar @ np.swapaxes(k.astype(np.float64), 2, 3)) / np.sqrt(32)
        P = np.exp(S - S.max(axis=3, keepdims=True))
        o = (P @ v.astype(np.float64)) / P.sum(axis=3, keepdims=True)
        assert np.abs(o[0] - e[:, b0:b0 + 128]).max() < 1e-12


def test_without_smoothing_or_per_token_p_it_is_the_i8f8_emulation():
    q, k, v = _inputs()
    a = A.attn_quant_emul_i8f8_smooth(q, k, v, smooth_q=False, p_per_token=False)
    b = A.attn_quant_emul_i8f8(q, k, v)
    assert np.abs(a - b).max() < 1e-12


def test_uniform_queries_give_mean_of_dequantised_v_in_every_variant():
    _, k, v = _inputs()
    q = np.zeros_like(k)
    v8, sv = Qz.quant_v_fp8(v[0, 0])
    want = (e4m3_decode(v8) * sv.astype(np.float64)[None, :]).mean(axis=0)
    for sq_, pt in ((True, False), (False, True), (True, True)):
        o = A.attn_quant_emul_i8f8_smooth(q, k, v, smooth_q=sq_, p_per_token=pt)[0]
        assert np.abs(o - want[None, :]).max() < 1e-12


def test_smoothing_removes_a_query_channel_bias_from_the_int8_error():
    """With a large per-channel bias in Q the INT8 step of a block is set by the
    bias; smoothing quantises only the deviations, so the result is closer to
    exact attention (the reason for outlier smoothing)."""
    q, k, v = _inputs(N=512, bias=8.0)
    e = A.attn_exact(q, k, v)
    plain = A.attn_quant_emul_i8f8_smooth(q, k, v, smooth_q=False)
    smooth = A.attn_quant_emul_i8f8_smooth(q, k, v, smooth_q=True)
    assert A.cosine(e, smooth) > A.cosine(e, plain)
    assert np.abs(smooth - e).mean() < np.abs(plain - e).mean()


@pytest.mark.parametrize("causal", [False, True])
def test_per_token_p_keeps_the_one_hot_and_causal_cases(causal):
    q, k, v = _inputs(N=200)
    o = A.attn_quant_emul_i8f8_smooth(q, k, v, causal=causal, smooth_q=False, p_per_token=True)
    z = A.attn_quant_emul_i8f8(q, k, v, causal=causal)
    assert np.isfinite(o).all()
    assert np.abs(o - z).max() < 3e-2          # same scheme up to the FP8 rounding of P
    e = A.attn_exact(q, k, v, causal=causal)
    assert A.cosine(e, o) > 0.999


def test_nvfp4_smoothing_without_bias_changes_little_and_with_bias_helps():
    q, k, v = _inputs(N=512, bias=8.0)
    e = A.attn_exact(q, k, v)
    plain = A.attn_quant_emul_nvfp4(q, k, v)
    smooth = A.attn_quant_emul_nvfp4(q, k, v, smooth_q=True)
    assert A.cosine(e, smooth) > A.cosine(e, plain)
