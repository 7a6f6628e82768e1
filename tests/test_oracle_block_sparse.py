"""Pins for block-sparse key skipping in the oracle (no GPU).

Reading (TurboDiffusion explainer, SLA section: part of the attention blocks
is skipped outright; here the skipped blocks come from a caller-given mask):
a mask [B, H, nblk, nblk] over 128 x 128 blocks of (query, key); the keys of a
skipped block are left out of the softmax of that block's queries, on top of
the causal mask; a row whose query block keeps no key block is zeros.
"""

import math

import numpy as np
import pytest

from oracle import attention as A
import workloads as W


def _inputs(N=300, d=16, seed=91):
    w = W.custom(1, 2, N, d, seed=seed)
    return tuple(t.float().numpy() for t in W.make_inputs(w))


def _mask(N, seed, keep=0.6):
    nb = (N + 127) // 128
    m = np.random.default_rng(seed).random((1, 2, nb, nb)) < keep
    m[:, :, np.arange(nb), np.arange(nb)] = True      # every query block keeps its diagonal block
    return m


def _brute(q, k, v, mask, causal, s):
    """Per row: the allowed keys listed explicitly, plain softmax over them."""
    N, d = q.shape
    out = np.zeros((N, d))
    for i in range(N):
        keys = [j for j in range(N) if mask[i // 128, j // 128] and (not causal or j <= i)]
        if not keys:
            continue
        sc = np.array([float(q[i].astype(np.float64) @ k[j].astype(np.float64)) * s for j in keys])
        p = np.exp(sc - sc.max())
        out[i] = (p[:, None] * v[keys].astype(np.float64)).sum(axis=0) / p.sum()
    return out


@pytest.mark.parametrize("causal", [False, True])
def test_exact_block_sparse_matches_brute_force(causal):
    q, k, v = _inputs()
    m = _mask(300, 3)
    o = A.attn_exact(q, k, v, causal=causal, block_mask=m)
    for h in range(2):
        ref = _brute(q[0, h], k[0, h], v[0, h], m[0, h], causal, 1 / math.sqrt(16))
        assert np.abs(o[h] - ref).max() < 1e-12


def test_all_ones_mask_is_dense():
    q, k, v = _inputs()
    ones = np.ones((1, 2, 3, 3), dtype=bool)
    for f in (A.attn_exact, A.attn_quant_emul_i8f8, A.attn_quant_emul_nvfp4):
        assert np.array_equal(f(q, k, v, block_mask=ones), f(q, k, v))


@pytest.mark.parametrize("causal,tau", [(False, 0.0), (True, 4.0)])
def test_streaming_with_skipped_tiles_equals_exact(causal, tau):
    q, k, v = _inputs()
    m = _mask(300, 4)
    a = A.attn_exact(q, k, v, causal=causal, block_mask=m)
    b = A.attn_online_unquantised(q, k, v, causal=causal, block_kv=128, tau=tau, block_mask=m)
    assert np.abs(a - b).max() < 1e-12


def test_query_block_without_keys_is_zero():
    q, k, v = _inputs()
    m = np.ones((1, 2, 3, 3), dtype=bool)
    m[0, 1, 2, :] = False                              # head 1, query block 2 keeps nothing
    for f in (A.attn_exact, A.attn_quant_emul_i8f8, A.attn_quant_emul_nvfp4):
        o = f(q, k, v, block_mask=m)
        assert np.all(o[1, 256:] == 0)
        assert np.all(np.isfinite(o))
        assert np.abs(o[1, :256]).max() > 0
