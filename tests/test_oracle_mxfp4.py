"""Pins for the MXFP4 ablation in the oracle (no GPU).

The SageAttention tag page (reportify.cn), SageAttention3 summary, FP4 bullet
[15], chooses NVFP4 (1 x 16 blocks, E4M3 scales) over MXFP4 (1 x 32 blocks,
E8M0 power-of-two scales) and reports it more accurate (99.52 % vs 98.37 %).
MXFP4 here is the OCP Microscaling definition: scale 2^(floor(log2 amax) - 2),
E2M1 elements, round-to-nearest-even, saturating at 6.
"""

import numpy as np
import pytest

from oracle import attention as A
from oracle import quant as Qz
from oracle.formats import e8m0_decode, mx_scale_code, e2m1_decode
import workloads as W


def test_e8m0_table():
    v = e8m0_decode(np.arange(256, dtype=np.uint8))
    assert np.isnan(v[255])
    for c in range(255):
        assert v[c] == 2.0 ** (c - 127)


def test_mx_scale_code_by_brute_force():
    rng = np.random.default_rng(5)
    amax = np.concatenate([np.exp2(rng.uniform(-40, 40, 500)), 2.0 ** np.arange(-20, 21),
                           2.0 ** np.arange(-20, 21) * (1 - 2 ** -20)])
    codes = mx_scale_code(amax, 2)
    tab = e8m0_decode(np.arange(255, dtype=np.uint8))
    for a, c in zip(amax, codes):
        # the largest scale whose element-range top binade [4, 8) still starts at or below amax
        want = max(i for i in range(255) if tab[i] * 4 <= a)
        assert c == want, (a, c, want)
        assert 4 * tab[c] <= a < 8 * tab[c]
    assert mx_scale_code(0.0, 2) == 0 and mx_scale_code(np.nan, 2) == 255


def test_mxfp4_block_bounds():
    w = W.custom(1, 1, 64, 64, seed=81)
    x = W.make_inputs(w)[0][0, 0].float().numpy()
    codes, sc_codes, sc = Qz.mxfp4_quant_rows(x)
    assert codes.shape == (64, 64) and sc.shape == (64, 2)
    deq = Qz.nvfp4_dequant_rows(codes, sc, block=32)
    xb = x.reshape(64, 2, 32).astype(np.float64)
    db = deq.reshape(64, 2, 32)
    s = sc[:, :, None]
    y = np.abs(xb) / s
    halfgap = np.where(y < 2, 0.25, np.where(y < 4, 0.5, 1.0))
    sat = np.maximum(0.0, np.abs(xb) - 6 * s)
    assert np.all(np.abs(xb - db) <= s * halfgap + sat + 1e-12)
    amax = np.abs(xb).max(axis=2)
    assert np.all((4 * sc <= amax) & (amax < 8 * sc))
    # codes are plain E2M1 values of x / scale
    assert np.array_equal(e2m1_decode(codes).reshape(64, 2, 32) * s, db)


@pytest.mark.parametrize("w,rows", [
    (W.SMALL, np.arange(0, 256, 4)),
    (W.MID, np.arange(0, 4096, 64)),
    (W.VIDEO_32760, np.linspace(0, 32759, 48).astype(np.int64)),
], ids=lambda x: getattr(x, "name", "rows"))
def test_nvfp4_is_more_accurate_than_mxfp4(w, rows):
    """The pages' ordering: the same scheme in NVFP4 beats it in MXFP4 (cosine to
    exact attention), on the first three workloads (sampled heads and rows)."""
    heads = [(0, 0), (0, w.H - 1)]
    q, k, v = W.make_heads_f32(w, heads)
    e = A.attn_exact(q, k, v, rows=rows)
    nv = A.attn_quant_emul_nvfp4(q, k, v, rows=rows)
    mx = A.attn_quant_emul_nvfp4(q, k, v, rows=rows, fmt="mxfp4")
    c_nv, c_mx = A.cosine(e, nv), A.cosine(e, mx)
    print(f"{w.name}: cos NVFP4 {c_nv:.5f}  MXFP4 {c_mx:.5f}")
    assert c_nv > c_mx


def test_quantize_head_mxfp4_matches_the_emulations_operands():
    """The per-head MXFP4 operands (the quantiser's target on the GPU) decode to
    the operands the MXFP4 emulation multiplies: Q, K - mean along channels, V
    along tokens; every block's largest magnitude lies in [4, 8) x its scale."""
    w = W.custom(1, 1, 77, 64, seed=82)
    q, k, v = (t[0, 0].float().numpy() for t in W.make_inputs(w))
    z = Qz.quantize_head_mxfp4(q, k, v)
    kp = Qz.smooth_k(k, Qz.k_channel_mean(k))
    for key, x in (("q", q), ("k", kp), ("vt", np.ascontiguousarray(v.T))):
        deq = Qz.nvfp4_dequant_rows(z[key], z[key + "_sc"], block=32)
        assert np.array_equal(deq[:, :x.shape[1]], Qz.fp4_rows(x, "mxfp4")[:, :x.shape[1]])
        xp = np.zeros(deq.shape)
        xp[:, :x.shape[1]] = x
        amax = np.abs(xp.reshape(xp.shape[0], -1, 32)).max(axis=2)
        sc = e8m0_decode(z[key + "_sc_codes"])
        live = amax > 0
        assert np.all((4 * sc[live] <= amax[live]) & (amax[live] < 8 * sc[live]))
    # V padded with zero tokens up to a multiple of 32
    assert z["vt"].shape == (64, 96) and not np.any(e2m1_decode(z["vt"][:, 77:]))
