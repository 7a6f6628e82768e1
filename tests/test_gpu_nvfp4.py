"""GPU parity of the NVFP4 path against the CPU oracle.

Quantiser outputs (E2M1 codes, E4M3 block scales, K mean) are compared bit for
bit.  Attention outputs are compared element by element with the oracle's
NVFP4 emulation: max |err| <= 6e-2 and mean |err| <= 6e-3, and with the exact
float64 attention by cosine similarity (>= 0.995, or no worse than the
emulation itself by 1e-3 where the scheme's own accuracy is lower).
"""

import numpy as np
import pytest
import torch

import bit_quantized_attention_smooth_b200 as sattn
from bit_quantized_attention_smooth_b200 import build as sattn_build
from oracle import attention as A
from oracle import quant as Qz
from oracle.formats import e2m1_decode
import workloads as W

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS, COS = 6e-2, 6e-3, 0.995


@pytest.fixture(scope="module", autouse=True)
def gpu_lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    sattn_build.build()
    sattn.lib()
    sattn.device_error(clear=True)
    yield
    assert sattn.device_error() == 0, "a kernel wait ran out of time"


def _unpack_nibbles(b):
    b = np.asarray(b, dtype=np.uint8)
    out = np.empty(b.shape[:-1] + (b.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = b & 0xF
    out[..., 1::2] = b >> 4
    return out


def _sf_unblock(blocks, rows, nblk_per_row):
    """[ntile][nslice][512] blocked scales -> [ntile*128 rows][nslice*4] codes."""
    ntile, nslice = blocks.shape[0], blocks.shape[1]
    out = np.zeros((ntile * 128, nslice * 4), dtype=np.uint8)
    r = np.arange(128)
    for t in range(ntile):
        for s in range(nslice):
            for b in range(4):
                out[t * 128 + r, s * 4 + b] = blocks[t, s, 16 * (r % 32) + 4 * (r // 32) + b]
    return out[:rows, :nblk_per_row]


def _same_fp4(a, b):
    # +0 and -0 encode the same value
    return np.array_equal(e2m1_decode(a), e2m1_decode(b))


QUANT_CASES = [W.custom(1, 2, 256, 64, "fp16", seed=31),
               W.custom(1, 2, 300, 128, seed=32, q_outlier_frac=1e-3),
               W.custom(2, 1, 129, 64, seed=33),
               W.custom(1, 1, 1, 128, seed=34)]


@pytest.mark.parametrize("w", QUANT_CASES, ids=lambda w: w.name)
def test_nvfp4_quantizer_bit_exact(w):
    q, k, v = W.make_inputs(w, "cuda")
    ws = sattn.quantize(q, k, v, mode="nvfp4")
    torch.cuda.synchronize()
    lay = sattn.workspace_layout(w.B, w.H, w.N, w.d, mode="nvfp4", dtype=q.dtype)
    h = ws.cpu().numpy()
    BH, N, d, nv, nb = w.B * w.H, w.N, w.d, lay["nv"], lay["nblk"]
    ns = d // 64

    def sec(key, n):
        return h[lay[key]: lay[key] + n]

    q4 = sec("q8", BH * N * d // 2).reshape(BH, N, d // 2)
    k4 = sec("k8", BH * N * d // 2).reshape(BH, N, d // 2)
    vt4 = sec("vt8", BH * d * nv // 2).reshape(BH, d, nv // 2)
    sfq = sec("sq", BH * nb * ns * 512).reshape(BH, nb, ns, 512)
    sfk = sec("sk", BH * nb * ns * 512).reshape(BH, nb, ns, 512)
    sfv = sec("sv", BH * nb * 1024).reshape(BH, nb, 2, 512)
    mu = sec("mu", BH * d * 4).view(np.float32).reshape(BH, d)
    qf, kf, vf = (t.float().cpu().numpy() for t in (q, k, v))
    for b in range(w.B):
        for hh in range(w.H):
            bh = b * w.H + hh
            z = Qz.quantize_head_nvfp4(qf[b, hh], kf[b, hh], vf[b, hh])
            assert np.array_equal(mu[bh], z["mu"])
            assert _same_fp4(_unpack_nibbles(q4[bh]), z["q"])
            assert _same_fp4(_unpack_nibbles(k4[bh]), z["k"])
            assert np.array_equal(_sf_unblock(sfq[bh], N, d // 16), z["q_sc_codes"])
            assert np.array_equal(_sf_unblock(sfk[bh], N, d // 16), z["k_sc_codes"])
            gv = _unpack_nibbles(vt4[bh])[:, :z["vt"].shape[1]]
            assert _same_fp4(gv[:, :N], z["vt"][:, :N])
            # V scales: rows are channels, blocks run along tokens
            gsv = np.zeros((d, nb * 8), dtype=np.uint8)
            for t in range(nb):
                gsv[:, t * 8:(t + 1) * 8] = _sf_unblock(sfv[bh, t][None], d, 8)
            nblk_tok = (N + 15) // 16
            assert np.array_equal(gsv[:, :nblk_tok], z["vt_sc_codes"][:, :nblk_tok])


def _check(w, causal, rows=None, heads=None, via_fwd=False):
    q, k, v = W.make_inputs(w, "cuda")
    if via_fwd:
        out = sattn.fwd(q, k, v, causal=causal, mode="nvfp4")
    else:
        ws = sattn.quantize(q, k, v, mode="nvfp4")
        out = sattn.fwd_quantized(ws, q.shape, causal=causal, mode="nvfp4", dtype=q.dtype)
    torch.cuda.synchronize()
    if heads is None:
        heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    rows_idx = np.arange(w.N) if rows is None else np.asarray(rows)
    qf, kf, vf = W.make_heads_f32(w, heads)
    emu = A.attn_quant_emul_nvfp4(qf, kf, vf, causal=causal, rows=rows_idx)
    exact = A.attn_exact(qf, kf, vf, causal=causal, rows=rows_idx)
    o = out.float().cpu().numpy()
    got = np.stack([o[b, h][rows_idx] for (b, h) in heads])
    err = np.abs(got - emu)
    cos_gpu, cos_emu = A.cosine(exact, got), A.cosine(exact, emu)
    print(f"{w.name} causal={causal}: max|err|={err.max():.3e} mean|err|={err.mean():.3e} "
          f"cos(gpu,exact)={cos_gpu:.6f} cos(emul,exact)={cos_emu:.6f}")
    assert np.isfinite(got).all()
    assert err.max() <= MAX_ABS
    assert err.mean() <= MEAN_ABS
    assert cos_gpu >= min(COS, cos_emu - 1e-3)


ATTN_CASES = [
    (W.custom(1, 2, 256, 64, "fp16", seed=41), False),
    (W.custom(1, 2, 1, 128, seed=42), False),
    (W.custom(1, 2, 17, 64, seed=43), True),
    (W.custom(1, 3, 129, 128, seed=44), True),
    (W.custom(2, 2, 300, 64, seed=45), False),
    (W.custom(1, 2, 1000, 128, seed=46, q_outlier_frac=1e-3), False),
    (W.custom(1, 2, 1100, 128, seed=47), True),
]


@pytest.mark.parametrize("w,causal", ATTN_CASES, ids=lambda x: getattr(x, "name", str(x)))
def test_nvfp4_attention_matches_oracle(w, causal):
    _check(w, causal)


def test_nvfp4_mid_workload_sampled():
    rows = np.concatenate([np.arange(0, 4096, 97), [4095]])
    _check(W.MID, False, rows=rows)


def test_nvfp4_video_32760_sampled():
    w = W.VIDEO_32760
    rows = np.concatenate([np.random.default_rng(2).choice(w.N, 40, replace=False), [0, 32759]])
    _check(w, False, rows=rows, heads=[(0, 0), (0, 6), (0, 11)], via_fwd=True)


def test_nvfp4_video_75600_sampled():
    w = W.VIDEO_75600
    rows = np.concatenate([np.random.default_rng(3).choice(w.N, 40, replace=False), [0, 75599]])
    _check(w, False, rows=rows, heads=[(0, 0), (0, 21), (0, 39)])


@pytest.mark.parametrize("d,N,causal", [(64, 2048, True), (128, 8192, False)])
def test_nvfp4_sweep_points_sampled(d, N, causal):
    w = W.sweep(d, N, causal)
    rows = np.concatenate([np.random.default_rng(N + 1).choice(N, 32, replace=False), [0, N - 1]])
    _check(w, causal, rows=rows, heads=[(0, 0), (3, 31)])
