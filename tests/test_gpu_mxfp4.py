"""GPU parity of the MXFP4 ablation of the NVFP4 mode against the CPU oracle.

The SageAttention tag page (reportify.cn), SageAttention3 summary, FP4 bullet
[15], compares NVFP4 (E4M3 scale per 16 values) with MXFP4 (E8M0 scale per 32
values) and reports NVFP4 more accurate.  SATTN_MXFP4 runs the NVFP4 scheme
with every FP4 operand in MXFP4 (OCP Microscaling: scale 2^(floor(log2
max|x|) - 2), E2M1 values).

Quantiser outputs (E2M1 codes, E8M0 scale codes, each stored at both 16-value
positions of its 32-value block, K mean) are compared bit for bit with the
oracle's.  Attention outputs are compared element by element with the
oracle's MXFP4 emulation, with the FP4 tolerance (max |err| <= 6e-2, mean
|err| <= 6e-3).  The scheme's cosine to exact attention is below 0.995 on every
input (strict expected failures carrying the emulation's value), and below
NVFP4's on the same input, as the pages report.
"""

import dataclasses

import numpy as np
import pytest
import torch

import bit_quantized_attention_smooth_b200 as sattn
from bit_quantized_attention_smooth_b200 import build as sattn_build
from oracle import attention as A
from oracle import quant as Qz
import workloads as W
from tests.gpu_parity import check_cosine_bar, check_parity, miss_params, run_case
from tests.test_gpu_nvfp4 import ATTN_CASES, QUANT_CASES, _same_fp4, _sf_unblock, _unpack_nibbles

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def gpu_lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    sattn_build.build()
    sattn.lib()
    sattn.device_error(clear=True)
    yield
    assert sattn.device_error() == 0, "a kernel wait ran out of time"


def _pairs_equal(blocks16, codes32):
    """Scale codes per 16-value position [rows, 2n] against per-32 codes [rows, n]."""
    n = codes32.shape[1]
    return (np.array_equal(blocks16[:, 0:2 * n:2], codes32) and
            np.array_equal(blocks16[:, 1:2 * n:2], codes32))


@pytest.mark.parametrize("w", QUANT_CASES, ids=lambda w: w.name)
def test_mxfp4_quantizer_bit_exact(w):
    q, k, v = W.make_inputs(w, "cuda")
    ws = sattn.quantize(q, k, v, mode="mxfp4")
    torch.cuda.synchronize()
    lay = sattn.workspace_layout(w.B, w.H, w.N, w.d, mode="mxfp4", dtype=q.dtype)
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
            z = Qz.quantize_head_mxfp4(qf[b, hh], kf[b, hh], vf[b, hh])
            assert np.array_equal(mu[bh], z["mu"])
            assert _same_fp4(_unpack_nibbles(q4[bh]), z["q"])
            assert _same_fp4(_unpack_nibbles(k4[bh]), z["k"])
            assert _pairs_equal(_sf_unblock(sfq[bh], N, d // 16), z["q_sc_codes"])
            assert _pairs_equal(_sf_unblock(sfk[bh], N, d // 16), z["k_sc_codes"])
            gv = _unpack_nibbles(vt4[bh])[:, :z["vt"].shape[1]]
            assert _same_fp4(gv[:, :N], z["vt"][:, :N])
            gsv = np.zeros((d, nb * 8), dtype=np.uint8)
            for t in range(nb):
                gsv[:, t * 8:(t + 1) * 8] = _sf_unblock(sfv[bh, t][None], d, 8)
            assert _pairs_equal(gsv, z["vt_sc_codes"])


# The MXFP4 emulation's cosine to exact attention on the NVFP4 test inputs
# (oracle, same rows and heads); NVFP4's is 0.94-0.9997 on the same inputs.
MX_COS = {
    "custom-B1H2N256d64": 0.96958,
    "custom-B1H2N1d128": 0.99353,
    "custom-B1H2N17d64-causal": 0.98599,
    "custom-B1H3N129d128-causal": 0.97773,
    "custom-B2H2N300d64": 0.97050,
    "custom-B1H2N1000d128": 0.83135,
    "custom-B1H2N1100d128-causal": 0.97671,
    "mid-B1H12N4096d128-sampled": 0.56385,
    "video-21x30x52-B1H12N32760d128-sampled": 0.69060,
    "video-21x45x80-B1H40N75600d128-sampled": 0.96956,
    "sweep-B4H32N2048d64-causal-sampled": 0.98892,
    "sweep-B4H32N8192d128-sampled": 0.96642,
}
MISS = ("MXFP4 E2M1 with E8M0 scales per 32 values: the scheme's own cosine to exact attention is {:.5f} "
        "here (a x20 Q outlier zeroes its whole 32-channel block and saturates near 6 x scale)")
MX_CASES = [dataclasses.replace(c, miss=MISS.format(MX_COS[c.id])) for c in ATTN_CASES]


@pytest.mark.parametrize("case", MX_CASES, ids=lambda c: c.id)
def test_mxfp4_attention_matches_oracle(case):
    check_parity(case, "mxfp4")


@pytest.mark.parametrize("case", miss_params(MX_CASES))
def test_mxfp4_cosine_bar_where_the_scheme_misses_it(case):
    check_cosine_bar(case, "mxfp4")


@pytest.mark.parametrize("i", [0, 5, 7, 11], ids=lambda i: ATTN_CASES[i].id)
def test_nvfp4_is_more_accurate_than_mxfp4_on_the_gpu(i):
    """The pages' ordering, measured on the kernels' outputs: cosine to exact
    attention of NVFP4 above that of MXFP4 on the same input."""
    c_mx = run_case(MX_CASES[i], "mxfp4")["cos_gpu"]
    c_nv = run_case(ATTN_CASES[i], "nvfp4")["cos_gpu"]
    assert c_nv > c_mx, (c_nv, c_mx)


@pytest.mark.parametrize("B,H,N,d,causal,keep,empty", [
    (1, 2, 1000, 128, False, 0.5, (0, 1, 2)),
    (1, 2, 700, 64, True, 0.6, (0, 0, 4)),
])
def test_mxfp4_block_sparse_matches_oracle(B, H, N, d, causal, keep, empty):
    w = W.custom(B, H, N, d, causal=causal, seed=N + 3 * d)
    q, k, v = W.make_inputs(w, "cuda")
    nb = (N + 127) // 128
    m = np.random.default_rng(N + 2).random((B, H, nb, nb)) < keep
    b, h, i = empty
    m[b, h, i, :] = False
    mt = torch.from_numpy(m.astype(np.uint8)).cuda()
    out = sattn.fwd_sparse(q, k, v, mt, causal=causal, mode="mxfp4")
    ones = sattn.fwd_sparse(q, k, v, torch.ones_like(mt), causal=causal, mode="mxfp4")
    dense = sattn.fwd(q, k, v, causal=causal, mode="mxfp4")
    torch.cuda.synchronize()
    assert torch.equal(ones, dense)
    got = out.float().cpu().numpy().reshape(B * H, N, d)
    qf, kf, vf = (t.float().cpu().numpy() for t in (q, k, v))
    emu = A.attn_quant_emul_nvfp4(qf, kf, vf, causal=causal, block_mask=m, fmt="mxfp4")
    err = np.abs(got - emu)
    print(f"mxfp4 block-sparse {w.name} causal={causal}: max|err|={err.max():.3e} mean|err|={err.mean():.3e}")
    assert np.isfinite(got).all()
    assert err.max() <= 6e-2 and err.mean() <= 6e-3
    assert np.all(got[b * H + h, i * 128:(i + 1) * 128] == 0)
