"""The INT8 tensor-core product of the I8QK_F8PV mode, bit for bit.

S_int = q8 . k8^T is the one exact integer step of the attention (TurboDiffusion
explainer, section 1: QK^T in INT8).  sattn_debug_scores runs it the way the
attention kernel does (same TMA tensor maps and swizzle, same shared-memory and
instruction descriptors, tcgen05.mma kind::i8 into tensor memory) and exports
the int32 accumulator.  It must equal the exact integer product of the oracle's
own INT8 codes of the same inputs, element by element; rows and columns past N
(zero-filled tiles) must be 0.
"""

import numpy as np
import pytest
import torch

import bit_quantized_attention_smooth_b200 as sattn
from bit_quantized_attention_smooth_b200 import build as sattn_build
from oracle import attention as A
from oracle import quant as Qz
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


@pytest.mark.parametrize("w,q_per_token", [
    (W.custom(1, 2, 300, 128, seed=71, q_outlier_frac=1e-3), False),
    (W.custom(2, 1, 129, 64, "fp16", seed=72), False),
    (W.custom(1, 1, 1, 128, seed=73), False),
    (W.custom(1, 2, 256, 64, seed=74), True),
], ids=lambda x: getattr(x, "name", str(x)))
def test_int8_scores_bit_exact(w, q_per_token):
    q, k, v = W.make_inputs(w, "cuda")
    ws = sattn.quantize(q, k, v, q_per_token=q_per_token)
    s = sattn.debug_scores(ws, q.shape, dtype=q.dtype, q_per_token=q_per_token)
    torch.cuda.synchronize()
    got = s.cpu().numpy()
    N = w.N
    assert not np.any(got[:, :, N:, :]) and not np.any(got[:, :, :, N:])
    qf, kf, vf = (t.float().cpu().numpy() for t in (q, k, v))
    for b in range(w.B):
        for h in range(w.H):
            z = Qz.quantize_head_i8f8(qf[b, h], kf[b, h], vf[b, h], block_q=1 if q_per_token else 128)
            want = A.int8_scores(z["q"], z["k"])
            assert np.array_equal(got[b, h, :N, :N].astype(np.int64), want), (b, h)


def test_scores_accessor_rejects_fp4_modes():
    w = W.custom(1, 1, 128, 64, seed=75)
    q, k, v = W.make_inputs(w, "cuda")
    ws = sattn.quantize(q, k, v, mode="nvfp4")
    with pytest.raises(sattn.SattnError):
        sattn.debug_scores(ws, q.shape, mode="nvfp4", dtype=q.dtype)
