"""The tensor-core products S = Q K^T of the quantised operands.

S_int = q8 . k8^T is the one exact integer step of the attention (TurboDiffusion
explainer, section 1: QK^T in INT8).  sattn_debug_scores runs it the way the
attention kernel does (same TMA tensor maps and swizzle, same shared-memory and
instruction descriptors, tcgen05.mma kind::i8 into tensor memory) and exports
the int32 accumulator.  It must equal the exact integer product of the oracle's
own INT8 codes of the same inputs, element by element; rows and columns past N
(zero-filled tiles) must be 0.  The FP4 modes' block-scaled product is checked
against the float64 product of the oracle's dequantised operands.
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


@pytest.mark.parametrize("w,mode", [
    (W.custom(1, 2, 300, 128, seed=76, q_outlier_frac=1e-3), "nvfp4"),
    (W.custom(2, 1, 129, 64, "fp16", seed=77), "nvfp4"),
    (W.custom(1, 2, 300, 128, seed=78, q_outlier_frac=1e-3), "mxfp4"),
    (W.custom(1, 1, 200, 64, seed=79), "mxfp4"),
], ids=lambda x: getattr(x, "name", str(x)))
def test_fp4_scores_are_the_dequantised_product(w, mode):
    """The block-scaled MMA applies the scale factors where the oracle puts
    them: S equals the float64 product of the oracle's dequantised operands up
    to float32 accumulation (1e-5 of the sum of |terms|).  For MXFP4 this pins
    the E8M0 codes stored at both 16-value positions of each 32-value block."""
    q, k, v = W.make_inputs(w, "cuda")
    ws = sattn.quantize(q, k, v, mode=mode)
    s = sattn.debug_scores(ws, q.shape, mode=mode, dtype=q.dtype)
    torch.cuda.synchronize()
    got = s.cpu().numpy().astype(np.float64)
    N, d = w.N, w.d
    assert not np.any(got[:, :, N:, :]) and not np.any(got[:, :, :, N:])
    qf, kf, vf = (t.float().cpu().numpy() for t in (q, k, v))
    head = Qz.quantize_head_nvfp4 if mode == "nvfp4" else Qz.quantize_head_mxfp4
    blk = 16 if mode == "nvfp4" else 32
    for b in range(w.B):
        for h in range(w.H):
            z = head(qf[b, h], kf[b, h], vf[b, h])
            qv = Qz.nvfp4_dequant_rows(z["q"], z["q_sc"], block=blk)[:, :d]
            kv = Qz.nvfp4_dequant_rows(z["k"], z["k_sc"], block=blk)[:, :d]
            want = qv @ kv.T
            bound = np.abs(qv) @ np.abs(kv).T
            err = np.abs(got[b, h, :N, :N] - want)
            assert np.all(err <= 1e-5 * bound), (b, h, float((err / np.maximum(bound, 1e-300)).max()))
