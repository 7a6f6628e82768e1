"""8-bit attention backward (SageBwd), written out step by step.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Source: the SageAttention tag page (reportify.cn), SageAttention3 summary,
8-bit training bullets: per-block INT8 for Q, K, V and per-token P with no
quantisation overhead [17]; in the backward, dO V^T stays in FP16 and the other
four matrix products are quantised [18].  The pages give no formulas; the
readings:

* Forward (recomputed in the backward as well): S = s_q s_k (q8 . k8) * sm_scale
  with per-128-token-block INT8 Q and K (K smoothed by its channel mean, which
  leaves the softmax unchanged); P = softmax(S) row by row (exact, float64);
  O = sum over key blocks of (s_P[i] s_v[blk]) (p8 . v8), where V is INT8 per
  128-token block and P is INT8 per query row and key block with
  s_P = rowmax(P in the block) / 127 ("per-token": the scale of a row is known
  from its softmax, so it costs nothing).
* Backward, with D_i = sum_c dO_ic O_ic (O the 8-bit forward's output):
    dP  = dO V^T               in FP16: dO and V rounded to float16, products
                               and sums in float32 (the one product kept at
                               16 bits)
    dS  = P * (dP - D)
    dV  = P^T dO               INT8: P and dO per 128 x 128 block / 128-token block
    dQ  = dS K' * sm_scale     INT8: dS per 128 x 128 block, K' per 128-token block
    dK  = dS^T Q * sm_scale    INT8: dS per 128 x 128 block, Q per 128-token block
  The recomputed S = Q K^T is the fourth quantised product.  Every scale is
  constant along its product's contraction within a block pair, so it is
  applied after the integer block product.  Subtracting the K channel mean
  does not change dK: the rows of dS sum to zero, so the mean's gradient
  vanishes.
Float64 after the codes.  ``quantise=False`` replaces every quantiser by the
identity (and dP by float64), giving the exact backward.
"""

import numpy as np

from .quant import k_channel_mean, smooth_k, int8_block_scales
from .formats import int8_quantize

BLK = 128


def _q8_rows(x, blk=BLK):
    """Per-block INT8 over row blocks of ``blk`` (all columns): (codes float64, scale per row float64)."""
    x = np.asarray(x, dtype=np.float32)
    s = int8_block_scales(x, blk)
    rs = np.repeat(s, blk)[:x.shape[0]]
    return int8_quantize(x, rs[:, None]).astype(np.float64), rs.astype(np.float64)


def _q8_tile(x):
    """INT8 of one block with one scale: (codes float64, scale)."""
    x = np.asarray(x, dtype=np.float32)
    amax = float(np.max(np.abs(x))) if x.size else 0.0
    s = np.float32(1.0) if amax == 0 else np.float32(amax) / np.float32(127)
    return int8_quantize(x, s).astype(np.float64), float(s)


def _blocked_product(A, B, blk=BLK):
    """sum over contraction blocks of (qa . qb) * sa * sb with A [M, K], B [K, N]:
    A quantised per (row block, contraction block) tile, B per contraction
    block (all its columns)."""
    M, K = A.shape
    out = np.zeros((M, B.shape[1]))
    for k0 in range(0, K, blk):
        qb, sb = _q8_tile(B[k0:k0 + blk])
        for m0 in range(0, M, blk):
            qa, sa = _q8_tile(A[m0:m0 + blk, k0:k0 + blk])
            out[m0:m0 + blk] += (qa @ qb) * (sa * sb)
    return out


def attn_fwd_bwd_8bit(q, k, v, do, sm_scale=None, quantise=True):
    """One head, no mask.  q, k, v, do: [N, d] float32.  Returns (O, dQ, dK, dV), float64."""
    N, d = q.shape
    s = 1.0 / np.sqrt(d) if sm_scale is None else float(sm_scale)
    if quantise:
        kp = smooth_k(k, k_channel_mean(k))
    else:
        kp = k.astype(np.float64) - k.astype(np.float64).mean(axis=0)
    if quantise:
        q8, sq = _q8_rows(q)
        k8, sk = _q8_rows(kp)
        S = (q8 @ k8.T) * sq[:, None] * sk[None, :] * s
    else:
        S = (q.astype(np.float64) @ kp.astype(np.float64).T) * s
    P = np.exp(S - S.max(axis=1, keepdims=True))
    P /= P.sum(axis=1, keepdims=True)
    # forward P V: P per row and key block (per-token), V per 128-token block
    O = np.zeros((N, d))
    for j0 in range(0, N, BLK):
        Pt = P[:, j0:j0 + BLK]
        if quantise:
            r = Pt.max(axis=1)
            sp = np.where(r > 0, r / 127.0, 1.0)
            p8 = np.clip(np.rint(Pt / sp[:, None]), 0, 127)
            v8, sv = _q8_tile(v[j0:j0 + BLK])
            O += (p8 @ v8) * sp[:, None] * sv
        else:
            O += Pt @ v[j0:j0 + BLK].astype(np.float64)
    # backward
    Dr = np.sum(do.astype(np.float64) * O, axis=1)
    if quantise:
        dP = (do.astype(np.float16).astype(np.float32) @ v.astype(np.float16).astype(np.float32).T).astype(np.float64)
        dS = P * (dP - Dr[:, None])
        dV = _blocked_product(P.T, do.astype(np.float64))
        dQ = _blocked_product(dS, kp.astype(np.float64)) * s
        dK = _blocked_product(dS.T, q.astype(np.float64)) * s
    else:
        dP = do.astype(np.float64) @ v.astype(np.float64).T
        dS = P * (dP - Dr[:, None])
        dV = P.T @ do.astype(np.float64)
        dQ = dS @ kp.astype(np.float64) * s
        dK = dS.T @ q.astype(np.float64) * s
    return O, dQ, dK, dV
