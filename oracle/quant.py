"""Quantisers of the attention scheme, written as plainly as possible.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

All arrays are per head: ``x`` has shape [N, d] (tokens x channels) and is the
float32 upcast of the stored bf16/fp16 tensor (exact).  Every step that the
device performs in float32 (mean, scale formula, division) is done here in
float32 with IEEE rounding, so that codes can be compared bit for bit.

Readings of the pages (which give no formulas):

* Smoothing ("outlier smoothing", TurboDiffusion explainer, wxsanhe.com post
  64219, section 1): K' = K - mean_over_tokens(K) per channel.  The mean is the
  exact float64 sum of the stored values divided by N in float64, rounded once
  to float32; the subtraction is one float32 operation.  Q is not smoothed.
* Per-block INT8 for Q and K (SageAttention tag page, reportify.cn,
  SageAttention3 summary, 8-bit bullet [17] "per-block INT8 for Q/K/V"): one
  float32 scale per block of 128 consecutive tokens of one head,
  s = max|x| / 127 (float32 division), q = RNE(x / s) clamped to +-127; an
  all-zero block has s = 1.
* FP8 V (explainer section 1, "PV in FP8"): one float32 scale per channel over
  all tokens of the head, s_v = max|V[:, c]| / 448; codes = E4M3(V / s_v);
  an all-zero channel has s_v = 1.
* NVFP4 (tag page, SageAttention3 summary, FP4 bullet [15]): blocks of 16
  consecutive values along the contraction axis, scale = E4M3(max|x| / 6)
  (float32 division, then E4M3 rounding), codes = E2M1(x / scale) with the
  division in float32; a block whose scale rounds to zero gets all-zero codes.
  No per-tensor second-level scale.
* NaN inputs (the pages say nothing): every maximum propagates NaN, so a NaN
  makes the scale it feeds NaN -- the rows of its Q block (or token), the K
  channel mean and with it every K scale of the head, or one V channel's
  scale -- and the outputs that use that scale are NaN.
"""

import numpy as np

from .formats import (e4m3_encode, e4m3_decode, e2m1_encode, e2m1_decode,
                      e8m0_decode, int8_quantize, mx_scale_code)

INT8_MAX = np.float32(127.0)
FP8_MAX = np.float32(448.0)
FP4_MAX = np.float32(6.0)


def k_channel_mean(k32):
    """Per-channel mean over tokens, float32.  k32: [N, d] float32."""
    n = k32.shape[0]
    s = np.sum(k32.astype(np.float64), axis=0)
    return (s / np.float64(n)).astype(np.float32)


def smooth_k(k32, mu32):
    """K' = K - mu, one float32 subtraction per element."""
    return (k32.astype(np.float32) - mu32[None, :].astype(np.float32)).astype(np.float32)


def int8_block_scales(x32, block):
    """Per token-block scales s = max|x|/127 (float32).  x32: [N, d]."""
    n = x32.shape[0]
    nblk = (n + block - 1) // block
    s = np.empty(nblk, dtype=np.float32)
    for b in range(nblk):
        amax = np.max(np.abs(x32[b * block:(b + 1) * block]))
        s[b] = np.float32(1.0) if amax == 0 else np.float32(amax) / INT8_MAX
    return s


def quant_int8_blocks(x32, block=128):
    """Per-block INT8 codes and scales.  Returns (q int8 [N, d], s float32 [nblk])."""
    s = int8_block_scales(x32, block)
    rows_scale = np.repeat(s, block)[:x32.shape[0]]
    q = int8_quantize(x32, rows_scale[:, None])
    return q, s


def quant_v_fp8(v32):
    """Per-channel FP8 E4M3 codes of V.  Returns (codes uint8 [N, d], s_v float32 [d])."""
    amax = np.max(np.abs(v32), axis=0).astype(np.float32)
    s_v = np.where(amax == 0, np.float32(1.0), amax / FP8_MAX).astype(np.float32)
    y = (v32.astype(np.float32) / s_v[None, :]).astype(np.float32)
    return e4m3_encode(y), s_v


def nvfp4_quant_rows(x32, block=16):
    """NVFP4 along the last axis: x32 [R, L] float32.

    Returns (codes uint8 [R, Lp] one E2M1 code per element, scale_codes uint8
    [R, Lp/16] E4M3, scales float32 [R, Lp/16] decoded), with Lp = L rounded
    up to a multiple of 16 and the padding treated as zeros.
    """
    x32 = np.asarray(x32, dtype=np.float32)
    r, L = x32.shape
    Lp = (L + block - 1) // block * block
    xp = np.zeros((r, Lp), dtype=np.float32)
    xp[:, :L] = x32
    xb = xp.reshape(r, Lp // block, block)
    amax = np.max(np.abs(xb), axis=2).astype(np.float32)
    sc_codes = e4m3_encode((amax / FP4_MAX).astype(np.float32))
    sc = e4m3_decode(sc_codes).astype(np.float32)
    safe = np.where(sc == 0, np.float32(1.0), sc).astype(np.float32)
    y = (xb / safe[:, :, None]).astype(np.float32)
    codes = e2m1_encode(y)
    codes = np.where(sc[:, :, None] == 0, np.uint8(0), codes).astype(np.uint8)
    return codes.reshape(r, Lp), sc_codes, sc


def mxfp4_quant_rows(x32, block=32):
    """MXFP4 along the last axis (the ablation of the tag page's FP4 bullet
    [15]): blocks of 32 values, scale = E8M0 2^(floor(log2 max|x|) - 2),
    codes = E2M1(x / scale) RNE satfinite (the division by a power of two is
    exact).  Returns (codes [R, Lp], scale codes [R, Lp/32], scales float64),
    Lp = L rounded up to 32, padding treated as zeros."""
    x32 = np.asarray(x32, dtype=np.float32)
    r, L = x32.shape
    Lp = (L + block - 1) // block * block
    xp = np.zeros((r, Lp), dtype=np.float32)
    xp[:, :L] = x32
    xb = xp.reshape(r, Lp // block, block).astype(np.float64)
    sc_codes = mx_scale_code(np.max(np.abs(xb), axis=2), 2)
    sc = e8m0_decode(sc_codes)
    codes = e2m1_encode(xb / sc[:, :, None])
    return codes.reshape(r, Lp), sc_codes, sc


def fp4_rows(x32, fmt):
    """Quantise-dequantise rows in an FP4 microscaling format ("nvfp4" or
    "mxfp4"); float64 [R, Lp]."""
    if fmt == "nvfp4":
        codes, _, sc = nvfp4_quant_rows(x32)
        return nvfp4_dequant_rows(codes, sc)
    if fmt == "mxfp4":
        codes, _, sc = mxfp4_quant_rows(x32)
        return nvfp4_dequant_rows(codes, sc, block=32)
    raise ValueError(fmt)


def nvfp4_dequant_rows(codes, scales, block=16):
    """Values of NVFP4 codes: e2m1(code) * scale, float64 [R, Lp]."""
    r, Lp = codes.shape
    vals = e2m1_decode(codes).reshape(r, Lp // block, block)
    return (vals * scales.astype(np.float64)[:, :, None]).reshape(r, Lp)


def quantize_head_i8f8(q32, k32, v32, block_q=128, block_kv=128):
    """All quantised operands of one head for the INT8-QK / FP8-PV mode."""
    mu = k_channel_mean(k32)
    kp = smooth_k(k32, mu)
    qi8, sq = quant_int8_blocks(q32, block_q)
    ki8, sk = quant_int8_blocks(kp, block_kv)
    v8, sv = quant_v_fp8(v32)
    return dict(mu=mu, q=qi8, sq=sq, k=ki8, sk=sk, v=v8, sv=sv)


def quantize_head_nvfp4(q32, k32, v32):
    """All quantised operands of one head for the NVFP4 mode.

    Q and K' are blocked along channels; V along tokens (the contraction axis
    of P V), so its codes are returned transposed, [d, Np].
    """
    mu = k_channel_mean(k32)
    kp = smooth_k(k32, mu)
    qc, qsc_codes, qsc = nvfp4_quant_rows(q32)
    kc, ksc_codes, ksc = nvfp4_quant_rows(kp)
    vc, vsc_codes, vsc = nvfp4_quant_rows(np.ascontiguousarray(v32.T))
    return dict(mu=mu, q=qc, q_sc=qsc, q_sc_codes=qsc_codes,
                k=kc, k_sc=ksc, k_sc_codes=ksc_codes,
                vt=vc, vt_sc=vsc, vt_sc_codes=vsc_codes)


def quantize_head_mxfp4(q32, k32, v32):
    """All quantised operands of one head for the MXFP4 ablation of the NVFP4
    mode (tag page, SageAttention3 summary, FP4 bullet [15]): the operands of
    ``quantize_head_nvfp4`` with blocks of 32 values and E8M0 scale codes
    (``mxfp4_quant_rows``); V blocked along tokens and returned transposed."""
    mu = k_channel_mean(k32)
    kp = smooth_k(k32, mu)
    qc, qsc_codes, qsc = mxfp4_quant_rows(q32)
    kc, ksc_codes, ksc = mxfp4_quant_rows(kp)
    vc, vsc_codes, vsc = mxfp4_quant_rows(np.ascontiguousarray(v32.T))
    return dict(mu=mu, q=qc, q_sc=qsc, q_sc_codes=qsc_codes,
                k=kc, k_sc=ksc, k_sc_codes=ksc_codes,
                vt=vc, vt_sc=vsc, vt_sc_codes=vsc_codes)
