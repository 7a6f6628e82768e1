"""Attention: the exact definition and step-by-step emulations of both modes.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Inputs are float32 numpy arrays [B, H, N, d] (the exact upcast of the stored
bf16/fp16 tensors).  ``heads`` selects (b, h) pairs and ``rows`` selects query
rows, so that large workloads can be sampled; quantisation always runs over
the full token range of every selected head, as the device does.

The emulations follow the order of the method:

1. quantise (``quant.quantize_head_*``);
2. for each query row, sweep the keys in tiles of ``block_kv`` with an online
   softmax: reference max m, P~ = 2^(S - m), rescale factor
   alpha = 2^(m_old - m_new), l accumulated from the unquantised P~
   (FlashAttention-style streaming, which the TurboDiffusion explainer,
   wxsanhe.com post 64219, section 1, says the method replaces).  The pages do
   not say when the reference max moves.  ``tau`` = 0 is the exact running max
   (m is the row max of every key seen so far, so P~ <= 1); ``tau`` > 0 is the
   lazy policy: m moves to a tile's row max only when that max exceeds m by
   more than ``tau``, so that P~ <= 2^tau and the accumulators are rescaled
   only when the max has grown by more than that;
3. quantise P~ per tile and accumulate its product with the quantised V.

Scores are carried in the base-2 domain: S2 = S * sm_scale * log2(e).

Float64 is used after the codes (exact integer S for INT8, dequantised
products, accumulations).  The FP32 rounding order of the device's two-level
accumulator does not change these results beyond FP32 rounding, so the
accumulation period G does not appear here.
"""

import math

import numpy as np

from .formats import e4m3_round, e4m3_decode, int8_quantize  # noqa: F401
from .quant import quantize_head_i8f8, quantize_head_nvfp4, nvfp4_dequant_rows, nvfp4_quant_rows, fp4_rows

LOG2E = 1.0 / math.log(2.0)
P_SCALE_FP8 = 448.0           # static scale of P~ in [0, 1] onto E4M3's range
P_STAGE1_DIV = 448.0 * 6.0    # two-stage P: row max of the tile maps to 6 * 448


def default_scale(d, sm_scale):
    return 1.0 / math.sqrt(d) if (sm_scale is None or sm_scale <= 0) else float(sm_scale)


def _sel(B, H, N, heads, rows):
    if heads is None:
        heads = [(b, h) for b in range(B) for h in range(H)]
    rows = np.arange(N) if rows is None else np.asarray(rows, dtype=np.int64)
    return heads, rows


BLOCK = 128   # query and key block of the block-sparse mask


def _valid_mask(rows, cols, n, causal, blocks=None):
    """Key j is valid for query i iff j < N and (not causal or j <= i) and, with
    a block-sparse mask ``blocks`` [nblk, nblk] of one head, the 128 x 128 block
    (i // 128, j // 128) is kept (nonzero)."""
    m = np.broadcast_to(cols[None, :] < n, (len(rows), len(cols))).copy()
    if causal:
        m &= cols[None, :] <= rows[:, None]
    if blocks is not None:
        m &= np.asarray(blocks, dtype=bool)[rows // BLOCK][:, cols // BLOCK]
    return m


def _head_blocks(block_mask, b, h):
    return None if block_mask is None else block_mask[b, h]


def _safe_div(acc, l):
    """acc / l per row; a row with no valid key (every block of its query block
    skipped) has l = 0 and is defined as zeros."""
    l = np.asarray(l, dtype=np.float64)
    with np.errstate(invalid="ignore", divide="ignore"):
        out = acc / l[:, None]
    return np.where(l[:, None] == 0, 0.0, out)


def attn_exact(q, k, v, causal=False, sm_scale=None, heads=None, rows=None, block_mask=None):
    """O = softmax(Q K^T * sm_scale [masked]) V in float64.

    ``block_mask`` [B, H, nblk, nblk] (nblk = ceil(N / 128)), optional: keys of
    a skipped 128 x 128 block are left out of the softmax of that block's
    queries, as if masked (the "skip" part of Sparse-Linear Attention in the
    TurboDiffusion explainer, SLA section, with a given mask); a row whose
    query block skips every key block is zeros.
    Returns [len(heads), len(rows), d] float64.
    """
    B, H, N, d = q.shape
    s = default_scale(d, sm_scale)
    heads, rows = _sel(B, H, N, heads, rows)
    out = np.empty((len(heads), len(rows), d))
    cols = np.arange(N)
    for t, (b, h) in enumerate(heads):
        qh = q[b, h].astype(np.float64)[rows]
        S = (qh @ k[b, h].astype(np.float64).T) * s
        valid = _valid_mask(rows, cols, N, causal, _head_blocks(block_mask, b, h))
        S = np.where(valid, S, -np.inf)
        mx = S.max(axis=1, keepdims=True)
        P = np.exp(S - np.where(np.isneginf(mx), 0.0, mx))
        out[t] = _safe_div(P @ v[b, h].astype(np.float64), P.sum(axis=1))
    return out


def _online_softmax(S2, valid, tile, p_quant, pv, tau=0.0):
    """Generic streaming softmax over key tiles.

    S2: [R, N] float64 base-2 scores; valid: [R, N] bool.
    p_quant(P~ tile) -> (Pq tile, row factor) : quantised P and the factor that
        multiplies the tile's contribution (1 for static scales).
    pv(Pq, j0, j1) -> [R, d] product of the quantised P tile with V rows j0:j1.
    tau: the reference max of a row moves to the tile's row max only when that
        max exceeds it by more than tau (0: exact running max).
    Returns (acc [R, d], l [R]) with O = acc / l up to the V scale.
    """
    R, N = S2.shape
    m = np.full(R, -np.inf)
    l = np.zeros(R)
    acc = None
    for j0 in range(0, N, tile):
        j1 = min(j0 + tile, N)
        St = np.where(valid[:, j0:j1], S2[:, j0:j1], -np.inf)
        m_tile = St.max(axis=1)
        m_new = np.where(m_tile > m + tau, m_tile, m)
        m_use = np.where(np.isneginf(m_new), 0.0, m_new)
        P = np.exp2(St - m_use[:, None])                 # 0 where masked
        alpha = np.exp2(np.where(np.isneginf(m), -np.inf, m - m_use))
        l = alpha * l + P.sum(axis=1)
        Pq, fac = p_quant(P)
        contrib = pv(Pq, j0, j1) * fac[:, None]
        acc = contrib if acc is None else alpha[:, None] * acc + contrib
        m = m_new
    return acc, l


def attn_online_unquantised(q, k, v, causal=False, sm_scale=None, heads=None,
                            rows=None, block_kv=128, tau=0.0, block_mask=None):
    """The same tiled online softmax with every quantiser replaced by identity.

    Equal to ``attn_exact`` up to float64 rounding for any ``tau`` (the
    reference max cancels in acc / l); pins the streaming logic.
    """
    B, H, N, d = q.shape
    s = default_scale(d, sm_scale)
    heads, rows = _sel(B, H, N, heads, rows)
    out = np.empty((len(heads), len(rows), d))
    cols = np.arange(N)
    for t, (b, h) in enumerate(heads):
        vh = v[b, h].astype(np.float64)
        S2 = (q[b, h].astype(np.float64)[rows] @ k[b, h].astype(np.float64).T) * (s * LOG2E)
        acc, l = _online_softmax(
            S2, _valid_mask(rows, cols, N, causal, _head_blocks(block_mask, b, h)), block_kv,
            lambda P: (P, np.ones(P.shape[0])),
            lambda Pq, j0, j1: Pq @ vh[j0:j1], tau)
        out[t] = _safe_div(acc, l)
    return out


def int8_scores(qh, kh):
    """Exact integer S = q k^T of int8 codes.

    Computed as a float64 matrix product: every product and partial sum is an
    integer of magnitude <= 127 * 127 * d < 2^53, so the result is exact and
    independent of summation order.  Returned as int64.
    """
    return (qh.astype(np.float64) @ kh.astype(np.float64).T).astype(np.int64)


def attn_quant_emul_i8f8(q, k, v, causal=False, sm_scale=None, heads=None, rows=None,
                         block_q=128, block_kv=128, tau=0.0, block_mask=None):
    """INT8 QK^T / FP8 PV emulation (the I8QK_F8PV mode).

    Steps (TurboDiffusion explainer, section 1: QK in INT8, PV in FP8, outlier
    smoothing, two-level accumulation; tag page SageAttention3 summary [17]:
    per-block INT8 for Q/K):
      S2[i,j] = (q8_i . k8_j) * s_q[blk(i)] * s_k[blk(j)] * sm_scale * log2 e
      P~ tile = 2^(S2 - m);  p8 = E4M3(c_P * P~),  c_P = 448 * 2^-tau
      acc     = alpha * acc + p8 @ v8;  l = alpha * l + rowsum(P~)
      O       = acc * s_v[c] / (c_P * l)
    m is the reference max of the row (see ``tau`` in the module docstring):
    P~ <= 2^tau, so the static scale c_P maps the largest possible P~ onto
    E4M3's largest finite value, 448.  ``block_q`` = 1 gives one Q scale per
    token, the finest token granularity ("thread-level quantization", QbitAI
    reprint, txrjy.com, SageAttention paragraph, with one query row per
    softmax thread).
    """
    B, H, N, d = q.shape
    s = default_scale(d, sm_scale)
    heads, rows = _sel(B, H, N, heads, rows)
    out = np.empty((len(heads), len(rows), d))
    cols = np.arange(N)
    for t, (b, h) in enumerate(heads):
        z = quantize_head_i8f8(q[b, h], k[b, h], v[b, h], block_q, block_kv)
        v8 = e4m3_decode(z["v"])
        Sint = int8_scores(z["q"][rows], z["k"]).astype(np.float64)
        sq_rows = z["sq"][rows // block_q].astype(np.float64)
        sk_cols = z["sk"][cols // block_kv].astype(np.float64)
        S2 = Sint * sq_rows[:, None] * sk_cols[None, :] * (s * LOG2E)
        c_p = P_SCALE_FP8 * 2.0 ** -tau
        acc, l = _online_softmax(
            S2, _valid_mask(rows, cols, N, causal, _head_blocks(block_mask, b, h)), block_kv,
            lambda P: (e4m3_round(c_p * P), np.ones(P.shape[0])),
            lambda Pq, j0, j1: Pq @ v8[j0:j1], tau)
        out[t] = _safe_div(acc * z["sv"].astype(np.float64)[None, :] / c_p, l)
    return out


def attn_quant_emul_i8f8_smooth(q, k, v, causal=False, sm_scale=None, heads=None, rows=None,
                                block_q=128, block_kv=128, smooth_q=True, p_per_token=False):
    """The I8QK_F8PV scheme with the two variants of the SageAttention pages
    that the kernels do not implement (tag page, SageAttention3 summary,
    8-bit bullet [17]: per-token P; TurboDiffusion explainer, section 1:
    outlier smoothing, here applied to Q as well as K):

    * Q smoothing: qbar[b] = per-channel mean of Q over the tokens of query
      block b (float64 sum / block length, rounded to float32);
      Q' = Q - qbar (one float32 subtraction) is INT8-quantised per block, and
      the correction qbar[b] . K'_j, the same for every query of block b, is
      added to the scores in float64:
        S2[i,j] = (q8'_i . k8_j) s_q s_k * c  +  (qbar[blk(i)] . K'_j) * c
      With exact arithmetic Q' K'^T + qbar K'^T = Q K'^T, so the softmax is
      unchanged.
    * Per-token P: per row and key tile, P~ is scaled so its tile maximum maps
      to 448, p8 = E4M3(448 P~ / r), r = rowmax_tile(P~), and the tile's
      contribution is multiplied back by r / 448.
    Exact (running) reference max; everything after the codes in float64.
    """
    from .quant import k_channel_mean, smooth_k, quant_int8_blocks, quant_v_fp8
    B, H, N, d = q.shape
    s = default_scale(d, sm_scale)
    heads, rows = _sel(B, H, N, heads, rows)
    out = np.empty((len(heads), len(rows), d))
    cols = np.arange(N)
    for t, (b, h) in enumerate(heads):
        kp = smooth_k(k[b, h], k_channel_mean(k[b, h]))
        qh = q[b, h].astype(np.float32)
        qbar = np.zeros((N, d), dtype=np.float32)
        if smooth_q:
            for b0 in range(0, N, block_q):
                blk = qh[b0:b0 + block_q]
                qbar[b0:b0 + block_q] = (blk.astype(np.float64).sum(axis=0) / blk.shape[0]).astype(np.float32)[None, :]
        qs = (qh - qbar).astype(np.float32)
        q8, sq = quant_int8_blocks(qs, block_q)
        k8, sk = quant_int8_blocks(kp, block_kv)
        v8c, sv = quant_v_fp8(v[b, h])
        v8 = e4m3_decode(v8c)
        Sint = int8_scores(q8[rows], k8).astype(np.float64)
        S2 = Sint * sq[rows // block_q].astype(np.float64)[:, None] * sk[cols // block_kv].astype(np.float64)[None, :]
        S2 = (S2 + qbar[rows].astype(np.float64) @ kp.astype(np.float64).T) * (s * LOG2E)

        def pq(P):
            if not p_per_token:
                return e4m3_round(P_SCALE_FP8 * P), np.ones(P.shape[0])
            r = P.max(axis=1)
            r = np.where(r > 0, r, 1.0)
            return e4m3_round(P_SCALE_FP8 * P / r[:, None]), r

        acc, l = _online_softmax(S2, _valid_mask(rows, cols, N, causal), block_kv, pq,
                                 lambda Pq, j0, j1: Pq @ v8[j0:j1])
        out[t] = _safe_div(acc * sv.astype(np.float64)[None, :] / P_SCALE_FP8, l)
    return out


def two_stage_p_nvfp4(P, fmt="nvfp4"):
    """Two-stage quantisation of one P~ tile [R, T] (T <= 128 keys).

    Stage 1 (per row of the tile): s1 = rowmax(P~) / (448 * 6), s1 = 1 for an
    all-zero row; P2 = P~ / s1, so the row maximum lands on 6 * 448 and the
    second-stage E4M3 scales use their whole range.  Stage 2: NVFP4 blocks of
    16 keys on P2.  (Tag page, SageAttention3 summary, FP4 bullets [15][16]:
    two-stage quantisation fixes the narrow range of P's scale factors.)
    ``fmt`` = "mxfp4" swaps the second stage for MXFP4 (the ablation).
    Returns (dequantised P2 [R, T] float64, s1 [R] float64).
    """
    r = P.max(axis=1)
    s1 = np.where(r > 0, r / P_STAGE1_DIV, 1.0)
    P2 = (P / s1[:, None]).astype(np.float32)
    T = P.shape[1]
    return fp4_rows(P2, fmt)[:, :T], s1


def attn_quant_emul_nvfp4(q, k, v, causal=False, sm_scale=None, heads=None, rows=None,
                          block_kv=128, fmt="nvfp4", block_mask=None, smooth_q=False):
    """NVFP4 microscaled emulation (the NVFP4 mode).

      Q^, K'^ : NVFP4 along channels;  V^ : NVFP4 along tokens
      S2      = (Q^ K'^T) * sm_scale * log2 e          (block scales applied exactly)
      per key tile: P~ = 2^(S2 - m_running); (P2^, s1) = two_stage_p_nvfp4(P~)
      acc     = alpha * acc + s1 * (P2^ @ V^);  l = alpha * l + rowsum(P~)
      O       = acc / l
    ``fmt`` = "mxfp4" runs the same scheme with every FP4 operand in MXFP4
    (1 x 32 blocks, E8M0 scales): the ablation that the tag page's
    SageAttention3 summary, FP4 bullet [15], reports NVFP4 winning.
    ``smooth_q``: Q smoothing as in ``attn_quant_emul_i8f8_smooth`` (the block
    mean of Q is subtracted before the FP4 quantisation and qbar . K'_j is
    added back to the scores in float64).
    """
    B, H, N, d = q.shape
    s = default_scale(d, sm_scale)
    heads, rows = _sel(B, H, N, heads, rows)
    out = np.empty((len(heads), len(rows), d))
    cols = np.arange(N)
    for t, (b, h) in enumerate(heads):
        if fmt == "nvfp4":
            z = quantize_head_nvfp4(q[b, h], k[b, h], v[b, h])
            qv = nvfp4_dequant_rows(z["q"], z["q_sc"])[:, :d]
            kv = nvfp4_dequant_rows(z["k"], z["k_sc"])[:, :d]
            vv = nvfp4_dequant_rows(z["vt"], z["vt_sc"])[:, :N].T      # [N, d]
        else:
            from .quant import k_channel_mean, smooth_k
            kp = smooth_k(k[b, h], k_channel_mean(k[b, h]))
            qv = fp4_rows(q[b, h], fmt)[:, :d]
            kv = fp4_rows(kp, fmt)[:, :d]
            vv = fp4_rows(np.ascontiguousarray(v[b, h].T), fmt)[:, :N].T
        if smooth_q:
            from .quant import k_channel_mean, smooth_k
            qh = q[b, h].astype(np.float32)
            qbar = np.zeros_like(qh)
            for b0 in range(0, N, 128):
                blk = qh[b0:b0 + 128]
                qbar[b0:b0 + 128] = (blk.astype(np.float64).sum(axis=0) / blk.shape[0]).astype(np.float32)[None, :]
            qv = fp4_rows((qh - qbar).astype(np.float32), fmt)[:, :d]
            kp = smooth_k(k[b, h], k_channel_mean(k[b, h])).astype(np.float64)
            S2 = (qv[rows] @ kv.T + qbar[rows].astype(np.float64) @ kp.T) * (s * LOG2E)
        else:
            S2 = (qv[rows] @ kv.T) * (s * LOG2E)
        acc, l = _online_softmax(
            S2, _valid_mask(rows, cols, N, causal, _head_blocks(block_mask, b, h)), block_kv,
            lambda P: two_stage_p_nvfp4(P, fmt),
            lambda Pq, j0, j1: Pq @ vv[j0:j1])
        out[t] = _safe_div(acc, l)
    return out


def cosine(a, b):
    a = np.asarray(a, dtype=np.float64).ravel()
    b = np.asarray(b, dtype=np.float64).ravel()
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b)))
