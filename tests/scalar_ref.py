"""Scalar, loop-by-loop re-statement of both quantised attention schemes.

Used only to pin the vectorised oracle on tiny inputs (N <= 64): it shares
no code with ``oracle/attention.py`` or ``oracle/quant.py``.  It uses only the
decoded code tables of ``oracle.formats`` (pinned against hand-derived values
in ``test_oracle_formats.py``) and does its own nearest-value rounding.
"""

import math

import numpy as np

from oracle.formats import e4m3_table, E2M1_VALUES

F32 = np.float32
_E4M3_POS = [float(v) for v in e4m3_table()[:127]]
_E2M1_POS = [float(v) for v in E2M1_VALUES]


def _nearest_even(a, table):
    best_i, best_d = 0, None
    for i, t in enumerate(table):
        dd = abs(t - a)
        if best_d is None or dd < best_d or (dd == best_d and i % 2 == 0):
            best_i, best_d = i, dd
    return table[best_i]


def fp8(x):
    x = float(x)
    return math.copysign(_nearest_even(abs(x), _E4M3_POS), x)


def fp4(x):
    x = float(x)
    return math.copysign(_nearest_even(abs(x), _E2M1_POS), x)


def _kmean(K, N, d):
    mu = []
    for c in range(d):
        s = 0.0
        for n in range(N):
            s += float(K[n][c])
        mu.append(F32(s / N))
    return mu


def _i8(x, s):
    y = F32(F32(x) / s)
    r = round(float(y))                  # Python round() is half-to-even
    return max(-127, min(127, r))


def i8f8_head(Q, K, V, causal, sm_scale, blk=128, blk_q=None, tau=0.0):
    """One head, lists of float32 rows.  Returns list of output rows (floats).

    blk: token block of the K scales and the key tile; blk_q: token block of
    the Q scales (default blk); tau: the row's reference max moves to a tile's
    max only when that max is more than tau above it."""
    N, d = len(Q), len(Q[0])
    blk_q = blk if blk_q is None else blk_q
    mu = _kmean(K, N, d)
    Kp = [[F32(F32(K[n][c]) - mu[c]) for c in range(d)] for n in range(N)]

    def block_q8(X, blk):
        codes, scales = [], []
        for b0 in range(0, N, blk):
            amax = F32(0.0)
            for n in range(b0, min(b0 + blk, N)):
                for c in range(d):
                    amax = max(amax, abs(F32(X[n][c])))
            s = F32(1.0) if amax == 0 else F32(amax / F32(127.0))
            scales.append(s)
            for n in range(b0, min(b0 + blk, N)):
                codes.append([_i8(X[n][c], s) for c in range(d)])
        return codes, scales

    q8, sq = block_q8(Q, blk_q)
    k8, sk = block_q8(Kp, blk)
    sv = []
    for c in range(d):
        amax = F32(0.0)
        for n in range(N):
            amax = max(amax, abs(F32(V[n][c])))
        sv.append(F32(1.0) if amax == 0 else F32(amax / F32(448.0)))
    v8 = [[fp8(F32(F32(V[n][c]) / sv[c])) for c in range(d)] for n in range(N)]

    c2 = sm_scale / math.log(2.0)
    cp = 448.0 / 2.0 ** tau             # static FP8 scale of P: 2^tau -> 448
    out = []
    for i in range(N):
        m, l = -math.inf, 0.0
        acc = [0.0] * d
        for j0 in range(0, N, blk):
            j1 = min(j0 + blk, N)
            s2 = {}
            for j in range(j0, j1):
                if causal and j > i:
                    continue
                dot = sum(q8[i][c] * k8[j][c] for c in range(d))
                s2[j] = dot * float(sq[i // blk_q]) * float(sk[j // blk]) * c2
            if not s2:
                continue
            top = max(s2.values())
            m_new = top if (m == -math.inf or top - m > tau) else m
            alpha = 0.0 if m == -math.inf else 2.0 ** (m - m_new)
            l *= alpha
            acc = [a * alpha for a in acc]
            for j, sv2 in s2.items():
                p = 2.0 ** (sv2 - m_new)
                assert p <= 2.0 ** tau
                l += p
                p8 = fp8(cp * p)
                for c in range(d):
                    acc[c] += p8 * v8[j][c]
            m = m_new
        out.append([acc[c] * float(sv[c]) / (cp * l) for c in range(d)])
    return out


def _fp4_block(vals):
    """NVFP4 quantise-dequantise one block of up to 16 float32 values."""
    amax = F32(0.0)
    for x in vals:
        amax = max(amax, abs(F32(x)))
    sc = fp8(F32(amax / F32(6.0)))
    if sc == 0.0:
        return [0.0] * len(vals)
    scf = F32(sc)
    return [fp4(F32(F32(x) / scf)) * sc for x in vals]


def _fp4_rows(X, L):
    out = []
    for row in X:
        r = list(row) + [0.0] * ((-len(row)) % 16)
        deq = []
        for b0 in range(0, len(r), 16):
            deq.extend(_fp4_block(r[b0:b0 + 16]))
        out.append(deq[:L])
    return out


def nvfp4_head(Q, K, V, causal, sm_scale, blk=128):
    N, d = len(Q), len(Q[0])
    mu = _kmean(K, N, d)
    Kp = [[F32(F32(K[n][c]) - mu[c]) for c in range(d)] for n in range(N)]
    qh = _fp4_rows(Q, d)
    kh = _fp4_rows(Kp, d)
    vt = _fp4_rows([[V[n][c] for n in range(N)] for c in range(d)], N)   # [d][N]
    c2 = sm_scale / math.log(2.0)
    out = []
    for i in range(N):
        m, l = -math.inf, 0.0
        acc = [0.0] * d
        for j0 in range(0, N, blk):
            j1 = min(j0 + blk, N)
            s2 = []
            for j in range(j0, j1):
                if causal and j > i:
                    s2.append(-math.inf)
                else:
                    s2.append(sum(qh[i][c] * kh[j][c] for c in range(d)) * c2)
            if max(s2) == -math.inf:
                continue
            m_new = max(m, max(s2))
            alpha = 0.0 if m == -math.inf else 2.0 ** (m - m_new)
            p = [2.0 ** (x - m_new) if x != -math.inf else 0.0 for x in s2]
            l = l * alpha + sum(p)
            rmax = max(p)
            s1 = rmax / 2688.0 if rmax > 0 else 1.0
            p2 = _fp4_rows([[F32(x / s1) for x in p]], len(p))[0]
            for c in range(d):
                acc[c] = acc[c] * alpha + s1 * sum(p2[t] * vt[c][j0 + t] for t in range(len(p)))
            m = m_new
        out.append([a / l for a in acc])
    return out
