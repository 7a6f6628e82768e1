"""Low-precision number formats used by the quantized attention scheme.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Formats
-------
* FP8 E4M3 ("fn" flavour, OCP 8-bit floating point): 1 sign, 4 exponent bits
  (bias 7), 3 mantissa bits, no infinities, NaN = S.1111.111, largest finite
  value 448, smallest normal 2^-6, subnormal spacing 2^-9.  The TurboDiffusion
  explainer (wxsanhe.com post 64219), section 1 "hybrid attention", states that
  P and V go through FP8 for the PV product.
* FP4 E2M1: 1 sign, 2 exponent bits (bias 1), 1 mantissa bit; the eight
  magnitudes are 0, 0.5, 1, 1.5, 2, 3, 4, 6.  Used with one unsigned E4M3 scale
  per 16 consecutive values (NVFP4 microscaling), which the SageAttention tag
  page (reportify.cn), SageAttention3 summary, FP4 bullet [15] names as the
  chosen format, and, for the ablation the same bullet compares it with, with
  one E8M0 power-of-two scale per 32 values (MXFP4, OCP Microscaling).

Rounding is round-to-nearest-even on the value, then saturation to the largest
finite magnitude ("satfinite"), which is the rounding the tensor-core
conversion instructions perform.  NaN maps to the NaN code (E4M3) and is not
defined for E2M1 (callers never pass it).

Two encoders are given for each format: an arithmetic one (binade, quantum,
``rint``) used by the attention emulation, and a brute-force nearest-value
search over the decoded code table, which the tests use to pin the arithmetic
encoder.
"""

import numpy as np

E4M3_MAX = 448.0
E2M1_MAX = 6.0


# ----------------------------------------------------------------------------
# FP8 E4M3
# ----------------------------------------------------------------------------

def e4m3_decode(codes):
    """Decode E4M3 codes (uint8 array) to float64 values; 0x7F/0xFF -> NaN."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    sub = m.astype(np.float64) / 8.0 * 2.0 ** -6
    nrm = (1.0 + m.astype(np.float64) / 8.0) * np.exp2(e.astype(np.float64) - 7.0)
    val = np.where(e == 0, sub, nrm)
    val = np.where((e == 15) & (m == 7), np.nan, val)
    return sign * val


def e4m3_table():
    """All 256 E4M3 code values, index = code."""
    return e4m3_decode(np.arange(256, dtype=np.uint8))


def e4m3_encode(x):
    """Round float values to E4M3 codes: round-to-nearest-even, saturate to +-448.

    The sign bit of the code is the sign bit of the input, so a negative value
    that rounds to zero gives the negative-zero code 0x80.
    """
    x = np.asarray(x, dtype=np.float64)
    neg = np.signbit(x)
    a = np.abs(x)
    nan = np.isnan(a)
    a = np.where(nan, 0.0, a)
    a = np.minimum(a, E4M3_MAX * 2.0)  # keeps frexp finite; saturated below
    # Binade exponent E with a = f * 2^E, f in [0.5, 1); the normal binade of a
    # is 2^(E-1).  Below 2^-6 the spacing is fixed at 2^-9 (subnormals).
    _, E = np.frexp(a)
    e_unb = np.maximum(E.astype(np.int64) - 1, -6)
    quantum = np.exp2((e_unb - 3).astype(np.float64))
    r = np.rint(a / quantum) * quantum           # exact: quantum is a power of 2
    r = np.minimum(r, E4M3_MAX)                  # satfinite
    # value -> bits
    _, Er = np.frexp(r)
    er = Er.astype(np.int64) - 1
    is_sub = r < 2.0 ** -6
    mant_sub = np.rint(r / 2.0 ** -9).astype(np.int64)
    exp_field = np.where(is_sub, 0, er + 7)
    mant_nrm = np.rint((r / np.exp2(er.astype(np.float64)) - 1.0) * 8.0).astype(np.int64)
    mant = np.where(is_sub, mant_sub, mant_nrm)
    code = (exp_field << 3) | mant
    code = np.where(nan, 0x7F, code)
    code = code | np.where(neg, 0x80, 0)
    return code.astype(np.uint8)


def e4m3_round(x):
    """Value of ``x`` after E4M3 rounding (float64)."""
    return e4m3_decode(e4m3_encode(x))


def e4m3_encode_bruteforce(x):
    """Reference encoder: nearest finite table value, ties to the even code.

    O(len(x) * 127); for tests on small arrays only.
    """
    x = np.asarray(x, dtype=np.float64).ravel()
    tab = e4m3_table()[:127]            # codes 0x00..0x7E, non-negative finite
    out = np.empty(x.shape, dtype=np.uint8)
    for i, xv in enumerate(x):
        if np.isnan(xv):
            out[i] = 0x7F
            continue
        a = abs(xv)
        dist = np.abs(tab - a)
        best = dist.min()
        cands = np.nonzero(dist == best)[0]
        if len(cands) > 1:
            cands = [c for c in cands if c % 2 == 0]
        code = int(cands[0])
        if np.signbit(xv):
            code |= 0x80
        out[i] = code
    return out


# ----------------------------------------------------------------------------
# FP4 E2M1
# ----------------------------------------------------------------------------

E2M1_VALUES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e2m1_decode(codes):
    """Decode 4-bit E2M1 codes (one per uint8, low nibble) to float64."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64) & 0xF
    sign = np.where(c & 0x8, -1.0, 1.0)
    e = (c >> 1) & 0x3
    m = c & 0x1
    val = np.where(e == 0, m * 0.5, (1.0 + m * 0.5) * np.exp2(e.astype(np.float64) - 1.0))
    return sign * val


def e2m1_encode(x):
    """Round float values to E2M1 codes: round-to-nearest-even, saturate to +-6."""
    x = np.asarray(x, dtype=np.float64)
    neg = np.signbit(x)
    a = np.minimum(np.abs(x), 2.0 * E2M1_MAX)
    _, E = np.frexp(a)
    e_unb = np.maximum(E.astype(np.int64) - 1, 0)   # below 1 the spacing is 0.5
    quantum = np.exp2((e_unb - 1).astype(np.float64))
    r = np.minimum(np.rint(a / quantum) * quantum, E2M1_MAX)
    # value -> code via the table (exact match guaranteed by construction)
    idx = np.searchsorted(E2M1_VALUES, r)
    code = idx.astype(np.int64) | np.where(neg, 0x8, 0)
    return code.astype(np.uint8)


def e2m1_round(x):
    return e2m1_decode(e2m1_encode(x))


def e2m1_encode_bruteforce(x):
    """Reference encoder for E2M1: nearest table value, ties to the even code."""
    x = np.asarray(x, dtype=np.float64).ravel()
    out = np.empty(x.shape, dtype=np.uint8)
    for i, xv in enumerate(x):
        a = abs(xv)
        dist = np.abs(E2M1_VALUES - a)
        best = dist.min()
        cands = [c for c in np.nonzero(dist == best)[0]]
        if len(cands) > 1:
            cands = [c for c in cands if c % 2 == 0]
        code = int(cands[0])
        if np.signbit(xv):
            code |= 0x8
        out[i] = code
    return out


# ----------------------------------------------------------------------------
# E8M0 (the shared scale of the OCP MX formats, used by the MXFP4 ablation)
# ----------------------------------------------------------------------------
# 8 exponent bits, no sign, no mantissa: code c is 2^(c - 127), c = 255 is NaN.

def e8m0_decode(codes):
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    return np.where(c == 255, np.nan, np.exp2((c - 127).astype(np.float64)))


def mx_scale_code(amax, emax_elem):
    """E8M0 code of the MX shared scale 2^(floor(log2 amax) - emax_elem).

    This is the OCP Microscaling rule: the block's largest magnitude lands in
    the element format's top binade (for E2M1, emax_elem = 2: [4, 8) before
    the elements saturate at 6).  amax = 0 gives the smallest code (the block
    is all zeros either way); NaN gives the NaN code.
    """
    a = np.asarray(amax, dtype=np.float64)
    nan = np.isnan(a)
    safe = np.where((a > 0) & ~nan, a, 1.0)
    _, E = np.frexp(safe)                     # safe = f * 2^E, f in [0.5, 1): floor(log2) = E - 1
    code = np.clip(E.astype(np.int64) - 1 - emax_elem + 127, 0, 254)
    code = np.where(a > 0, code, 0)
    return np.where(nan, 255, code).astype(np.uint8)


# ----------------------------------------------------------------------------
# INT8 with a float32 scale
# ----------------------------------------------------------------------------

def int8_quantize(x32, s32):
    """q = RNE(x / s) with the division in float32, clamped to [-127, 127].

    ``x32`` and ``s32`` are float32 arrays that broadcast together.  A NaN
    quotient (a NaN input or a NaN scale) gives code 0; its scale carries the
    NaN on to the scores.
    """
    x32 = np.asarray(x32, dtype=np.float32)
    s32 = np.asarray(s32, dtype=np.float32)
    with np.errstate(invalid="ignore"):
        y = (x32 / s32).astype(np.float32)      # IEEE float32 division
    y = np.where(np.isnan(y), np.float32(0), y)
    return np.clip(np.rint(y), -127, 127).astype(np.int8)
