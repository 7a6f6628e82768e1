"""Pins for the oracle's number formats (no GPU).

The expected values below are written from the format definitions
(sign / exponent / mantissa fields and biases), not from the oracle.
"""

import numpy as np
import pytest
import torch

from oracle import formats as F


# --- E4M3 ---------------------------------------------------------------------

# (code, value) pairs derived by hand: value = 2^(e-7) * (1 + m/8), subnormal
# m/8 * 2^-6, bias 7, S.1111.111 = NaN.
E4M3_HAND = [
    (0x00, 0.0), (0x01, 2.0 ** -9), (0x07, 7 * 2.0 ** -9), (0x08, 2.0 ** -6),
    (0x09, 1.125 * 2.0 ** -6), (0x30, 0.5), (0x38, 1.0), (0x39, 1.125), (0x3F, 1.875),
    (0x40, 2.0), (0x48, 4.0), (0x70, 128.0), (0x76, 224.0), (0x77, 240.0), (0x78, 256.0),
    (0x7E, 448.0),
]


def test_e4m3_hand_values():
    tab = F.e4m3_table()
    for code, val in E4M3_HAND:
        assert tab[code] == val, hex(code)
        assert tab[code | 0x80] == -val, hex(code | 0x80)
    assert np.isnan(tab[0x7F]) and np.isnan(tab[0xFF])


def test_e4m3_table_structure():
    tab = F.e4m3_table()
    pos = tab[:127]
    assert np.all(np.diff(pos) > 0), "non-negative codes must be strictly increasing"
    assert np.sum(np.isfinite(tab)) == 254
    assert pos.max() == 448.0
    # spacing: 2^-9 in the subnormal range and the first normal binade
    assert np.allclose(np.diff(pos[:16]), 2.0 ** -9)


def _midpoints_and_neighbours():
    pos = F.e4m3_table()[:127]
    mids = (pos[:-1] + pos[1:]) / 2
    eps = np.spacing(mids.astype(np.float32)).astype(np.float64)
    pts = np.concatenate([pos, mids, mids + eps, mids - eps, [449, 460, 463.99, 464, 465, 1e4, 1e-4, 1e-30]])
    return np.concatenate([pts, -pts])


def test_e4m3_encoder_matches_bruteforce_on_all_midpoints():
    pts = _midpoints_and_neighbours()
    a = F.e4m3_encode(pts)
    b = F.e4m3_encode_bruteforce(pts)
    assert np.array_equal(a, b)


def test_e4m3_encoder_matches_bruteforce_random():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(4000) * np.exp2(rng.uniform(-12, 10, 4000))).astype(np.float32)
    assert np.array_equal(F.e4m3_encode(x), F.e4m3_encode_bruteforce(x))


def test_e4m3_ties_go_to_even():
    # 1.0 (0x38) and 1.125 (0x39): midpoint 1.0625 -> 0x38 (even)
    assert F.e4m3_encode(np.array([1.0625]))[0] == 0x38
    # 1.875 (0x3F) and 2.0 (0x40): midpoint 1.9375 -> 0x40 (even)
    assert F.e4m3_encode(np.array([1.9375]))[0] == 0x40
    # subnormal midpoint 1.5 * 2^-9 -> 2 * 2^-9 (0x02)
    assert F.e4m3_encode(np.array([1.5 * 2.0 ** -9]))[0] == 0x02
    # 0.5 * 2^-9 -> 0 (even)
    assert F.e4m3_encode(np.array([0.5 * 2.0 ** -9]))[0] == 0x00


def test_e4m3_saturates():
    x = np.array([448.0, 460.0, 464.0, 500.0, 1e9, -1e9])
    assert list(F.e4m3_decode(F.e4m3_encode(x))) == [448, 448, 448, 448, 448, -448]


def test_e4m3_matches_torch_cast_in_range():
    # torch's float8_e4m3fn cast is a library second opinion (RNE), in range only
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(20000) * np.exp2(rng.uniform(-10, 8, 20000))).astype(np.float32)
    x = np.clip(x, -448, 448)
    t = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = F.e4m3_encode(x)
    # torch may emit +0 where we keep the sign of a negative input that rounds to 0
    same = (ours == t) | (((ours & 0x7F) == 0) & ((t & 0x7F) == 0))
    assert same.all()


# --- E2M1 ---------------------------------------------------------------------

def test_e2m1_table_by_hand():
    # e=0: m*0.5; e>=1: (1 + m/2) * 2^(e-1), bias 1
    hand = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert list(F.e2m1_decode(np.arange(8))) == hand
    assert list(F.e2m1_decode(np.arange(8, 16))) == [-h for h in hand]


def test_e2m1_ties_and_saturation():
    x = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.5, 7.0, 100.0, -5.0, -0.25])
    want = [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, 6.0, 6.0, 6.0, -4.0, 0.0]
    got = F.e2m1_round(x)
    assert list(got) == want


def test_e2m1_encoder_matches_bruteforce():
    vals = F.E2M1_VALUES
    mids = (vals[:-1] + vals[1:]) / 2
    eps = 1e-6
    rng = np.random.default_rng(2)
    pts = np.concatenate([vals, mids, mids + eps, mids - eps, rng.uniform(-8, 8, 3000)])
    assert np.array_equal(F.e2m1_encode(pts), F.e2m1_encode_bruteforce(pts))


# --- INT8 ---------------------------------------------------------------------

def test_int8_roundtrip_bound_and_extremes():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((128, 64)).astype(np.float32) * 5
    amax = np.float32(np.abs(x).max())
    s = amax / np.float32(127)
    q = F.int8_quantize(x, s)
    assert np.abs(q).max() == 127
    err = np.abs(x.astype(np.float64) - np.float64(s) * q)
    # half a step, plus the float32 rounding of x / s (|x/s| <= 127)
    assert err.max() <= np.float64(s) * (0.5 + 127 * 2.0 ** -23)


def test_int8_rne_on_exact_halves():
    s = np.float32(1.0)
    x = np.array([0.5, 1.5, 2.5, -0.5, -2.5, 126.5, 127.4, 200.0], dtype=np.float32)
    assert list(F.int8_quantize(x, s)) == [0, 2, 2, 0, -2, 126, 127, 127]
