"""Pins for the oracle's E4M3 codec (CPU only).

The codec is checked against things other than itself: hand-computed anchor
values of the OCP E4M3 definition, torch's own float8_e4m3fn conversion
(a library routine), and a brute-force nearest-value search over the 254
finite codes that shares no step with the oracle's frexp/rint route.
"""

import numpy as np
import pytest
import torch

from oracle import e4m3

ALL = np.arange(256, dtype=np.uint8)
FINITE_POS = np.arange(0x7F, dtype=np.uint8)          # 0x00 .. 0x7E


# --- decode -----------------------------------------------------------------

@pytest.mark.parametrize("code,value", [
    (0x00, 0.0), (0x01, 2.0 ** -9), (0x02, 2.0 ** -8), (0x07, 7 * 2.0 ** -9),
    (0x08, 2.0 ** -6), (0x0F, 1.875 * 2.0 ** -6), (0x30, 0.5), (0x38, 1.0),
    (0x3C, 1.5), (0x40, 2.0), (0x77, 240.0), (0x78, 256.0), (0x7E, 448.0),
    (0x81, -(2.0 ** -9)), (0xB8, -1.0), (0xFE, -448.0),
])
def test_decode_anchors(code, value):
    assert e4m3.decode(np.uint8(code)) == value


def test_decode_signed_zero_and_nan():
    z = e4m3.decode(np.uint8(0x80))
    assert z == 0.0 and np.signbit(z)
    assert np.isnan(e4m3.decode(np.uint8(0x7F)))
    assert np.isnan(e4m3.decode(np.uint8(0xFF)))
    assert np.isnan(e4m3.decode(ALL)).sum() == 2


def test_decode_matches_torch_float8_all_codes():
    ours = e4m3.decode(ALL)
    ref = torch.from_numpy(ALL.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    both_nan = np.isnan(ours) & np.isnan(ref)
    assert np.array_equal(ours[~both_nan], ref[~both_nan])
    assert np.array_equal(np.signbit(ours[~both_nan]), np.signbit(ref[~both_nan]))


def test_decode_positive_codes_strictly_increase_and_negatives_mirror():
    pos = e4m3.decode(FINITE_POS)
    assert np.all(np.diff(pos) > 0)
    assert np.array_equal(e4m3.decode(FINITE_POS | 0x80), -pos)


# --- encode -----------------------------------------------------------------

def brute_force_encode(y):
    """Nearest finite code by exhaustive search; ties to the even code;
    |y| >= 448 saturates; sign kept."""
    y = np.asarray(y, dtype=np.float64)
    table = e4m3.decode(FINITE_POS)                    # 127 non-negative values
    a = np.abs(y)
    dist = np.abs(table[None, :] - a[:, None])
    best = dist.min(axis=1, keepdims=True)
    cand = dist == best
    even = cand & ((FINITE_POS[None, :] & 1) == 0)
    pick = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))
    code = FINITE_POS[pick].astype(np.int64)
    code = np.where(a >= 448.0, 0x7E, code)
    code = np.where(np.signbit(y), code | 0x80, code)
    return code.astype(np.uint8)


def test_encode_every_finite_code_value_roundtrips():
    codes = np.concatenate([FINITE_POS, FINITE_POS | 0x80])
    vals = e4m3.decode(codes).astype(np.float32)
    assert np.array_equal(e4m3.encode_value(vals), codes)


def test_encode_midpoints_tie_to_even_and_neighbours():
    table = e4m3.decode(FINITE_POS)
    lo, hi = table[:-1], table[1:]
    mid = (lo + hi) / 2                                   # exact in fp32 (dyadic)
    assert np.array_equal(mid.astype(np.float32).astype(np.float64), mid)
    got = e4m3.encode_value(mid.astype(np.float32))
    c_lo, c_hi = FINITE_POS[:-1], FINITE_POS[1:]
    want = np.where(c_lo % 2 == 0, c_lo, c_hi)
    assert np.array_equal(got, want)
    # one fp32 ulp either side of the midpoint decides the direction
    up = np.nextafter(mid.astype(np.float32), np.float32(np.inf))
    dn = np.nextafter(mid.astype(np.float32), np.float32(-np.inf))
    assert np.array_equal(e4m3.encode_value(up), c_hi)
    assert np.array_equal(e4m3.encode_value(dn), c_lo)
    assert np.array_equal(e4m3.encode_value(-mid.astype(np.float32)), want | 0x80)


@pytest.mark.parametrize("y,code", [
    (448.0, 0x7E), (449.0, 0x7E), (463.99, 0x7E), (464.0, 0x7E), (480.0, 0x7E),
    (1e6, 0x7E), (np.inf, 0x7E), (-448.0, 0xFE), (-1e6, 0xFE), (-np.inf, 0xFE),
    (447.9, 0x7E), (432.0, 0x7E), (431.9, 0x7D), (416.0, 0x7D), (-0.0, 0x80), (0.0, 0x00),
    (2.0 ** -10, 0x00), (-(2.0 ** -10), 0x80), (1.5 * 2.0 ** -10, 0x01),
    (1e-30, 0x00), (-1e-30, 0x80), (1e-45, 0x00), (np.nan, 0x7F),
])
def test_encode_special_values(y, code):
    assert int(e4m3.encode_value(np.float32(y))) == code


def test_encode_matches_brute_force_on_random_values():
    rng = np.random.default_rng(1234)
    n = 200_000
    mags = np.exp(rng.uniform(np.log(1e-4), np.log(600.0), n))
    y = (mags * rng.choice([-1.0, 1.0], n)).astype(np.float32)
    assert np.array_equal(e4m3.encode_value(y), brute_force_encode(y))


def test_encode_matches_torch_below_saturation():
    rng = np.random.default_rng(99)
    y = (rng.standard_normal(1_000_000) * 60).astype(np.float32)
    y = y[np.abs(y) < 448.0]
    ref = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(e4m3.encode_value(y), ref)


def test_encode_divides_in_fp32():
    # scale 0.1f is not a power of two: the fp32 quotient is what is coded
    x = np.float32(0.7)
    s = np.float32(0.1)
    y = np.float32(x) / np.float32(s)
    assert int(e4m3.encode(x, s)) == int(brute_force_encode(np.array([y]))[0])
    # dequantising gives back the code's value times the scale
    x = np.float32(3.25) * np.float32(0.125)
    assert e4m3.decode(e4m3.encode(x, np.float32(0.125))) == 3.25


# (x, scale) bit patterns whose fp32 quotient sits next to an E4M3 rounding
# midpoint, so that the division reading and a multiply-by-reciprocal reading
# give different codes.  Found by a seeded search over midpoints.
DIVISION_CASES = [(1024306369, 994385121), (979265552, 1027295785),
                  (1046172938, 1021470797), (1082060011, 1026643687)]


def _fp32_round_exact(fr):
    """Nearest binary32 to the rational ``fr`` (ties to even mantissa)."""
    from fractions import Fraction
    approx = np.float32(float(fr))
    cands = [approx, np.nextafter(approx, np.float32(np.inf)),
             np.nextafter(approx, np.float32(-np.inf))]
    dist = [abs(Fraction(float(c)) - fr) for c in cands]
    best = min(dist)
    tied = [c for c, d in zip(cands, dist) if d == best]
    tied.sort(key=lambda c: int(np.float32(c).view(np.uint32)) & 1)
    return tied[0]


@pytest.mark.parametrize("xb,sb", DIVISION_CASES)
def test_encode_uses_ieee_division_not_reciprocal(xb, sb):
    from fractions import Fraction
    x = np.uint32(xb).view(np.float32)
    s = np.uint32(sb).view(np.float32)
    y = _fp32_round_exact(Fraction(float(x)) / Fraction(float(s)))
    want = int(brute_force_encode(np.array([y]))[0])
    assert int(e4m3.encode(x, s)) == want
    recip = np.float32(x) * (np.float32(1.0) / np.float32(s))
    assert int(brute_force_encode(np.array([recip]))[0]) != want
