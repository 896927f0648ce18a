"""OCP OFP8 E4M3 ("FN" variant) decode and encode, written from the format
definition.  Test infrastructure only (see the package docstring).

Format: one byte ``s eeee mmm``, exponent bias 7.
  * e > 0:                value = (-1)^s * 2^(e-7) * (1 + m/8)
  * e = 0:                value = (-1)^s * 2^(-6)  * (m/8)      (subnormal)
  * e = 15 and m = 7:     NaN (codes 0x7F and 0xFF); there are no infinities.
Largest finite magnitude 448 (0x7E), smallest subnormal 2^-9 (0x01).

The pages name only "FP8" (Atlas deep-dive, ainews.cool, "Quantisation"
paragraph; GB10 page, ainews.surl.tw, "paged FP8 KV cache").  Readings taken
where they are silent (each listed in the design notes):
  * the quotient ``y = fp32(x) / fp32(scale)`` is an IEEE fp32 division,
    rounded to nearest (not a multiply by a reciprocal);
  * |y| >= 448 saturates to +-448 instead of producing NaN;
  * ties round to the code whose mantissa LSB is 0 (round-half-even);
  * the sign of a zero result is kept (-0 -> 0x80); NaN input -> 0x7F.
"""

import numpy as np

MAX_FINITE = 448.0
_SAT_CODE = 0x7E
_NAN_CODE = 0x7F


def decode(codes) -> np.ndarray:
    """Exact float64 value of each E4M3 code (uint8 array in, float64 out).

    Closed form of the format definition above, evaluated per element.
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    s = c >> 7
    e = (c >> 3) & 0xF
    m = c & 0x7
    sign = np.where(s == 1, -1.0, 1.0)
    normal = np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int32))
    subnormal = np.ldexp(m / 8.0, -6)
    mag = np.where(e > 0, normal, subnormal)
    val = sign * mag
    val = np.where((e == 15) & (m == 7), np.nan, val)
    return val


def quotient_f32(x, scale) -> np.ndarray:
    """``fp32(x) / fp32(scale)`` as one IEEE binary32 division (round to
    nearest even), broadcast over the arrays."""
    xf = np.asarray(x, dtype=np.float32)
    sf = np.asarray(scale, dtype=np.float32)
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        return np.divide(xf, sf, dtype=np.float32)


def encode_value(y) -> np.ndarray:
    """E4M3 code (uint8) of already-divided fp32 values ``y``.

    Route: split |y| into exponent and significand (frexp), round the
    significand to 3 fractional bits with round-half-even (np.rint), and let a
    mantissa carry move into the exponent by integer addition of the code.
    Subnormals are the same rounding on a fixed 2^-9 grid, which meets the
    normal range continuously (code 0x08 = 2^-6).
    """
    y = np.asarray(y, dtype=np.float32)
    a = np.abs(y).astype(np.float64)
    neg = np.signbit(y)
    codes = np.zeros(y.shape, dtype=np.int64)

    finite = np.isfinite(a)
    sat = finite & (a >= MAX_FINITE)
    small = finite & (a < 2.0 ** -6)
    normal = finite & ~sat & ~small

    # subnormal grid: value = k * 2^-9, k = 0..8 (k = 8 is the first normal)
    codes = np.where(small, np.rint(np.where(small, a, 0.0) * 2.0 ** 9).astype(np.int64), codes)

    # normal: a = f * 2^E with f in [0.5, 1) -> a = (1 + q/8) * 2^(E-1)
    f, E = np.frexp(np.where(normal, a, 1.0))
    q = (2.0 * f - 1.0) * 8.0
    m = np.rint(q).astype(np.int64)
    ncode = ((E.astype(np.int64) - 1 + 7) << 3) + m
    codes = np.where(normal, ncode, codes)

    codes = np.where(sat, _SAT_CODE, codes)
    codes = np.where(neg, codes | 0x80, codes)
    codes = np.where(np.isnan(y), _NAN_CODE, codes)
    # +-inf input saturates like any |y| >= 448
    codes = np.where(np.isinf(y), np.where(neg, 0x80 | _SAT_CODE, _SAT_CODE), codes)
    return codes.astype(np.uint8)


def encode(x, scale) -> np.ndarray:
    """Quantise ``x`` with ``scale``: ``encode_value(fp32(x) / fp32(scale))``."""
    return encode_value(quotient_f32(x, scale))


def row_scale(x) -> np.ndarray:
    """Dynamic per-row scale of the finer-grained reading (one scale per token
    and KV head): ``fp32(max |x|) / fp32(448)`` over the last axis, as one
    IEEE binary32 division; an all-zero row gets 1.0.  The Atlas deep-dive
    (ainews.cool, "Quantisation" paragraph) names per-group scale factors; a
    token's row of one head is the finest group."""
    a = np.max(np.abs(np.asarray(x, dtype=np.float32)), axis=-1)
    with np.errstate(divide="ignore", invalid="ignore"):
        s = np.divide(a, np.float32(MAX_FINITE), dtype=np.float32)
    return np.where(a > 0, s, np.float32(1.0)).astype(np.float32)


def encode_rows(x):
    """(codes, scales): each row (last axis) of ``x`` quantised with its own
    :func:`row_scale`."""
    s = row_scale(x)
    return encode(x, s[..., None]), s
