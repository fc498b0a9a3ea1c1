"""OCP FP8 E4M3 (e4m3fn) codec, written from the format definition.

The K2 checkpoint stores expert weights as `fmt: e4m3` ("Kimi K2 · Down
projection", OpenModelAtlas, config.json quantization_config excerpt). The
format: 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits.
  exponent field 0      -> subnormal: (-1)^s * 2^-6 * m/8   (step 2^-9)
  exponent field 1..15  -> normal:    (-1)^s * 2^(e-7) * (1 + m/8)
  e=15, m=7             -> NaN (no infinities), so the largest finite is
                           2^8 * 1.75 = 448.
Encoding rounds to nearest, ties to even, and saturates finite values beyond
448 to +-448 (the "satfinite" reading; the pages state no rounding rule).
NaN encodes to 0x7F (sign kept).

Pinned by tests/test_oracle_e4m3.py: exhaustive decode of all 256 codes and
round-trip against torch.float8_e4m3fn, and encode against torch's cast for
in-range values.
"""
from __future__ import annotations

import math

import numpy as np

E4M3_MAX = 448.0


def decode_scalar(code: int) -> float:
    """Value of one e4m3 code (0..255)."""
    s = -1.0 if (code >> 7) & 1 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * (m / 8.0) * 2.0 ** -6
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


_DECODE_TABLE = np.array([decode_scalar(c) for c in range(256)], dtype=np.float64)


def decode(codes: np.ndarray) -> np.ndarray:
    """Vectorised decode of uint8 codes to float64 (a lookup in the table of
    decode_scalar's 256 values; the codes are widened to int32 indices first,
    which numpy gathers several times faster than uint8 ones)."""
    return np.take(_DECODE_TABLE, np.asarray(codes, dtype=np.uint8).astype(np.int32))


def _round_half_even(v: float) -> int:
    f = math.floor(v)
    r = v - f
    if r > 0.5:
        return f + 1
    if r < 0.5:
        return f
    return f + (f & 1)


def encode_scalar(v: float) -> int:
    """Nearest-even, saturating encode of one real value."""
    if math.isnan(v):
        return 0x7F
    sign = 0x80 if (v < 0 or (v == 0 and math.copysign(1.0, v) < 0)) else 0
    a = abs(v)
    if a >= E4M3_MAX:
        return sign | 0x7E
    if a < 2.0 ** -6:
        # subnormal grid, step 2^-9; a result of 8 steps is the smallest normal
        n = _round_half_even(a * 2.0 ** 9)
        if n == 8:
            return sign | 0x08
        return sign | n
    ex = math.floor(math.log2(a))
    # guard against log2 rounding at exact powers of two
    if 2.0 ** ex > a:
        ex -= 1
    elif 2.0 ** (ex + 1) <= a:
        ex += 1
    n = _round_half_even(a * 2.0 ** (3 - ex))  # in [8, 16]
    if n == 16:
        n = 8
        ex += 1
    e_field = ex + 7
    if e_field > 15 or (e_field == 15 and n - 8 == 7):
        return sign | 0x7E  # rounded past 448: saturate
    return sign | (e_field << 3) | (n - 8)


def encode(values: np.ndarray) -> np.ndarray:
    """Vectorised nearest-even, saturating encode; float64 in, uint8 codes out.

    Uses the same steps as encode_scalar: split |v| into exponent and a
    3-bit mantissa grid, round half to even on that grid, carry into the
    exponent, saturate at 448, subnormals on the 2^-9 grid.
    """
    v = np.asarray(values, dtype=np.float64)
    isnan = np.isnan(v)
    a = np.abs(np.where(isnan, 0.0, v))
    sign = np.where(np.signbit(v), 0x80, 0).astype(np.int64)
    out = np.zeros(v.shape, dtype=np.int64)

    sub = a < 2.0 ** -6
    n_sub = np.rint(np.minimum(a, 2.0 ** -6) * 2.0 ** 9)  # numpy rint rounds half to even
    out = np.where(sub, n_sub.astype(np.int64), out)  # n_sub == 8 -> 0x08 = smallest normal

    with np.errstate(divide="ignore", invalid="ignore"):
        m, ex = np.frexp(np.where(sub, 1.0, a))  # a = m * 2^ex, m in [0.5, 1)
    ex = ex - 1  # a = (2m) * 2^ex, 2m in [1, 2)
    a_n = np.minimum(a, 2.0 * E4M3_MAX)  # larger values saturate below anyway
    n = np.rint(a_n * np.ldexp(1.0, 3 - ex)).astype(np.int64)  # in [8, 16]
    carry = n == 16
    n = np.where(carry, 8, n)
    ex = np.where(carry, ex + 1, ex)
    e_field = ex + 7
    normal = (e_field << 3) | (n - 8)
    over = (e_field > 15) | ((e_field == 15) & (n - 8 == 7))
    normal = np.where(over, 0x7E, normal)
    out = np.where(sub, out, normal)
    out = np.where(a >= E4M3_MAX, 0x7E, out)
    out = out | sign
    out = np.where(isnan, 0x7F, out)
    return out.astype(np.uint8)
