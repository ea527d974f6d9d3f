"""OCP FP8 e4m3fn codec in plain numpy.  Test infrastructure (see oracle/__init__.py).

The pages name the format only as "FP8 e4m3" ([ZYFA-pt] TL;DR; [ZYFA-fr] "L'essentiel en
30 secondes").  Reading: the OCP 8-bit float "e4m3fn" variant -- 1 sign bit, 4 exponent
bits with bias 7, 3 mantissa bits, no infinities, S.1111.111 is NaN, largest finite
magnitude 448, subnormals m * 2^-9.
"""
import numpy as np

E4M3_MAX = 448.0


def e4m3_decode(codes):
    """Decode uint8 e4m3fn codes to float64 by the format definition."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    out = sign * mag
    return np.where((c & 0x7F) == 0x7F, np.nan, out)


# the 127 finite non-negative magnitudes, code 0 .. 126, strictly increasing
_TABLE = e4m3_decode(np.arange(127, dtype=np.uint8))


def e4m3_encode(x):
    """Round float32 values to e4m3fn codes: nearest value, ties to the even code,
    magnitudes beyond 448 saturate to 448 (the 'satfinite' reading), NaN -> 0x7F.

    The nearest neighbour is found directly from the table of representable values, so the
    rule can be read off the definition: no bit tricks.
    """
    x = np.asarray(x, dtype=np.float32)
    a = np.abs(x.astype(np.float64))
    lo = np.searchsorted(_TABLE, a, side="right") - 1          # _TABLE[lo] <= a
    lo = np.clip(lo, 0, 126)
    hi = np.minimum(lo + 1, 126)
    d_lo = a - _TABLE[lo]
    d_hi = _TABLE[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (lo % 2 == 1))
    code = np.where(pick_hi, hi, lo)
    code = np.where(a >= E4M3_MAX, 126, code)                   # saturate
    sign = np.signbit(x).astype(np.int64) << 7
    code = (code | sign).astype(np.uint8)
    return np.where(np.isnan(x), np.uint8(0x7F), code).astype(np.uint8)
