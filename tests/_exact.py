"""Exact (rational) helpers for the oracle pins.

Nothing here is shared with the oracle or the CUDA library: the value grids
are built from the bit-field definitions of the formats, rounding is decided
by exact distance comparison with Python Fractions, and the Hadamard matrix
comes from scipy.
"""
from __future__ import annotations

import bisect
from fractions import Fraction

import numpy as np


def _grid(codes_and_values):
    pairs = sorted(codes_and_values, key=lambda cv: cv[1])
    return [c for c, _ in pairs], [v for _, v in pairs]


def e4m3_grid():
    """(codes, values) of the non-negative finite E4M3 codes, sorted by value.

    Bit fields: e = bits 6..3, m = bits 2..0; e == 0 is m * 2^-9, otherwise
    (1 + m/8) * 2^(e-7) = (8 + m) * 2^(e-10); e == 15, m == 7 is NaN.
    """
    out = []
    for code in range(0x7F):
        e, m = code >> 3, code & 7
        if e == 0:
            v = Fraction(m, 2 ** 9)
        else:
            v = Fraction(8 + m) * Fraction(2) ** (e - 10)
        out.append((code, v))
    return _grid(out)


def e2m1_grid():
    """(codes, values) of the non-negative E2M1 codes: e = bits 2..1 (bias 1), m = bit 0."""
    out = []
    for code in range(8):
        e, m = code >> 1, code & 1
        v = Fraction(m, 2) if e == 0 else Fraction(2 + m, 2) * Fraction(2) ** (e - 1)
        out.append((code, v))
    return _grid(out)


def nearest_code(x: Fraction, codes, values, sign_bit: int, negative: bool) -> int:
    """Round |x| to the nearest grid value, ties to the even code, saturating."""
    a = abs(x)
    if a >= values[-1]:
        c = codes[-1]
    else:
        i = bisect.bisect_left(values, a)
        if values[i] == a:
            c = codes[i]
        else:
            lo, hi = i - 1, i
            dlo, dhi = a - values[lo], values[hi] - a
            if dlo < dhi:
                c = codes[lo]
            elif dhi < dlo:
                c = codes[hi]
            else:
                c = codes[lo] if codes[lo] % 2 == 0 else codes[hi]
    return c | (sign_bit if negative else 0)


def near_midpoint(x: Fraction, values, rel: float = 2.0 ** -20) -> bool:
    """True when x lies within rel (relative) of a midpoint between grid values."""
    a = abs(x)
    if a == 0:
        return False
    i = bisect.bisect_left(values, a)
    for j in (i - 1, i):
        if 0 <= j < len(values) - 1:
            mid = (values[j] + values[j + 1]) / 2
            if abs(a - mid) <= Fraction(rel) * a:
                return True
    return False


def is_negative(v: float) -> bool:
    return bool(np.signbit(np.float32(v)))


def frac(v) -> Fraction:
    return Fraction(float(v))
