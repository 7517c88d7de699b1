"""Independent brute-force restatements used to pin the oracle (tiny inputs only).

Nothing here is shared with the oracle's C code: the E2M1 values come from the
bit format itself (1 sign, 2 exponent, 1 mantissa bit, exponent bias 1, a
subnormal at exponent 0), the rounding is a search over all 16 codes, and the
E8M0 exponent is a search over integers rather than a frexp.
"""
from __future__ import annotations

import math
from fractions import Fraction

import numpy as np


def e2m1_decode(code: int) -> float:
    s = (code >> 3) & 1
    e = (code >> 1) & 3
    m = code & 1
    mag = m * 0.5 if e == 0 else 2.0 ** (e - 1) * (1.0 + m / 2.0)
    return -mag if s else mag


def e2m1_nearest(u: float) -> int:
    """Nearest of the 16 codes whose sign bit matches u's sign; exact ties -> even mantissa bit."""
    neg = math.copysign(1.0, u) < 0
    best, bestd = None, None
    for c in range(16):
        if ((c >> 3) & 1) != int(neg):
            continue
        d = abs(abs(Fraction(u)) - abs(Fraction(e2m1_decode(c))))   # exact distance
        if best is None or d < bestd or (d == bestd and (c & 1) == 0 and (best & 1) == 1):
            best, bestd = c, d
    return best


def e8m0_search(amax: float) -> int:
    """Scale byte: the e with 4 <= amax * 2^-e < 8 (largest E2M1 binade), clamped to [-127, 127]."""
    if math.isnan(amax) or math.isinf(amax):
        return 0xFF
    if amax == 0.0:
        return 0
    a = Fraction(amax)
    e0 = a.numerator.bit_length() - a.denominator.bit_length() - 2   # within 1 of the answer
    for e in range(e0 - 3, e0 + 4):
        v = a / Fraction(2) ** e                       # exact
        if 4 <= v < 8:
            return min(127, max(-127, e)) + 127
    raise AssertionError("no exponent found")


def quantize_group(y) -> tuple[int, list[int]]:
    """Brute-force MXFP4 of one group of 32 values that are already fp32 numbers."""
    y = [float(v) for v in y]
    if any(math.isnan(v) or math.isinf(v) for v in y):
        return 0xFF, [0] * 32
    amax = max(abs(v) for v in y)
    byte = e8m0_search(amax)
    e = byte - 127
    return byte, [e2m1_nearest(math.ldexp(v, -e)) for v in y]


def pack(codes) -> np.ndarray:
    codes = np.asarray(codes, np.uint8).reshape(-1, 2)
    return (codes[:, 0] | (codes[:, 1] << 4)).astype(np.uint8)
