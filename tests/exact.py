"""Exact rational arithmetic helpers for pinning the oracle.

These do not call the oracle: a value is computed exactly with fractions and
then rounded once to binary32 (round to nearest, ties to even).
"""
from fractions import Fraction

import numpy as np


def f32_exact(x) -> Fraction:
    """The exact rational value of a finite binary32 number."""
    return Fraction(float(np.float32(x)))


def round_to_f32(x: Fraction) -> np.float32:
    """Round an exact rational to the nearest binary32 (ties to even); overflow -> inf."""
    if x == 0:
        return np.float32(0.0)
    sign = -1 if x < 0 else 1
    a = abs(x)
    # e = floor(log2 a)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    elif Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, -126)
    quantum = Fraction(2) ** (e - 23)
    q, r = divmod(a, quantum)
    q = int(q)
    if r > quantum / 2 or (r == quantum / 2 and q % 2 == 1):
        q += 1
    val = q * quantum
    if val >= Fraction(2) ** 128:
        return np.float32(sign * np.inf)
    return np.float32(sign * float(val))


def _neg(x) -> bool:
    return bool(np.signbit(np.float32(x)))


def rn_mul(a, b) -> np.float32:
    r = round_to_f32(f32_exact(a) * f32_exact(b))
    if r == 0:   # IEEE: the sign of a zero product is the xor of the operand signs
        return np.float32(-0.0) if _neg(a) != _neg(b) else np.float32(0.0)
    return r


def rn_add(a, b) -> np.float32:
    r = round_to_f32(f32_exact(a) + f32_exact(b))
    if r == 0:   # IEEE round-to-nearest: an exact zero sum is +0 unless both addends are -0
        return np.float32(-0.0) if (_neg(a) and _neg(b)) else np.float32(0.0)
    return r


def rn_div(a, b) -> np.float32:
    return round_to_f32(f32_exact(a) / f32_exact(b))


def rn_fma(a, b, c) -> np.float32:
    return round_to_f32(f32_exact(a) * f32_exact(b) + f32_exact(c))
