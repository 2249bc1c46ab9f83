"""Host model of the compression kernel's division, against the exact quotient.

The nested quantize scales each centred outer absmax c by the group's d = max(absmax2, 1e-8) with
an IEEE fp32 division (the reading of the pages' quantize rule). The kernel forms it without a
division instruction per value: y = RN(1/d) once per group, then q0 = RN(c y), r = fma(-d, q0, c)
(exact), q = fma(r, y, q0). By Markstein's theorem (y within half an ulp of 1/d, q0 within one ulp
of c/d, no underflow) q = RN(c/d); the kernel takes the IEEE division instead whenever
!(|q0| >= 2^-100) (zero, tiny, NaN). This file computes that sequence with exact rationals and
single roundings to fp32 and checks it against RN(c/d) on the compression's domain (|c| <= d,
d >= 1e-8) and on adversarial divisors. No GPU is involved.
"""
from fractions import Fraction

import numpy as np


def rn32(x: Fraction) -> np.float32:
    """Round a rational to the nearest fp32 (ties to even), no overflow handling needed here."""
    f = np.float32(float(x))                       # float(x) is RN to binary64; fix up to RN fp32
    for cand in (np.nextafter(f, np.float32(-np.inf)), np.nextafter(f, np.float32(np.inf))):
        if abs(Fraction(float(cand)) - x) < abs(Fraction(float(f)) - x):
            f = cand
    # ties: even significand
    lo = np.nextafter(f, np.float32(-np.inf))
    hi = np.nextafter(f, np.float32(np.inf))
    for cand in (lo, hi):
        if abs(Fraction(float(cand)) - x) == abs(Fraction(float(f)) - x) and int(cand.view(np.uint32)) % 2 == 0:
            f = cand
    return np.float32(f)


def markstein(c: np.float32, d: np.float32):
    if not np.isfinite(c):
        return None                                # q0 is NaN or infinite: the guard fails
    C, D = Fraction(float(c)), Fraction(float(d))
    y = rn32(1 / D)
    q0 = rn32(C * Fraction(float(y)))
    if not abs(float(q0)) >= 2.0 ** -100:
        return None                                # the kernel divides instead
    r = rn32(C - D * Fraction(float(q0)))          # one rounding (fma)
    return rn32(Fraction(float(r)) * Fraction(float(y)) + Fraction(float(q0)))


def check(pairs):
    used = 0
    for c, d in pairs:
        q = markstein(np.float32(c), np.float32(d))
        if q is None:
            continue
        used += 1
        want = rn32(Fraction(float(np.float32(c))) / Fraction(float(np.float32(d))))
        assert q.view(np.uint32) == want.view(np.uint32), (float(c), float(d), float(q), float(want))
    return used


def test_compression_domain():
    rng = np.random.default_rng(1)
    pairs = []
    for _ in range(3000):
        d = np.float32(10.0 ** rng.uniform(-8, 2))
        c = np.float32(rng.uniform(-1, 1) * d)
        pairs.append((c, d))
    assert check(pairs) > 2900


def test_adversarial_divisors_and_numerators():
    rng = np.random.default_rng(2)
    pairs = []
    # divisors just around powers of two and with long significands; numerators at +-d and at
    # quotients that land near rounding boundaries of fp32
    for e in range(-26, 8):
        for dm in (1.0, np.nextafter(np.float32(1.0), np.float32(2.0)), np.nextafter(np.float32(2.0), np.float32(1.0)),
                   np.float32(1.5), np.float32(1.9999999)):
            d = np.float32(np.float32(dm) * np.float32(2.0 ** e))
            if not d >= 1e-8:
                continue
            for _ in range(12):
                q = np.float32(rng.uniform(-1, 1))
                half = np.float32(q) + np.float32(2.0 ** -25) * np.sign(q)   # a quotient near a midpoint
                for target in (q, half):
                    c = np.float32(np.float32(target) * d)
                    pairs.append((c, d))
                    pairs.append((np.nextafter(c, np.float32(np.inf)), d))
            pairs.append((d, d))
            pairs.append((-d, d))
    assert check(pairs) > 1000


def test_the_guard_takes_zero_and_tiny_quotients():
    assert markstein(np.float32(0.0), np.float32(0.5)) is None
    assert markstein(np.float32(1e-40), np.float32(1.0)) is None      # subnormal numerator
    assert markstein(np.float32(np.nan), np.float32(1.0)) is None
