"""Host model of the quantize kernel's per-CTA threshold search, against brute force.

The fast quantize path needs, for each pair of neighbouring codebook entries a < b, the
smallest fp32 value T at which entry b is strictly nearer than entry a under the exact rule of
the k-bit patch series (kQuantizeBlockwise_kbit: fp32 distance fabsf(xn - c), first index on
ties), i.e. fl(b - T) < fl(T - a). The kernel finds T with 8 lanes per threshold: candidates
at the rounding boundaries of the two distances near (b - a) / 2, the smallest one where the
rule holds kept if the rule fails one fp32 value below it; otherwise a checked bracket around
the midpoint and 9-way splits of its ordered keys. This file restates that arithmetic on the
host (uint32 keys, fp32 subtractions, fp64 breakpoints, directed conversions) and checks that it
returns exactly the brute-force T (bisection over all fp32 keys with the rule itself) within
its step bound, for the codebooks the library uses and for adversarial pairs. No GPU is
involved.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from blockwise_bit_codebook_b200 import synthetic

NINTH = 477218588          # floor(2^32 / 9)
MASK = 0xFFFFFFFF


def f32(x) -> np.float32:
    return np.float32(x)


def okey(f) -> int:
    b = int(np.float32(f).view(np.uint32))
    m = (0xFFFFFFFF if b >> 31 else 0) | 0x80000000
    return b ^ m


def okey_f32(k: int) -> np.float32:
    k &= MASK
    m = (0xFFFFFFFF if not (k >> 31) else 0) | 0x80000000
    return np.uint32(k ^ m).view(np.float32)


def beats(a, b, v) -> bool:
    with np.errstate(over="ignore", invalid="ignore"):
        return bool(f32(b) - f32(v) < f32(v) - f32(a))


def d2f_rd(x: float) -> np.float32:
    f = np.float32(x)
    if float(f) > x:
        f = np.nextafter(f, np.float32(-np.inf))
    return f


def d2f_ru(x: float) -> np.float32:
    f = np.float32(x)
    if float(f) < x:
        f = np.nextafter(f, np.float32(np.inf))
    return f


def fsub_ru(b, a) -> np.float32:
    exact = Fraction(float(b)) - Fraction(float(a))
    f = np.float32(float(exact))          # within one rounding of exact; fix up to round upward
    while Fraction(float(f)) < exact:
        f = np.nextafter(f, np.float32(np.inf))
    while True:
        g = np.nextafter(f, np.float32(-np.inf))
        if Fraction(float(g)) >= exact:
            f = g
        else:
            break
    return f


def umulhi(x: int, y: int) -> int:
    return ((x & MASK) * (y & MASK)) >> 32


def model_threshold(a, b):
    """The kernel's group search for one threshold; returns (T, converged, search steps).

    One candidate round (each of 8 lanes takes one rounding boundary beta of the distances near
    (b - a) / 2 and tests the smallest fp32 at or above b - beta and a + beta and the next
    values); the smallest candidate where the rule holds is kept if the rule fails one fp32
    below it. Otherwise the bracket (m, m + ulp(b - a) / 2], checked at both ends, and 9-way
    splits of its ordered keys."""
    a, b = f32(a), f32(b)
    lo, hi = okey(a), okey(b)
    w = fsub_ru(b, a)
    uh = float(np.uint32(int(w.view(np.uint32)) & 0x7F800000).view(np.float32)) * 2.0 ** -24
    h = 0.5 * (float(b) - float(a))
    best_all = []
    for r in range(8):
        k0 = (okey(d2f_rd(h - uh)) - 1 + r) & MASK
        beta = 0.5 * (float(okey_f32(k0)) + float(okey_f32(k0 + 1)))
        c1 = okey(d2f_ru(float(b) - beta))
        c2 = okey(d2f_ru(float(a) + beta))
        best = hi
        for i in range(4):
            c = ((c2 if i & 2 else c1) + (i & 1)) & MASK
            if lo < c < best and beats(a, b, okey_f32(c)):
                best = c
        best_all.append(best)
    best = min(best_all)
    if best > lo and not beats(a, b, okey_f32(best - 1)) and beats(a, b, okey_f32(best)):
        return okey_f32(best), True, 0
    m = 0.5 * float(a) + 0.5 * float(b)
    lo1 = (okey(d2f_rd(m)) - 1) & MASK
    hi1 = (okey(d2f_ru(m + uh)) + 1) & MASK
    lo1, hi1 = max(lo1, lo), min(hi1, hi)
    if not beats(a, b, okey_f32(lo1)) and beats(a, b, okey_f32(hi1)) and lo1 < hi1:
        lo, hi = lo1, hi1
    steps = 0
    for _ in range(12):
        rng = (hi - lo) & MASK
        if rng <= 1:
            break
        steps += 1
        pts = [(lo + umulhi(rng, (r + 1) * NINTH)) & MASK for r in range(8)]
        p = [beats(a, b, okey_f32(x)) for x in pts]
        below = 8 - sum(p)
        nlo = (lo + umulhi(rng, below * NINTH)) & MASK
        nhi = hi if below == 8 else (lo + umulhi(rng, (below + 1) * NINTH)) & MASK
        lo, hi = nlo, nhi
    return okey_f32(hi), ((hi - lo) & MASK) <= 1, max(steps, 1)


def brute_threshold(a, b):
    """Smallest fp32 v in (a, b] with fl(b - v) < fl(v - a), by bisection over ordered keys."""
    a, b = f32(a), f32(b)
    lo, hi = okey(a), okey(b)
    assert not beats(a, b, a) and beats(a, b, b)
    while hi - lo > 1:
        mid = (lo + hi) // 2
        if beats(a, b, okey_f32(mid)):
            hi = mid
        else:
            lo = mid
    return okey_f32(hi)


def _check(pairs):
    worst = 0
    for a, b in pairs:
        if not f32(b) - f32(a) >= f32(2.0 ** -19):
            continue                  # not a pair the fast path accepts (e.g. -0 and +0)
        T, conv, steps = model_threshold(a, b)
        want = brute_threshold(a, b)
        assert conv, (a, b)
        assert T.view(np.uint32) == want.view(np.uint32), (float(a), float(b), float(T), float(want))
        worst = max(worst, steps)
    assert worst <= 11
    return worst


def _fallbacks(pairs):
    return sum(1 for a, b in pairs if f32(b) - f32(a) >= f32(2.0 ** -19) and model_threshold(a, b)[2] > 0)


def _neighbours(cb):
    cb = np.asarray(cb, np.float32)
    return list(zip(cb[:-1], cb[1:]))


@pytest.mark.parametrize("K", [2, 3, 4, 5])
def test_normal_float_codebooks(K):
    pairs = _neighbours(oracle.normal_float_codebook(K))
    _check(pairs)
    assert _fallbacks(pairs) == 0          # one candidate round settles every threshold


def test_stand_in_tables():
    fp4 = np.sort(synthetic.fp4_table())
    g8 = synthetic.general8_table()
    _check(_neighbours(fp4))
    _check(_neighbours(g8[::7]))          # a spread of the 256-entry table's neighbours
    _check(_neighbours(g8[100:140]))


def test_adversarial_pairs():
    rng = np.random.default_rng(11)
    pairs = []
    one = np.float32(1.0)
    for b in (np.float32(0.5), one, np.float32(0.3), np.float32(1e-3), np.float32(2.0 ** -19)):
        pairs.append((-b, b))                                     # symmetric: midpoint 0
        pairs.append((np.nextafter(-b, np.float32(0)), b))        # midpoint a hair above 0
        pairs.append((-b, np.nextafter(b, np.float32(0))))        # and below
        pairs.append((np.float32(0.0), b))                        # an entry at zero
        pairs.append((np.float32(-0.0), b))
    # midpoints on exact rounding boundaries of the distances
    for _ in range(200):
        a = np.float32(rng.uniform(-1, 1))
        e = np.float32(2.0 ** rng.integers(-20, 0))
        b = np.float32(a + e)
        if b > a:
            pairs.append((a, b))
            pairs.append((a, np.nextafter(b, np.float32(np.inf))))
    # tightest spacing the fast path accepts, at several magnitudes
    for c in (np.float32(0.9), np.float32(-0.37), np.float32(1e-4)):
        gap = np.float32(2.0 ** -19 * 2)
        pairs.append((c, np.float32(c + gap)))
    # random sorted codebooks of every size
    for K in (2, 3, 4, 5):
        for _ in range(4):
            cb = np.sort(rng.standard_normal(1 << K).astype(np.float32))
            cb /= np.abs(cb).max()
            pairs += _neighbours(np.unique(cb))
    # entries far apart in magnitude (fp64 breakpoints inexact): the check sends these to the search
    pairs += [(np.float32(1e-30), np.float32(0.5)), (np.float32(-0.5), np.float32(3e-33)),
              (np.float32(-1e-20), np.float32(2.0 ** -19))]
    _check(pairs)


def test_zero_crossing_settles_in_the_candidate_round():
    # near zero the bracket holds ~2^30 keys; the candidate round finds the threshold directly
    for b in (0.25, 0.3, 1.0, 2.0 ** -19):
        T, conv, steps = model_threshold(np.float32(-b), np.float32(b))
        assert conv and steps == 0
        assert T.view(np.uint32) == brute_threshold(np.float32(-b), np.float32(b)).view(np.uint32)


def test_fallback_search_alone_is_exact():
    # the key search that backs the candidate round, run from the full range
    rng = np.random.default_rng(5)
    for _ in range(300):
        a, b = np.sort(rng.uniform(-1, 1, 2).astype(np.float32))
        if not b - a >= 2.0 ** -19:
            continue
        lo, hi = okey(a), okey(b)
        for _ in range(12):
            r_ = (hi - lo) & MASK
            if r_ <= 1:
                break
            pts = [(lo + umulhi(r_, (r + 1) * NINTH)) & MASK for r in range(8)]
            below = 8 - sum(beats(a, b, okey_f32(x)) for x in pts)
            lo, hi = ((lo + umulhi(r_, below * NINTH)) & MASK,
                      hi if below == 8 else (lo + umulhi(r_, (below + 1) * NINTH)) & MASK)
        assert hi - lo <= 1
        assert okey_f32(hi).view(np.uint32) == brute_threshold(a, b).view(np.uint32)


def test_hint_check_accepts_only_the_threshold():
    # a cached threshold is kept only where the rule holds at it and fails one fp32 value below;
    # the rule being monotone, only the exact threshold passes (neighbours and other pairs' fail)
    rng = np.random.default_rng(3)
    cb = oracle.normal_float_codebook(5)
    Ts = [brute_threshold(a, b) for a, b in _neighbours(cb)]
    for j, (a, b) in enumerate(_neighbours(cb)):
        T = Ts[j]
        for d in range(-3, 4):
            h = okey_f32(okey(T) + d)
            keep = beats(a, b, h) and not beats(a, b, okey_f32(okey(h) - 1)) and okey(a) < okey(h) <= okey(b)
            assert keep == (d == 0)
        for other in rng.choice(len(Ts), 5):
            h = Ts[other]
            keep = beats(a, b, h) and not beats(a, b, okey_f32(okey(h) - 1)) and okey(a) < okey(h) <= okey(b)
            assert keep == (other == j)
