"""Host model of the General8 compression kernel's bucket search (nested quantize), checked
against brute force without a GPU.

The kernel finds p, the last table index with t_p <= xn, from a table over 64 buckets per binade
of |xn| (2^-24 to 1, both signs; 3074 buckets) and a short forward scan. This model restates
that index arithmetic (bucket of a value, first bucket at or above a value, the table built from
a histogram and a prefix sum, base | count << 9 entries) and checks, for ascending tables of
several shapes, that every bucket index is in range, that each entry holds what its definition
says, that the scan from a bucket's base never needs more steps than the bucket's count, and
that the p found equals the brute-force count of entries <= xn.
"""
import numpy as np
import pytest

SHIFT = 17
E0 = (127 - 24) << (23 - SHIFT)
HALF = 24 << (23 - SHIFT)
NBUCKETS = 2 * HALF + 2


def bits(x):
    return np.asarray(x, np.float32).view(np.uint32).astype(np.int64)


def bucket(xn):
    """Bucket of values with |xn| <= 1."""
    b = bits(xn)
    k = np.clip(((b & 0x7FFFFFFF) >> SHIFT) - E0, 0, HALF)
    return np.where(b >> 31, HALF - k, HALF + 1 + k)


def first_at_or_above(x):
    """First bucket whose lower point is >= x (NBUCKETS if none)."""
    x = np.asarray(x, np.float32)
    b = bits(x)
    k = ((b & 0x7FFFFFFF) >> SHIFT) - E0
    neg = np.maximum(HALF + 1 - np.maximum(k, 0), 0)
    edge = ((b & ((1 << SHIFT) - 1)) == 0) & (k >= 1)
    pos = np.minimum(HALF + 1 + np.maximum(np.where(edge, k, k + 1), 1), NBUCKETS)
    out = np.where(b >> 31, neg, np.where(b == 0, HALF + 1, pos))
    return np.where(np.isnan(x), NBUCKETS, out)


def lower_points():
    j = np.arange(NBUCKETS)
    mag = lambda k: (((k + E0) << SHIFT).astype(np.uint32)).view(np.float32)  # noqa: E731
    neg = -mag(np.clip(HALF - j + 1, 0, None))
    pos = np.where(j == HALF + 1, np.float32(0), mag(np.clip(j - HALF - 1, 0, None)))
    return np.where(j <= HALF, neg, pos).astype(np.float32)


def build_table(t):
    hist = np.bincount(first_at_or_above(t), minlength=NBUCKETS + 1)
    s = np.cumsum(hist)
    return s[:NBUCKETS] | (np.minimum(hist[1:], 127) << 9)


def tables():
    rng = np.random.default_rng(3)
    i = np.arange(256)
    yield "cubes", (((i - 127.5) / 127.5) ** 3).astype(np.float32)
    yield "uniform", np.sort(rng.uniform(-1, 1, 256)).astype(np.float32)
    yield "duplicates", np.sort(np.concatenate([rng.uniform(-1, 1, 200), np.zeros(20), np.full(36, 0.5)]))
    yield "tiny", np.sort(rng.standard_normal(256) * 1e-5)
    yield "cluster", np.sort(np.concatenate([np.linspace(0.5, 0.5001, 200), rng.uniform(-1, 1, 56)]))
    yield "infinite_ends", np.sort(np.concatenate([[-np.inf], rng.uniform(-1, 1, 254), [np.inf]]))


@pytest.mark.parametrize("name,t", list(tables()))
def test_bucket_search_matches_brute_force(name, t):
    t = np.asarray(t, np.float32)
    assert np.all(t[:-1] <= t[1:])
    lp = lower_points()
    assert np.all(np.diff(lp) > 0), "lower points ascend"
    # first_at_or_above agrees with a search over the lower points
    probes = np.concatenate([t, lp, np.nextafter(lp, np.float32(-2)), np.nextafter(lp, np.float32(2)),
                             np.array([0.0, -0.0, 1e-45, -1e-45, 3.0, -3.0], np.float32)]).astype(np.float32)
    assert np.array_equal(first_at_or_above(probes), np.searchsorted(lp, probes, side="left"))
    lut = build_table(t)
    base, count = lut & 511, lut >> 9
    # each entry: entries at or below the bucket's lower point, and those inside the bucket
    nxt = np.append(lp[1:], np.float32(np.inf))
    assert np.array_equal(base, np.searchsorted(t, lp, side="right"))
    inside = np.searchsorted(t, nxt, side="right") - base
    inside[-1] = np.sum(t > lp[-1])
    assert np.array_equal(count, np.minimum(inside, 127))
    # the search: base - 1, then forward while the next entry is <= xn
    rng = np.random.default_rng(11)
    xs = np.concatenate([rng.uniform(-1, 1, 4000), rng.uniform(-1, 1, 1000) * 1e-6, t,
                         np.nextafter(t, np.float32(2)), np.nextafter(t, np.float32(-2)), lp,
                         np.nextafter(lp, np.float32(-2))]).astype(np.float32)
    xs = xs[np.abs(xs) <= 1]
    j = bucket(xs)
    assert j.min() >= 0 and j.max() < NBUCKETS
    assert np.all(lp[j] <= xs), "a value lies at or above its bucket's lower point"
    p = base[j] - 1
    steps = np.searchsorted(t, xs, side="right") - 1 - p
    assert np.all(steps >= 0) and np.all((steps <= count[j]) | (count[j] == 127))
