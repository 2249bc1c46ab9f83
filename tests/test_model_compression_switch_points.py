"""Host model of the compression kernel's fast table form, against the verbatim rule.

The nested quantize compresses each centred outer absmax to the first General8 entry nearest to
xn = RN(c / d), distances taken in fp32 (the pages' nearest-entry rule, first index on ties).
For a finite, strictly ascending table whose neighbouring gaps lie within a factor 2^20 of each
other (and, when the last entry is below 1, whose last gap is at least 2^-20 (1 + |t_254|)), the
kernel instead counts the switch points D_i <= xn, D_i being the smallest fp32 in (t_{i-1}, t_i]
at which t_i is strictly nearer than t_{i-1}, found by bisection over ordered keys (from a
checked bracket around the midpoint when it holds the change). This file
restates that arithmetic with numpy fp32 and checks the count against the verbatim rule
(np.argmin of the fp32 distances) for |xn| <= 1 on random values and on every value within a few
ulps of each entry and switch point, and shows that a table outside the condition can break it.
No GPU is involved.
"""
import numpy as np

from blockwise_bit_codebook_b200 import synthetic

F32 = np.float32


def okey(f):
    b = np.asarray(f, F32).view(np.uint32).astype(np.uint64)
    return np.where(b >> 31, b ^ 0xFFFFFFFF, b | 0x80000000).astype(np.uint64)


def from_okey(k):
    k = np.asarray(k, np.uint64)
    b = np.where(k >> 31, k & 0x7FFFFFFF, k ^ 0xFFFFFFFF).astype(np.uint32)
    return b.view(F32)


def rule(a, b, v):
    return F32(b) - v < v - F32(a)          # fp32 subtractions, strict: ties stay with a


def switch_point(a, b):
    lo, hi = int(okey(a)), int(okey(b))
    # the kernel's bracket of 16 keys around the midpoint, taken only when checked at both ends
    c = int(okey(F32(0.5 * (float(a) + float(b)))))
    l2, h2 = max(lo, c - 8), min(hi, c + 8)
    if l2 < h2 and not rule(a, b, from_okey(l2)) and rule(a, b, from_okey(h2)):
        lo, hi = l2, h2
    while hi - lo > 1:
        mid = lo + ((hi - lo) >> 1)
        if rule(a, b, from_okey(mid)):
            hi = mid
        else:
            lo = mid
    return from_okey(hi)


def fast_form_ok(t):
    t = np.asarray(t, F32)
    if not (np.all(np.isfinite(t)) and np.all(t[:-1] < t[1:])):
        return False
    g = np.diff(t.astype(np.float64))
    if not (np.all(g[:-1] >= 2.0 ** -20 * g[1:]) and np.all(g[1:] >= 2.0 ** -20 * g[:-1])):
        return False
    if t[-1] < 1 and not g[-1] >= 2.0 ** -20 * (1 + abs(float(t[-2]))):
        return False
    return True


def verbatim(xn, t):
    d = np.abs(xn[:, None].astype(F32) - t[None, :].astype(F32))
    return np.argmin(d, axis=1)              # first index of the minimum


def counted(xn, D):
    return np.searchsorted(D, xn, side="right")    # #{i : D_i <= xn}


def probes(t, D, rng, n_random=20000):
    pts = [rng.uniform(-1, 1, n_random).astype(F32), np.array([-1, 1, 0, -0.0], F32),
           np.array([1e-30, -1e-30, 1e-40, -1e-40], F32)]
    for base in (t, D):
        base = base[np.abs(base) <= 1]
        for k in range(-3, 4):
            pts.append(from_okey((okey(base).astype(np.int64) + k).astype(np.uint64)))
    xn = np.concatenate(pts).astype(F32)
    return xn[np.isfinite(xn) & (np.abs(xn) <= 1)]


def check_table(t, rng):
    t = np.asarray(t, F32)
    assert fast_form_ok(t)
    D = np.array([switch_point(t[i - 1], t[i]) for i in range(1, 256)], F32)
    assert np.all(D > t[:-1]) and np.all(D <= t[1:]) and np.all(D[:-1] < D[1:])
    xn = probes(t, D, rng)
    want = verbatim(xn, t)
    got = counted(xn, D)
    bad = np.flatnonzero(got != want)
    assert bad.size == 0, (xn[bad[:5]], got[bad[:5]], want[bad[:5]])
    return xn.size


def decade_table():
    """A signed table built by decades (18 magnitudes per decade from 1e-7 to 1, two more tiny
    ones, mirrored around 0): the shape of a dynamic 8-bit code, neighbouring gaps up to a factor
    ~10 apart."""
    mags = np.concatenate([np.linspace(10.0 ** (e - 1), 10.0 ** e, 19)[1:] for e in range(-6, 1)])
    pos = np.concatenate([[5e-8], mags])                       # 127 positive magnitudes, last 1
    neg = -np.concatenate([[2e-8], pos])[::-1]                 # 128 negative ones
    return np.concatenate([neg, [0.0], pos]).astype(F32)


def test_stand_in_general8_table():
    rng = np.random.default_rng(5)
    assert check_table(synthetic.general8_table(), rng) > 20000


def test_decade_table_and_scaled_copies():
    rng = np.random.default_rng(6)
    t = decade_table()
    assert np.unique(t).size == 256
    check_table(t, rng)
    # last entry below 1: quotients between t_255 and 1 must still pick entry 255
    check_table((t * F32(0.9)).astype(F32), rng)


def test_random_tables_in_the_condition():
    rng = np.random.default_rng(7)
    done = 0
    while done < 4:
        t = np.sort(rng.uniform(-1, 1, 256).astype(F32))
        t[0], t[-1] = F32(-1), F32(1)
        if fast_form_ok(t):
            check_table(t, rng)
            done += 1


def test_dense_cluster_in_the_condition():
    rng = np.random.default_rng(8)
    cluster = np.linspace(0.3 - 2e-4, 0.3 + 2e-4, 160, dtype=F32)
    rest = np.linspace(-1, 1, 96, dtype=F32)
    t = np.sort(np.concatenate([cluster, rest]))
    check_table(t, rng)              # several switch points per bucket of the kernel's table


def test_a_table_outside_the_condition_can_break_the_count():
    """Two tiny entries (1e-30, 2e-30) beside gaps of ~0.01: for xn between 2e-30 and the next
    entry their fp32 distances round alike, the verbatim rule keeps the first, and the count of
    switch points does not. The kernel takes the exact ascending search for such tables."""
    t = np.linspace(-1, 1, 256).astype(F32)
    t[127], t[128] = F32(1e-30), F32(2e-30)
    assert np.all(t[:-1] < t[1:]) and not fast_form_ok(t)
    D = np.array([switch_point(t[i - 1], t[i]) for i in range(1, 256)], F32)
    xn = np.linspace(t[128], t[129], 4001).astype(F32)
    assert np.any(counted(xn, D) != verbatim(xn, t))
