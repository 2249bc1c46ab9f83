"""Pins for the oracle's k-bit codec (bitsandbytes k-bit patch series).

What pins what:
- bit-plane format: the worked K=3 pattern (golden file) and numpy.unpackbits
  on random indices (a library bit routine), plus pack/unpack identity;
- nearest-entry rule: its defining property (a first minimiser of the fp32
  distance), exact hits, and constructed exact ties (lowest index wins);
- absmax: numpy max(|x|) per block;
- division and search together: exact rational division rounded once, on
  random and adversarial inputs;
- round trip: the pages' per-block error bound, MSE falling with K, and the
  SQNR floors of Stage 6 (K=2..5: 5, 10, 15, 20 dB on 1M N(0,1) values);
- dequant: special cases (absmax 1 gives the codebook entry; powers of two
  scale exactly; bf16/fp16 output equals a library cast of the fp32 product).
"""
import math
import os

import numpy as np
import pytest
import torch

from tests.exact import rn_div, rn_mul

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_pattern():
    d = {}
    for line in open(os.path.join(GOLDEN, "kbit_pack_k3_pattern.txt")):
        if line.startswith("#") or not line.strip():
            continue
        key, *vals = line.split()
        d[key] = vals
    return int(d["K"][0]), np.array(d["indices"], np.uint8), [int(w, 16) for w in d["words"]]


def test_known_pattern_k3(orc):
    K, idx, words = _read_pattern()
    packed = orc.kbit_pack(idx, K)
    assert [int(w) for w in packed] == words
    assert np.array_equal(orc.kbit_unpack(packed, K, idx.size), idx)


@pytest.mark.parametrize("K", [2, 3, 4, 5])
@pytest.mark.parametrize("n", [1, 31, 32, 33, 64, 65, 1000])
def test_pack_unpack_identity(orc, K, n):
    rng = np.random.default_rng(K * 1000 + n)
    idx = rng.integers(0, 1 << K, n, dtype=np.uint8)
    packed = orc.kbit_pack(idx, K)
    assert packed.size == ((n + 31) // 32) * K
    assert np.array_equal(orc.kbit_unpack(packed, K, n), idx)


@pytest.mark.parametrize("K", [2, 3, 4, 5])
def test_pack_matches_unpackbits(orc, K):
    rng = np.random.default_rng(7 + K)
    n = 32 * 50
    idx = rng.integers(0, 1 << K, n, dtype=np.uint8)
    packed = orc.kbit_pack(idx, K).reshape(-1, K)
    # bit i (little-endian) of word j of block b must equal bit j of idx[32b+i]
    wordbits = np.unpackbits(packed.view(np.uint8).reshape(-1, K, 4), axis=2, bitorder="little")
    idxbits = np.unpackbits(idx.reshape(-1, 32, 1), axis=2, bitorder="little")[:, :, :K]
    assert np.array_equal(wordbits, idxbits.transpose(0, 2, 1))


def _first_min_ok(xn, cb, i):
    d = np.abs(np.float32(xn) - cb.astype(np.float32)).astype(np.float32)
    return bool(np.all(d[i] <= d) and np.all(d[:i] > d[i]))


@pytest.mark.parametrize("K", [2, 3, 4, 5])
def test_nearest_entry_defining_property(orc, K):
    cb = orc.normal_float_codebook(K)
    rng = np.random.default_rng(K)
    xs = list(rng.uniform(-1, 1, 3000).astype(np.float32))
    mids = [(np.float32(a) + np.float32(b)) / np.float32(2) for a, b in zip(cb[:-1], cb[1:])]
    for m in mids:
        for s in range(-3, 4):   # the midpoint and its fp32 neighbours
            xs.append(np.nextafter(m, np.float32(np.inf) if s > 0 else np.float32(-np.inf)) if s else m)
            m2 = m
            for _ in range(abs(s)):
                m2 = np.nextafter(m2, np.float32(np.inf) if s > 0 else np.float32(-np.inf))
            xs.append(m2)
    xs += [np.float32(v) for v in (-1.0, 1.0, 0.0, -0.0, 1e-40, -1e-40, 1e-30)]
    for x in xs:
        i = orc.nearest_entry(float(x), cb)
        assert _first_min_ok(x, cb, i), (x, i)


def test_nearest_entry_exact_hits_and_ties(orc):
    cb = np.array([-1.0, -0.5, 0.25, 1.0], np.float32)
    for i, c in enumerate(cb):
        assert orc.nearest_entry(float(c), cb) == i
    # exact fp32 ties: equal rounded distances go to the lower index
    assert orc.nearest_entry(-0.75, cb) == 0     # |-.75+1| == |-.75+.5| == .25
    assert orc.nearest_entry(-0.125, cb) == 1    # .375 == .375
    assert orc.nearest_entry(0.625, cb) == 2     # .375 == .375
    # NF codebooks have no zero entry: 0.0 is an exact tie between the two centre entries
    for k in (2, 3, 4, 5):
        cbk = orc.normal_float_codebook(k)
        assert orc.nearest_entry(0.0, cbk) == (1 << k) // 2 - 1


@pytest.mark.parametrize("K", [2, 3, 4, 5])
@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_absmax_is_block_max_abs(orc, K, dtype):
    rng = np.random.default_rng(11)
    x = rng.standard_normal(32 * 40 + 7).astype(np.float32)
    if dtype == "f32":
        A, xf = x, x
    elif dtype == "f16":
        A = x.astype(np.float16).view(np.uint16)
        xf = x.astype(np.float16).astype(np.float32)
    else:
        t = torch.from_numpy(x).to(torch.bfloat16)
        A = t.view(torch.int16).numpy().view(np.uint16)
        xf = t.float().numpy()
    _, absmax = orc.kbit_quantize(A, dtype, K, orc.normal_float_codebook(K))
    pad = np.zeros(((xf.size + 31) // 32) * 32, np.float32)
    pad[: xf.size] = xf
    assert np.array_equal(absmax, np.abs(pad.reshape(-1, 32)).max(axis=1))


def _indices_by_exact_division(x, cb):
    """Each element's index from an exactly rounded quotient and the defining property."""
    x = x.astype(np.float32)
    out = []
    for blk in x.reshape(-1, 32):
        amax = np.float32(np.abs(blk).max())
        d = max(amax, np.float32(1e-8))
        for v in blk:
            xn = rn_div(v, d)
            dist = np.abs(xn - cb).astype(np.float32)
            out.append(int(np.flatnonzero(dist == dist.min())[0]))
    return np.array(out, np.uint8)


@pytest.mark.parametrize("K", [2, 3, 4, 5])
def test_quantize_indices_exact_division(orc, K):
    cb = orc.normal_float_codebook(K)
    rng = np.random.default_rng(100 + K)
    x = rng.standard_normal(32 * 24).astype(np.float32)
    x[::97] *= 20.0                       # outliers
    x[32:64] = rng.uniform(-1e-9, 1e-9, 32)   # a block under the 1e-8 clamp
    x[64:96] = 0.0                        # an all-zero block
    x[96:128] = rng.standard_normal(32).astype(np.float32) * 1e-39   # subnormal inputs
    _, _, idx = orc.kbit_quantize(x, "f32", K, cb, return_indices=True)
    assert np.array_equal(idx, _indices_by_exact_division(x, cb))


def test_padding_lanes_encode_zero(orc):
    K = 4
    cb = orc.normal_float_codebook(K)
    x = np.random.default_rng(3).standard_normal(33).astype(np.float32)
    packed, absmax, idx = orc.kbit_quantize(x, "f32", K, cb, return_indices=True)
    z = orc.nearest_entry(0.0, cb)
    assert np.all(idx[33:64] == z)
    assert absmax[1] == abs(x[32])


def _roundtrip(orc, x, K):
    cb = orc.normal_float_codebook(K)
    packed, absmax = orc.kbit_quantize(x, "f32", K, cb)
    y = orc.kbit_dequantize(packed, absmax, cb, K, x.size, "f32")
    return cb, absmax, y


@pytest.mark.parametrize("K", [2, 3, 4, 5])
def test_roundtrip_error_bound(orc, K):
    x = np.random.default_rng(42).standard_normal(1 << 16).astype(np.float32)
    cb, absmax, y = _roundtrip(orc, x, K)
    max_gap = float(np.diff(cb).max())
    err = np.abs(x.astype(np.float64) - y).reshape(-1, 32).max(axis=1)
    assert np.all(err <= max_gap / 2 * absmax + 1e-6)


def test_mse_decreases_and_sqnr_floors(orc):
    x = np.random.default_rng(123).standard_normal(1 << 20).astype(np.float32)
    mse = {}
    for K in (2, 3, 4, 5):
        _, _, y = _roundtrip(orc, x, K)
        mse[K] = float(np.mean((x.astype(np.float64) - y) ** 2))
        sqnr = 10 * math.log10(float(np.mean(x.astype(np.float64) ** 2)) / mse[K])
        assert sqnr > {2: 5, 3: 10, 4: 15, 5: 20}[K], (K, sqnr)
    for K in (3, 4, 5):
        assert mse[K] <= mse[K - 1] * 1.05


def test_all_zero_input(orc):
    K = 3
    cb = orc.normal_float_codebook(K)
    x = np.zeros(64, np.float32)
    packed, absmax = orc.kbit_quantize(x, "f32", K, cb)
    assert np.all(absmax == 0)
    y = orc.kbit_dequantize(packed, absmax, cb, K, 64, "f32")
    assert np.all(y == 0)                   # c * 0 is a signed zero


@pytest.mark.parametrize("K", [2, 3, 4, 5])
def test_dequant_special_cases(orc, K):
    cb = orc.normal_float_codebook(K)
    rng = np.random.default_rng(5)
    n = 32 * 8 + 3
    idx = rng.integers(0, 1 << K, n, dtype=np.uint8)
    packed = orc.kbit_pack(idx, K)
    nb = (n + 31) // 32
    ones = np.ones(nb, np.float32)
    # absmax 1, fp32: the codebook entry itself
    assert np.array_equal(orc.kbit_dequantize(packed, ones, cb, K, n, "f32"), cb[idx])
    # powers of two scale exactly
    p2 = (2.0 ** rng.integers(-20, 20, nb)).astype(np.float32)
    y = orc.kbit_dequantize(packed, p2, cb, K, n, "f32")
    assert np.array_equal(y, cb[idx] * p2[np.arange(n) // 32])
    # general absmax: one exact-rounded fp32 product, then a library cast
    am = rng.uniform(0.01, 50, nb).astype(np.float32)
    prod = np.array([rn_mul(cb[idx[m]], am[m // 32]) for m in range(n)], np.float32)
    assert np.array_equal(orc.kbit_dequantize(packed, am, cb, K, n, "f32"), prod)
    assert np.array_equal(orc.kbit_dequantize(packed, am, cb, K, n, "f16"),
                          prod.astype(np.float16).view(np.uint16))
    bf = torch.from_numpy(prod).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(orc.kbit_dequantize(packed, am, cb, K, n, "bf16"), bf)


def test_dtypes_input_exact_widening(orc):
    """fp16/bf16 inputs give the same result as their exact fp32 values."""
    K = 4
    cb = orc.normal_float_codebook(K)
    x = np.random.default_rng(9).standard_normal(32 * 30 + 5).astype(np.float32)
    h = x.astype(np.float16)
    a = orc.kbit_quantize(h.view(np.uint16), "f16", K, cb)
    b = orc.kbit_quantize(h.astype(np.float32), "f32", K, cb)
    assert all(np.array_equal(u, v) for u, v in zip(a, b))
    t = torch.from_numpy(x).to(torch.bfloat16)
    a = orc.kbit_quantize(t.view(torch.int16).numpy().view(np.uint16), "bf16", K, cb)
    b = orc.kbit_quantize(t.float().numpy(), "f32", K, cb)
    assert all(np.array_equal(u, v) for u, v in zip(a, b))
