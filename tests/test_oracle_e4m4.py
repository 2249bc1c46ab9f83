"""Pins of the oracle's E4M4 absmax codec (bitsandbytes k-bit series, PATCH 005 "Add
vectorized dequant kernel and E4M4 uint8 absmax support": encode_absmax_e4m4 and
decode_absmax_e4m4 in functional.py, decode_e4m4_absmax in ops.cu, and the E4M4 tests).

Each check ties the oracle to something other than its own formula: values the patch
prints, the kernel's bit-construction form of the decode, brute-force nearest-code search,
the round trip of every code, and the patch's stated SQNR cost.
"""
import math
import struct

import numpy as np
import pytest

import oracle

ALL = np.arange(256, dtype=np.uint8)


def _bits_decode(code: int) -> float:
    """The patch's kernel form: IEEE fields built directly, subnormals as m * 2^(1-bias-4)."""
    e, m = code >> 4, code & 15
    if e == 0:
        return m * 2.0 ** (1 - 11 - 4)
    return struct.unpack("<f", struct.pack("<I", ((e - 11 + 127) << 23) | (m << 19)))[0]


def test_decode_matches_the_bit_construction_for_every_code():
    d = oracle.e4m4_decode(ALL)
    for c in range(256):
        assert float(d[c]) == _bits_decode(c), c


def test_decode_range_printed_by_the_patch():
    # the patch states that bias 11 spans about 6.1e-5 up to 31.0; code 0 is 0.0; exponent
    # field 11 is 2^0
    d = oracle.e4m4_decode(ALL)
    assert d[0] == 0.0
    assert d[1] == 2.0 ** -14 and abs(d[1] - 6.1e-5) < 1e-6
    assert d[255] == 31.0
    assert d[0xB0] == 1.0
    assert np.all(np.diff(d.astype(np.float64)) > 0), "decode must be strictly increasing"


def test_every_code_is_a_fixed_point_of_encode():
    assert np.array_equal(oracle.e4m4_encode(oracle.e4m4_decode(ALL)), ALL)


def test_patch_roundtrip_values():
    # the patch's test_encode_decode_roundtrip values: zero exact, relative error < 12.5 %
    v = np.array([0.0, 0.001, 0.01, 0.05, 0.1, 0.5, 1.0, 2.0, 5.0, 10.0, 25.0], np.float32)
    d = oracle.e4m4_decode(oracle.e4m4_encode(v))
    assert d[0] == 0.0
    rel = np.abs(d[1:].astype(np.float64) - v[1:]) / v[1:]
    assert np.all(rel < 0.125), rel


def _nearest_in_binade(a: float) -> int:
    """Brute force: the nearest code among those sharing a's binade (ties to the even mantissa);
    below 2^-10 the 16 subnormal codes m * 2^-14."""
    if a < 2.0 ** -10:
        cands = [(m, m * 2.0 ** -14) for m in range(16)]
        ef = 0
    else:
        e = math.frexp(a)[1] - 1
        ef = e + 11
        assert 1 <= ef <= 15
        cands = [(m, 2.0 ** e * (1 + m / 16)) for m in range(16)]
    best = min(abs(v - a) for _, v in cands)
    ms = [m for m, v in cands if abs(v - a) == best]
    m = ms[0] if len(ms) == 1 else [x for x in ms if x % 2 == 0][0]
    return (ef << 4) | m


def test_encode_is_the_nearest_code_of_the_binade():
    rng = np.random.default_rng(7)
    # log-uniform over the whole representable range, plus the awkward spots of each binade
    a = np.exp2(rng.uniform(-16.0, 5.0, 20000)).astype(np.float32)
    spots = []
    for e in range(-14, 5):
        for m in range(16):
            base = 2.0 ** e * (1 + m / 16)
            half = base + 2.0 ** e / 32           # midpoint to the next step: a tie
            spots += [base, half, np.nextafter(np.float32(half), np.float32(0)),
                      np.nextafter(np.float32(half), np.float32(np.inf))]
        spots += [np.nextafter(np.float32(2.0 ** (e + 1)), np.float32(0))]   # just below 2^(e+1)
    a = np.concatenate([a, np.array(spots, np.float32)])
    a = a[(a > 0) & (a < 32)]
    got = oracle.e4m4_encode(a)
    for x, c in zip(a.tolist(), got.tolist()):
        assert c == _nearest_in_binade(x), (x, hex(c))


def test_encode_special_inputs():
    v = np.array([0.0, -0.0, -1.0, np.nan, np.inf, 1e-30, 2.0 ** -15, 32.0, 64.0, 100.0], np.float32)
    got = oracle.e4m4_encode(v).tolist()
    assert got[:4] == [0, 0, 0, 0]                 # not > 0: code 0 (the patch's nonzero mask)
    assert got[4] == 0xFF                          # reading: infinity saturates
    assert got[5] == 0 and got[6] == 0             # rounds to the zero subnormal (2^-15: a tie to m=0)
    # reading: at and above 32 the exponent field clamps to 15 and the mantissa keeps a's own
    # binade (the patch computes m with the unclamped exponent)
    assert got[7:] == [0xF0, 0xF0, 0xF9]


@pytest.mark.parametrize("K", [2, 3, 4, 5])
def test_sqnr_cost_stated_by_the_patch(K):
    """'SQNR degradation is <0.4 dB across all K values' (1M N(0,1) fp32 values)."""
    x = np.random.default_rng(0).standard_normal(1 << 20).astype(np.float32)
    cb = oracle.normal_float_codebook(K)
    packed, am = oracle.kbit_quantize(x, "f32", K, cb)
    p2, am8 = oracle.kbit_quantize_e4m4(x, "f32", K, cb)
    assert np.array_equal(packed, p2)
    y = oracle.kbit_dequantize(packed, am, cb, K, x.size, "f32").astype(np.float64)
    y8 = oracle.kbit_dequantize_e4m4(packed, am8, cb, K, x.size, "f32").astype(np.float64)
    sig = np.sum(x.astype(np.float64) ** 2)
    sqnr = 10 * np.log10(sig / np.sum((x - y) ** 2))
    sqnr8 = 10 * np.log10(sig / np.sum((x - y8) ** 2))
    assert sqnr - sqnr8 < 0.4, (sqnr, sqnr8)
    assert sqnr8 > {2: 5, 3: 10, 4: 15, 5: 20}[K] - 0.4


def test_storage_bits_per_element():
    # the patch gives 5.0 bits per element at K=4 with fp32 absmax and 4.25 with one E4M4 byte:
    # K bits + one absmax per 32 elements
    assert 4 + 32 / 32 == 5.0 and 4 + 8 / 32 == 4.25
