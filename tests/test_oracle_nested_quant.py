"""Pins of the oracle's nested 4-bit quantize (the inverse of the nested dequant).

The nested-dequant page ("Fuse nested 4-bit scale reconstruction on SM103") defines only the
decode; the quantize steps are readings: the k-bit rule of the bitsandbytes k-bit series
(absmax, fmaxf(absmax, 1e-8f), IEEE division, first nearest entry) per outer block, the offset as
the mean of the outer absmax (pairwise binary64 sum), and General8 codes of the centred absmax
per group of 256 outer blocks. Each pin checks against something other than the oracle's own
code: numpy brute force on small inputs, exact rationals, the already-pinned dequant, and the
error bounds the k-bit pages state.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from blockwise_bit_codebook_b200 import synthetic

NF4 = oracle.normal_float_codebook(4)
FP4 = synthetic.fp4_table()
G8 = synthetic.general8_table()


def _widen(x_bits, dt):
    if dt == "f32":
        return x_bits.astype(np.float32)
    return (oracle.f16_bits_to_f32 if dt == "f16" else oracle.bf16_bits_to_f32)(x_bits)


def _brute_quantize_4bit(x32: np.ndarray, bs: int, code4: np.ndarray):
    n = x32.size
    nbo = (n + bs - 1) // bs
    absmax = np.array([np.max(np.abs(x32[b * bs:(b + 1) * bs])) for b in range(nbo)], np.float32)
    idx = np.empty(n, np.uint8)
    for b in range(nbo):
        d = np.float32(max(absmax[b], np.float32(1e-8)))
        seg = x32[b * bs:(b + 1) * bs]
        xn = (seg / d).astype(np.float32)
        dist = np.abs(xn[:, None] - code4[None, :].astype(np.float32))
        idx[b * bs:b * bs + seg.size] = np.argmin(dist, axis=1)          # first minimum
    codes = np.zeros((n + 1) // 2, np.uint8)
    codes |= (idx[0::2] << 4).astype(np.uint8)
    codes[: n // 2] |= idx[1::2]
    return codes, absmax


@pytest.mark.parametrize("dt", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("table", ["nf4", "fp4"])
def test_quantize_4bit_brute_force(dt, table):
    code4 = NF4 if table == "nf4" else FP4
    rng = np.random.default_rng(1)
    for n, bs in [(1, 32), (31, 32), (64, 64), (65, 64), (1000, 128), (4097, 4096), (300, 32)]:
        x = (rng.standard_normal(n) * rng.choice([1e-3, 0.02, 3.0])).astype(np.float32)
        x[rng.random(n) < 0.05] = 0.0
        if dt == "f32":
            xb = x
        else:
            xb = (oracle.f32_to_f16_bits if dt == "f16" else oracle.f32_to_bf16_bits)(x)
        codes, absmax = oracle.quantize_4bit(xb, dt, bs, code4)
        ref_c, ref_a = _brute_quantize_4bit(_widen(xb, dt), bs, code4)
        assert np.array_equal(absmax.view(np.uint32), ref_a.view(np.uint32)), (n, bs)
        assert np.array_equal(codes, ref_c), (n, bs)
        if n % 2:
            assert codes[-1] & 0x0F == 0                        # unused low nibble


def test_zero_and_tiny_blocks():
    x = np.zeros(64, np.float32)
    x[32:] = 1e-30
    codes, absmax = oracle.quantize_4bit(x, "f32", 32, NF4)
    assert absmax[0] == 0.0 and absmax[1] == np.float32(1e-30)
    zero_code = int(np.argmin(np.abs(NF4)))                      # nearest entry to 0.0
    assert np.all(codes[:16] == (zero_code << 4 | zero_code))   # 0 / 1e-8 = 0
    assert np.all(codes[16:] == (zero_code << 4 | zero_code))   # 1e-30 / 1e-8 rounds near 0


def test_exact_code_values_survive_the_roundtrip():
    """x made of exact code values times each block's absmax: quantize then the pinned plain
    4-bit dequant gives x back bit for bit (this also pins the nibble order to the dequant's)."""
    rng = np.random.default_rng(2)
    for code4 in (NF4, FP4):
        for bs in (32, 64, 4096):
            n = 3 * bs + 7
            nbo = (n + bs - 1) // bs
            scales = np.float32(2.0) ** rng.integers(-6, 6, nbo).astype(np.float32)
            v = rng.integers(0, 16, n)
            x = (code4[v] * np.repeat(scales, bs)[:n]).astype(np.float32)
            x[np.arange(nbo) * bs] = np.repeat(scales, 1)[:nbo]     # an element at +absmax
            codes, absmax = oracle.quantize_4bit(x, "f32", bs, code4)
            assert np.array_equal(absmax, scales)
            y = oracle.dequantize_4bit(codes, absmax, code4, n, bs, "f32")
            # FP4's -0.0 (code 8) ties with +0.0 (code 0) and the first entry wins: same value,
            # other sign bit; every other element comes back bit for bit
            neg0 = (x == 0) & np.signbit(x)
            assert np.array_equal(y.view(np.uint32)[~neg0], x.view(np.uint32)[~neg0]), bs
            assert np.all(y[neg0] == 0) and not np.any(np.signbit(y[neg0]))


@pytest.mark.parametrize("bs", [32, 64, 256])
def test_quantize_error_bound(bs):
    """Per-block error of dequant(quantize(x)) <= max_gap/2 * absmax (+ rounding), the k-bit
    pages' analytic bound applied to the 16-entry table."""
    x = np.random.default_rng(3).standard_normal(1 << 16).astype(np.float32)
    codes, absmax = oracle.quantize_4bit(x, "f32", bs, NF4)
    y = oracle.dequantize_4bit(codes, absmax, NF4, x.size, bs, "f32")
    half_gap = np.max(np.diff(np.sort(NF4.astype(np.float64)))) / 2
    bound = np.repeat(absmax.astype(np.float64), bs)[: x.size] * (half_gap + 1e-6) + 1e-6
    assert np.all(np.abs(y.astype(np.float64) - x) <= bound)


def test_offset_is_the_mean():
    rng = np.random.default_rng(4)
    for nbo in (1, 2, 3, 7, 2048, 2049, 10000, 70001):
        a = np.abs(rng.standard_normal(nbo)).astype(np.float32) * np.float32(0.05)
        off = oracle.absmax_offset(a)
        exact = sum(Fraction(float(v)) for v in a) / nbo
        # within one ulp of the exact mean (the binary64 sums lose far less than that)
        # and equal to a pairwise binary64 sum done here with numpy's own float64 adds
        p = 1 << max(0, (nbo - 1).bit_length())
        v = np.zeros(p, np.float64)
        v[:nbo] = a
        while v.size > 1:
            v = v[0::2] + v[1::2]
        assert off == np.float32(v[0] / nbo), nbo
        ulp = np.spacing(np.float32(float(exact)))
        assert abs(Fraction(float(off)) - exact) <= Fraction(float(ulp)), nbo
    assert oracle.absmax_offset(np.full(5000, 0.3, np.float32)) == np.float32(0.3)   # equal values
    assert np.isnan(oracle.absmax_offset(np.array([1.0, np.nan], np.float32)))


def test_absmax_compression_brute_force():
    rng = np.random.default_rng(5)
    for nbo in (1, 255, 256, 257, 1000):
        a = (np.abs(rng.standard_normal(nbo)) * 0.04 + 0.01).astype(np.float32)
        off = oracle.absmax_offset(a)
        q, a2 = oracle.quantize_absmax_nested(a, float(off), G8, 256)
        c = (a - off).astype(np.float32)
        for g in range(a2.size):
            seg = c[g * 256:(g + 1) * 256]
            assert a2[g] == np.max(np.abs(seg))
            d = np.float32(max(a2[g], np.float32(1e-8)))
            xn = (seg / d).astype(np.float32)
            dist = np.abs(xn[:, None] - G8[None, :])
            assert np.array_equal(q[g * 256:(g + 1) * 256], np.argmin(dist, axis=1))
        # the nested decode rebuilds each absmax within half a General8 gap of its group
        rebuilt = np.array([oracle.nested_scale(float(G8[q[b]]), float(a2[b // 256]), float(off))
                            for b in range(nbo)], np.float64)
        gap = np.max(np.diff(G8.astype(np.float64)))
        assert np.all(np.abs(rebuilt - a) <= np.repeat(a2.astype(np.float64), 256)[:nbo] * gap / 2 + 1e-6)


def test_nested_roundtrip_bound():
    x = synthetic.weights(64 * 256 * 3 + 100, std=0.02, seed=6).numpy()
    codes, q, a2, off = oracle.quantize_4bit_nested(x, "f32", 64, NF4, G8)
    y = oracle.nested_dequantize(codes, q, G8, a2, float(off), NF4, x.size, 64, 256, "f32")
    rel = np.max(np.abs(y - x)) / np.max(np.abs(x))
    assert rel < 0.15
    assert np.isfinite(off) and off > 0
