"""Pins for the oracle's nested 4-bit dequant ("Fuse nested 4-bit scale
reconstruction on SM103", Summary and Implementation).

What pins what:
- the scale is an fp32 multiply then a separate fp32 add (no fused
  multiply-add): triples where fma and two roundings differ are searched with
  exact rational arithmetic, and the oracle must return the two-rounding value;
- index structure (outer block m // bs, inner group b // bs2) through powers of
  two that make every product exact;
- nibble order (golden file, a stated reading);
- with a unit scale the output reduces to a library cast of code4[v];
- the full 256 x 16 code sweep against exact rationals rounded step by step.
"""
import os

import numpy as np
import pytest
import torch

from tests.exact import rn_add, rn_fma, rn_mul

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _cast(prod_f32: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f32":
        return prod_f32.astype(np.float32)
    if dtype == "f16":
        with np.errstate(over="ignore"):
            return prod_f32.astype(np.float16).view(np.uint16)
    return torch.from_numpy(prod_f32.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def find_nofma_triples(count=16, seed=0):
    rng = np.random.default_rng(seed)
    found = []
    while len(found) < count:
        a = np.float32(rng.uniform(-1, 1))
        b = np.float32(rng.uniform(0.01, 0.1))
        c = np.float32(rng.normal(0.03, 0.005))
        two = rn_add(rn_mul(a, b), c)
        fused = rn_fma(a, b, c)
        if two != fused:
            found.append((a, b, c, two, fused))
    return found


def test_scale_is_multiply_then_add(orc):
    for a, b, c, two, fused in find_nofma_triples():
        got = np.float32(orc.nested_scale(float(a), float(b), float(c)))
        assert got == two and got != fused


def test_nofma_triples_through_dequant(orc):
    triples = find_nofma_triples(8, seed=1)
    code2 = np.zeros(256, np.float32)
    code4 = np.ones(16, np.float32)
    for i, (a, b, c, two, _) in enumerate(triples):
        code2[:] = a
        out = orc.nested_dequantize(np.zeros(32, np.uint8), np.zeros(1, np.uint8), code2,
                                    np.array([b], np.float32), float(c), code4, 64, 64, 256, "f32")
        assert np.all(out == two)


def _read_nibble_cases():
    cases = []
    for line in open(os.path.join(GOLDEN, "nested_nibble_order.txt")):
        if not line.startswith("case"):
            continue
        _, n, codes, outs = [s.strip() for s in line.replace("case", "case|", 1).split("|")]
        cases.append((int(n), bytes.fromhex(codes.replace(" ", "")), [float(v) for v in outs.split()]))
    return cases


def test_nibble_order_golden(orc):
    code4 = np.arange(16, dtype=np.float32)
    for n, codes, expect in _read_nibble_cases():
        out = orc.nested_dequantize(np.frombuffer(codes, np.uint8), np.zeros(1, np.uint8),
                                    np.ones(256, np.float32), np.ones(1, np.float32), 0.0,
                                    code4, n, 32, 256, "f32")
        assert list(out) == expect


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_unit_scale_reduces_to_cast(orc, dtype):
    rng = np.random.default_rng(2)
    code4 = rng.standard_normal(16).astype(np.float32) * np.float32(3.0)
    n = 4096 + 7
    codes = rng.integers(0, 256, (n + 1) // 2, dtype=np.uint8)
    nbo = (n + 63) // 64
    out = orc.nested_dequantize(codes, rng.integers(0, 256, nbo, dtype=np.uint8),
                                np.ones(256, np.float32), np.ones((nbo + 255) // 256, np.float32),
                                0.0, code4, n, 64, 256, dtype)
    nib = np.empty(n, np.int64)
    nib[0::2] = codes[: (n + 1) // 2] >> 4
    nib[1::2] = codes[: n // 2] & 15
    assert np.array_equal(out, _cast(code4[nib], dtype))


@pytest.mark.parametrize("bs", [32, 64, 128, 256, 1024, 4096])
def test_index_structure_powers_of_two(orc, bs):
    """code2[q] = 2^(q-128), absmax2[g] = 2^-g, offset 0, code4 = 1: out = 2^(q_b - 128 - g)."""
    rng = np.random.default_rng(bs)
    bs2 = 256
    n = bs * bs2 * 2 + bs * 3 + 5          # 2 full inner groups, a partial one, a partial block
    nbo = (n + bs - 1) // bs
    nbi = (nbo + bs2 - 1) // bs2
    code2 = np.array([2.0 ** (q - 128) for q in range(256)], np.float32)
    absmax2 = np.array([2.0 ** -g for g in range(nbi)], np.float32)
    q = rng.integers(0, 256, nbo, dtype=np.uint8)
    codes = rng.integers(0, 256, (n + 1) // 2, dtype=np.uint8)
    out = orc.nested_dequantize(codes, q, code2, absmax2, 0.0, np.ones(16, np.float32),
                                n, bs, bs2, "f32")
    m = np.arange(n)
    b = m // bs
    expect = np.ldexp(np.float32(1.0), (q[b].astype(np.int64) - 128 - b // bs2).astype(np.int32))
    assert np.array_equal(out, expect.astype(np.float32))


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_full_code_sweep_exact(orc, dtype):
    """Every General8 code x every 4-bit code, several inner absmax values and offsets."""
    rng = np.random.default_rng(17)
    code2 = np.sort(rng.uniform(-1, 1, 256).astype(np.float32))
    code2[0], code2[128], code2[255] = -1.0, 0.0, 1.0
    code4 = rng.standard_normal(16).astype(np.float32)
    bs, bs2 = 32, 256
    for absmax2_val, offset in [(1.0, 0.0), (0.0371, 0.0), (0.0523, 0.0312), (3.5, -0.75)]:
        absmax2_val = np.float32(absmax2_val)
        offset = np.float32(offset)
        # element m: code byte gives (hi, lo) = all 256 byte values per block; q = block index
        codes = np.concatenate([np.arange(256, dtype=np.uint8)] * 16)[: 256 * bs // 2]
        q = np.arange(256, dtype=np.uint8)
        n = 256 * bs
        out = orc.nested_dequantize(codes, q, code2, np.array([absmax2_val], np.float32),
                                    float(offset), code4, n, bs, bs2, dtype)
        scales = [rn_add(rn_mul(code2[i], absmax2_val), offset) for i in range(256)]
        nib = np.empty(n, np.int64)
        nib[0::2] = codes >> 4
        nib[1::2] = codes & 15
        prod = np.array([rn_mul(code4[nib[m]], scales[m // bs]) for m in range(n)], np.float32)
        assert np.array_equal(out, _cast(prod, dtype))
        # every 4-bit code appears
        assert set(nib.tolist()) == set(range(16))


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_plain_4bit_special_cases(orc, dtype):
    """Plain 4-bit decode: unit absmax is a cast, powers of two scale exactly, general absmax is
    one exact-rational product then a cast."""
    rng = np.random.default_rng(23)
    n, bs = 64 * 40 + 9, 64
    nb = (n + bs - 1) // bs
    code4 = rng.standard_normal(16).astype(np.float32)
    codes = rng.integers(0, 256, (n + 1) // 2, dtype=np.uint8)
    nib = np.empty(n, np.int64)
    nib[0::2] = codes[: (n + 1) // 2] >> 4
    nib[1::2] = codes[: n // 2] & 15
    ones = np.ones(nb, np.float32)
    assert np.array_equal(orc.dequantize_4bit(codes, ones, code4, n, bs, dtype), _cast(code4[nib], dtype))
    p2 = (2.0 ** rng.integers(-10, 10, nb)).astype(np.float32)
    assert np.array_equal(orc.dequantize_4bit(codes, p2, code4, n, bs, dtype),
                          _cast((code4[nib] * p2[np.arange(n) // bs]).astype(np.float32), dtype))
    am = rng.uniform(0.001, 3, nb).astype(np.float32)
    prod = np.array([rn_mul(code4[nib[m]], am[m // bs]) for m in range(n)], np.float32)
    assert np.array_equal(orc.dequantize_4bit(codes, am, code4, n, bs, dtype), _cast(prod, dtype))


def test_plain_4bit_composes_with_nested_scale(orc):
    """Feeding the pinned nested scale to the plain decode reproduces the nested dequant."""
    rng = np.random.default_rng(29)
    n, bs = 64 * 600 + 11, 64
    nbo = (n + bs - 1) // bs
    code2 = np.sort(rng.uniform(-1, 1, 256).astype(np.float32))
    code4 = orc.normal_float_codebook(4)
    codes = rng.integers(0, 256, (n + 1) // 2, dtype=np.uint8)
    q = rng.integers(0, 256, nbo, dtype=np.uint8)
    a2 = rng.uniform(0.01, 0.1, (nbo + 255) // 256).astype(np.float32)
    off = float(np.float32(0.031))
    scales = np.array([orc.nested_scale(float(code2[q[b]]), float(a2[b // 256]), off) for b in range(nbo)],
                      np.float32)
    for dt in ("f32", "bf16"):
        assert np.array_equal(orc.dequantize_4bit(codes, scales, code4, n, bs, dt),
                              orc.nested_dequantize(codes, q, code2, a2, off, code4, n, bs, 256, dt))
