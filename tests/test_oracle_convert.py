"""Pins for the oracle's own fp32 -> fp16 / bfloat16 rounding.

The oracle rounds to nearest, ties to even, in C on the bit patterns. These
tests hold it against library conversions that are independent of it: numpy's
float32 -> float16 cast and torch's float32 -> bfloat16 cast (both IEEE
round-to-nearest-even). NaN inputs are compared by class only.
"""
import numpy as np
import pytest
import torch


def _structured_f32_patterns():
    """Bit patterns that hit every rounding corner of the narrow formats."""
    rng = np.random.default_rng(1234)
    pats = [rng.integers(0, 2**32, size=1 << 22, dtype=np.uint64).astype(np.uint32)]
    # every exponent x a set of mantissas around the fp16 (13 dropped bits) and
    # bf16 (16 dropped bits) rounding points, both signs
    lows = np.array([0, 1, 2, 0x0FFF, 0x1000, 0x1001, 0x1FFF, 0x2000, 0x3000, 0x7FFF,
                     0x8000, 0x8001, 0xFFFF, 0x10000, 0x18000, 0x7FFFFF, 0x400000, 0x7FE000,
                     0x7FF000, 0x7FEFFF, 0x7FF001], dtype=np.uint32)
    highs = (np.arange(0, 1 << 7, dtype=np.uint32) << 16)     # a spread of upper mantissa bits
    mant = (highs[:, None] | lows[None, :]).reshape(-1) & 0x7FFFFF
    exps = np.arange(0, 256, dtype=np.uint32) << 23
    body = (exps[:, None] | mant[None, :]).reshape(-1)
    pats.append(body)
    pats.append(body | 0x80000000)
    # fp16 subnormal / overflow neighbourhoods, all mantissas
    for e in (101, 102, 103, 110, 112, 113, 142, 143):
        allm = (np.uint32(e) << 23) | np.arange(0, 1 << 23, 37, dtype=np.uint32)
        pats.append(allm)
        pats.append(allm | 0x80000000)
    return np.concatenate(pats).astype(np.uint32)


def test_f32_to_f16_matches_numpy(orc):
    bits = _structured_f32_patterns()
    x = bits.view(np.float32)
    ours = orc.f32_to_f16_bits(x)
    with np.errstate(over="ignore", invalid="ignore"):
        ref = x.astype(np.float16).view(np.uint16)
    nan = np.isnan(x)
    assert np.array_equal(ours[~nan], ref[~nan])
    # NaN class only: exponent all ones, nonzero mantissa
    assert np.all((ours[nan] & 0x7C00) == 0x7C00) and np.all((ours[nan] & 0x3FF) != 0)


def test_f32_to_bf16_matches_torch(orc):
    bits = _structured_f32_patterns()
    x = bits.view(np.float32)
    ours = orc.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    nan = np.isnan(x)
    assert np.array_equal(ours[~nan], ref[~nan])
    assert np.all((ours[nan] & 0x7F80) == 0x7F80) and np.all((ours[nan] & 0x7F) != 0)


def test_f16_to_f32_exhaustive(orc):
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ours = orc.f16_bits_to_f32(h)
    ref = h.view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(ours[~nan].view(np.uint32), ref[~nan].view(np.uint32))
    assert np.all(np.isnan(ours[nan]))


@pytest.mark.slow
def test_f32_narrowing_all_patterns(orc):
    """Every one of the 2^32 binary32 patterns (run with -m slow)."""
    step = 1 << 24
    for start in range(0, 1 << 32, step):
        bits = np.arange(start, start + step, dtype=np.uint64).astype(np.uint32)
        x = bits.view(np.float32)
        nan = np.isnan(x)
        with np.errstate(over="ignore", invalid="ignore"):
            r16 = x.astype(np.float16).view(np.uint16)
        assert np.array_equal(orc.f32_to_f16_bits(x)[~nan], r16[~nan])
        rb = torch.from_numpy(x.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(orc.f32_to_bf16_bits(x)[~nan], rb[~nan])
