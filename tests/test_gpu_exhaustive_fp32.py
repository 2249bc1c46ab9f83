"""Exhaustive check of the fp32 quantize path's threshold table against the oracle (-m slow).

The quantize kernel decides each index from per-CTA thresholds and a 256-cell table instead of
the pages' brute-force search (kQuantizeBlockwise_kbit: first index minimising fabsf(xn - c),
xn = x / max(absmax, 1e-8f)). Here every fp32 value in [-1, 1] is quantized once per K in blocks
whose absmax is exactly 1 (element 0 of each block is +-1, so xn = x), through the fp32
half-block path (fp32 input always takes it), and the packed words are compared bit for bit with
the C oracle run on all host cores. Then a strided subset of the same values, scaled into blocks
whose maxima are not powers of two, exercises the exact two-FMA test with real divisors.
"""
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import oracle
from tests.gpu_util import to_host

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

CHUNK = 1 << 26                 # test values per GPU launch (31 per block of 32)


@pytest.fixture(scope="module")
def bbc():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from blockwise_bit_codebook_b200 import build
    build.build()
    import blockwise_bit_codebook_b200 as m
    m.load_library()
    return m


def _oracle_packed(x: np.ndarray, K: int, cb: np.ndarray) -> np.ndarray:
    """The oracle's packed words for x (a whole number of blocks), on all host cores."""
    nb = x.size // 32
    threads = max(1, os.cpu_count() or 1)
    per = -(-nb // threads)
    ranges = [(b, min(nb, b + per)) for b in range(0, nb, per)]
    out = np.empty(nb * K, np.uint32)

    def one(r):
        lo, hi = r
        out[lo * K:hi * K] = oracle.kbit_quantize(x[lo * 32:hi * 32], "f32", K, cb)[0]

    with ThreadPoolExecutor(max_workers=len(ranges)) as ex:
        list(ex.map(one, ranges))
    return out


def _blocks(values: np.ndarray, lead: np.ndarray) -> np.ndarray:
    """Blocks of 32: element 0 = lead[b] (the block's absmax), elements 1..31 = the next 31 values."""
    nb = -(-values.size // 31)
    v = np.zeros(nb * 31, np.float32)
    v[:values.size] = values
    x = np.empty((nb, 32), np.float32)
    x[:, 0] = lead[:nb]
    x[:, 1:] = v.reshape(nb, 31)
    return x.reshape(-1)


def _run(bbc, x: np.ndarray, K: int, cb: np.ndarray, what: str):
    xd = torch.from_numpy(x).cuda()
    packed, _ = bbc.kbit_quantize(xd, K, torch.from_numpy(cb).cuda())
    torch.cuda.synchronize()
    got = to_host(packed)
    want = _oracle_packed(x, K, cb)
    bad = np.flatnonzero(got != want)
    assert bad.size == 0, f"{what}: {bad.size} differing words, first at word {bad[0]}"


@pytest.mark.parametrize("K", [2, 3, 4, 5])
def test_every_fp32_in_unit_interval(bbc, K):
    cb = oracle.normal_float_codebook(K)
    top = np.uint32(0x3F800000)                                  # bits of 1.0
    # the positive values 0 .. 1 and the negative ones -0 .. -1, in chunks of CHUNK patterns
    for sign in (0, 0x80000000):
        for start in range(0, int(top) + 1, CHUNK):
            bits = np.arange(start, min(start + CHUNK, int(top) + 1), dtype=np.uint32) | np.uint32(sign)
            lead = np.where(np.arange(-(-bits.size // 31)) % 2 == 0, 1.0, -1.0).astype(np.float32)
            _run(bbc, _blocks(bits.view(np.float32), lead), K, cb, f"K={K} sign={sign:#x} start={start:#x}")


@pytest.mark.parametrize("K", [3, 5])
@pytest.mark.parametrize("amax", [0.7071067690849304, 1.3716789484024048])
def test_strided_values_with_other_block_maxima(bbc, K, amax):
    cb = oracle.normal_float_codebook(K)
    a = np.float32(amax)
    bits = np.arange(0, 0x3F800001, 61, dtype=np.uint32)          # every 61st pattern in [0, 1]
    vals = np.concatenate([bits, bits | np.uint32(0x80000000)]).view(np.float32) * a
    for start in range(0, vals.size, CHUNK):
        chunk = vals[start:start + CHUNK]
        lead = np.full(-(-chunk.size // 31), a, np.float32)
        _run(bbc, _blocks(chunk.astype(np.float32), lead), K, cb, f"K={K} amax={amax} start={start}")
