"""GPU parity of the E4M4-absmax k-bit codec against the oracle (bit-exact), through the C ABI.

bitsandbytes k-bit series, PATCH 005 "Add vectorized dequant kernel and E4M4 uint8 absmax
support": the packed words are those of the fp32-absmax quantize, the stored absmax is its
E4M4 code, and dequant multiplies by the code's exact value.
"""
import numpy as np
import pytest
import torch

import oracle
from blockwise_bit_codebook_b200 import synthetic
from tests.gpu_util import DTYPES, assert_bits_equal, to_host

pytestmark = pytest.mark.gpu
NAMES = {torch.float16: "f16", torch.bfloat16: "bf16", torch.float32: "f32"}


@pytest.fixture(scope="module")
def bbc():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from blockwise_bit_codebook_b200 import build
    build.build()
    import blockwise_bit_codebook_b200 as m
    m.load_library()
    return m


def roundtrip(bbc, x_host, K, x_dev=None, absmax_buf=None, what=""):
    dt = NAMES[x_host.dtype]
    n = x_host.numel()
    nb = (n + 31) // 32
    cb_np = oracle.normal_float_codebook(K)
    cb = torch.from_numpy(cb_np).cuda()
    ref_p, ref_a = oracle.kbit_quantize_e4m4(to_host(x_host), dt, K, cb_np)
    p, a = bbc.kbit_quantize_e4m4(x_host.cuda() if x_dev is None else x_dev, K, cb, absmax=absmax_buf)
    torch.cuda.synchronize()
    assert_bits_equal(to_host(a)[:nb], ref_a, f"e4m4 absmax {what} K={K} {dt}")
    assert_bits_equal(to_host(p)[:nb * K], ref_p, f"packed {what} K={K} {dt}")
    ref_y = oracle.kbit_dequantize_e4m4(ref_p, ref_a, cb_np, K, n, dt)
    y = bbc.kbit_dequantize_e4m4(p, a, cb, K, n, x_host.dtype)
    torch.cuda.synchronize()
    assert_bits_equal(to_host(y)[:n], ref_y, f"e4m4 dequant {what} K={K} {dt}")


@pytest.mark.parametrize("K", [2, 3, 4, 5])
@pytest.mark.parametrize("dt", ["f16", "bf16", "f32"])
def test_c2_sweep(bbc, K, dt):
    """4096x4096 N(0, 0.02) with 0.1 % outliers x20, every K and dtype."""
    x = synthetic.weights(4096 * 4096, std=0.02, seed=1, dtype=DTYPES[dt], outlier_frac=0.001)
    roundtrip(bbc, x, K, what="c2")


@pytest.mark.parametrize("dt", ["f16", "bf16", "f32"])
def test_ragged_and_unaligned(bbc, dt):
    for n in [1, 31, 33, 1000, 32 * 1024 + 17, 32 * 1024 * 2 + 32 * 7]:
        roundtrip(bbc, synthetic.weights(n, std=0.5, seed=n, dtype=DTYPES[dt]), 4, what=f"n={n}")
    n = 32 * 3000 + 5
    x = synthetic.weights(n + 1, std=1.0, seed=9, dtype=DTYPES[dt])
    buf = torch.zeros((n + 31) // 32 + 1, dtype=torch.uint8, device="cuda")
    roundtrip(bbc, x[1:].contiguous(), 3, x_dev=x.cuda()[1:], absmax_buf=buf[1:], what="offset pointers")
    assert int(buf[0]) == 0


def _blocks_with_absmax(a: np.ndarray) -> np.ndarray:
    """fp32 blocks whose absmax is exactly a[b]: a[b] at a varying lane, the rest smaller."""
    rng = np.random.default_rng(3)
    nb = a.size
    x = (rng.uniform(-1, 1, (nb, 32)) * 0.5).astype(np.float32) * a[:, None].astype(np.float32)
    lane = rng.integers(0, 32, nb)
    x[np.arange(nb), lane] = a * np.where(rng.random(nb) < 0.5, -1.0, 1.0).astype(np.float32)
    return x.reshape(-1)


def test_absmax_codes_ties_and_edges(bbc):
    """Block absmax at every code value, every half-step tie and its fp32 neighbours, just
    below each power of two, tiny and subnormal values, >= 32, and zero / NaN / inf blocks."""
    codes = oracle.e4m4_decode(np.arange(1, 256, dtype=np.uint8)).astype(np.float64)
    a = list(codes)
    for e in range(-14, 6):
        for m in range(16):
            t = np.float32(2.0 ** e * (1 + (m + 0.5) / 16))
            a += [t, np.nextafter(t, np.float32(0)), np.nextafter(t, np.float32(np.inf))]
        a.append(np.nextafter(np.float32(2.0 ** e), np.float32(0)))
    a += [3e-5, 2.0 ** -15, 2.0 ** -16 * 3, 1e-9, 1e-30, 32.0, 33.5, 64.0, 100.0, 1e6, 1e30]
    a = np.array(a, np.float32)
    a = a[np.isfinite(a) & (a > 0)]
    x = _blocks_with_absmax(a)
    x = np.concatenate([x, np.zeros(32, np.float32), np.full(32, np.nan, np.float32),
                        np.r_[np.float32(np.inf), np.ones(31, np.float32)]])
    for dt in (torch.float32, torch.bfloat16, torch.float16):
        xt = torch.from_numpy(x).to(dt)
        roundtrip(bbc, xt, 4, what=f"edges {dt}")
        roundtrip(bbc, xt, 5, what=f"edges {dt}")


@pytest.mark.parametrize("dt", ["f16", "bf16", "f32"])
def test_dequant_every_code(bbc, dt):
    """Random packed words with the absmax of block b set to code b % 256: all 256 codes decode."""
    K, nb = 5, 256 * 7 + 3
    n = nb * 32 - 11
    rng = np.random.default_rng(11)
    packed = rng.integers(0, 2 ** 32, nb * K, dtype=np.uint64).astype(np.uint32)
    am = (np.arange(nb) % 256).astype(np.uint8)
    cb_np = oracle.normal_float_codebook(K)
    ref = oracle.kbit_dequantize_e4m4(packed, am, cb_np, K, n, dt)
    y = bbc.kbit_dequantize_e4m4(torch.from_numpy(packed.view(np.int32)).cuda(), torch.from_numpy(am).cuda(),
                                 torch.from_numpy(cb_np).cuda(), K, n, DTYPES[dt])
    torch.cuda.synchronize()
    assert_bits_equal(to_host(y)[:n], ref, f"every code {dt}")


def test_packed_matches_fp32_absmax_path(bbc):
    """The E4M4 quantize writes exactly the fp32-absmax quantize's words."""
    x = synthetic.weights(1 << 20, std=0.02, seed=5, dtype=torch.bfloat16, device="cuda")
    cb = torch.from_numpy(oracle.normal_float_codebook(3)).cuda()
    p1, a1 = bbc.kbit_quantize(x, 3, cb)
    p2, a2 = bbc.kbit_quantize_e4m4(x, 3, cb)
    torch.cuda.synchronize()
    assert torch.equal(p1, p2)
    assert_bits_equal(to_host(a2), oracle.e4m4_encode(to_host(a1)), "encode of the fp32 absmax")


def test_dequant_long_stream_half_block_path(bbc):
    """A 16-bit output stream of at least 2^26 elements takes the half-block dequant form for K=4."""
    K, n = 4, (1 << 26) + 37
    nb = (n + 31) // 32
    rng = np.random.default_rng(23)
    packed = rng.integers(0, 2 ** 32, nb * K, dtype=np.uint64).astype(np.uint32)
    am = rng.integers(0, 256, nb, dtype=np.uint64).astype(np.uint8)
    cb_np = oracle.normal_float_codebook(K)
    ref = oracle.kbit_dequantize_e4m4(packed, am, cb_np, K, n, "bf16")
    y = bbc.kbit_dequantize_e4m4(torch.from_numpy(packed.view(np.int32)).cuda(), torch.from_numpy(am).cuda(),
                                 torch.from_numpy(cb_np).cuda(), K, n, torch.bfloat16)
    torch.cuda.synchronize()
    assert_bits_equal(to_host(y)[:n], ref, "long stream e4m4 K=4 bf16")
