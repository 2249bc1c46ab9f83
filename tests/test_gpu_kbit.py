"""GPU parity of k-bit quantize / dequantize against the oracle (bit-exact).

All calls go through the C ABI (libbbc.so via the ctypes binding). Inputs are
seeded synthetic tensors generated on the host and copied to the device; the
oracle runs on the same host values.
"""
import numpy as np
import pytest
import torch

import oracle
from blockwise_bit_codebook_b200 import synthetic
from tests.gpu_util import DTYPES, assert_bits_equal, f32_key, float_keys_to_f32, to_host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bbc():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from blockwise_bit_codebook_b200 import build
    build.build()
    import blockwise_bit_codebook_b200 as m
    m.load_library()
    return m


def gpu_quantize(bbc, x_dev, K, cb_np):
    n = x_dev.numel()
    nb = (n + 31) // 32
    cb = torch.from_numpy(np.ascontiguousarray(cb_np, np.float32)).cuda()
    packed, absmax = bbc.kbit_quantize(x_dev, K, cb)
    torch.cuda.synchronize()
    return to_host(packed)[: nb * K], to_host(absmax)[:nb]


def check_quantize(bbc, x_host: torch.Tensor, K, cb_np, x_dev=None, what=""):
    dt = {torch.float16: "f16", torch.bfloat16: "bf16", torch.float32: "f32"}[x_host.dtype]
    ref_p, ref_a = oracle.kbit_quantize(to_host(x_host), dt, K, cb_np)
    got_p, got_a = gpu_quantize(bbc, x_host.cuda() if x_dev is None else x_dev, K, cb_np)
    assert_bits_equal(got_a, ref_a, f"absmax {what}")
    assert_bits_equal(got_p, ref_p, f"packed {what}")
    return ref_p, ref_a


def gpu_dequantize(bbc, packed_np, absmax_np, cb_np, K, n, dtype, out=None):
    p = torch.from_numpy(packed_np.view(np.int32).copy()).cuda()
    a = torch.from_numpy(absmax_np.copy()).cuda()
    cb = torch.from_numpy(np.ascontiguousarray(cb_np, np.float32)).cuda()
    y = bbc.kbit_dequantize(p, a, cb, K, n, dtype, out=out)
    torch.cuda.synchronize()
    return y


def check_dequantize(bbc, packed_np, absmax_np, cb_np, K, n, dtname, what=""):
    ref = oracle.kbit_dequantize(packed_np, absmax_np, cb_np, K, n, dtname)
    y = gpu_dequantize(bbc, packed_np, absmax_np, cb_np, K, n, DTYPES[dtname])
    assert_bits_equal(to_host(y)[:n], ref, f"dequant {what} {dtname}")


# ---------------------------------------------------------------- workloads

def test_c1_roundtrip_k4_fp32(bbc):
    """1,048,576 fp32 values ~ N(0,1) from seed 0, K=4, normal-float codebook."""
    x = synthetic.weights(1 << 20, std=1.0, seed=0)
    cb = oracle.normal_float_codebook(4)
    p, a = check_quantize(bbc, x, 4, cb, what="C1")
    check_dequantize(bbc, p, a, cb, 4, x.numel(), "f32", "C1")


@pytest.mark.parametrize("K", [2, 3, 4, 5])
@pytest.mark.parametrize("dt", ["f16", "bf16", "f32"])
def test_c2_sweep(bbc, K, dt):
    """4096x4096 ~ N(0, 0.02), 0.1% of entries x20, quantize then dequantize."""
    x = synthetic.weights(4096 * 4096, std=0.02, seed=1, dtype=DTYPES[dt], outlier_frac=0.001,
                          outlier_seed=2)
    cb = oracle.normal_float_codebook(K)
    p, a = check_quantize(bbc, x, K, cb, what=f"C2 K{K} {dt}")
    check_dequantize(bbc, p, a, cb, K, x.numel(), dt, f"C2 K{K}")


# ---------------------------------------------------------------- sizes, alignment

SIZES = [1, 7, 8, 9, 31, 32, 33, 37, 63, 64, 65, 255, 256, 257, 1000, 4097, 100003, 8 * 4096 + 5]


@pytest.mark.parametrize("dt", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("K", [2, 3, 5])
def test_ragged_sizes(bbc, dt, K):
    cb = oracle.normal_float_codebook(K)
    for n in SIZES:
        x = synthetic.weights(n, seed=n, dtype=DTYPES[dt])
        p, a = check_quantize(bbc, x, K, cb, what=f"n={n}")
        check_dequantize(bbc, p, a, cb, K, n, dt, f"n={n}")


@pytest.mark.parametrize("dt", ["f16", "bf16", "f32"])
def test_unaligned_pointers_take_scalar_path(bbc, dt):
    """Buffers offset by one element (not 16-byte aligned) give identical results."""
    K = 4
    cb = oracle.normal_float_codebook(K)
    n = 32 * 1000 + 13
    x = synthetic.weights(n + 1, seed=5, dtype=DTYPES[dt])
    xd = x.cuda()[1:]
    assert xd.data_ptr() % 16 != 0
    p, a = check_quantize(bbc, x[1:].contiguous(), K, cb, x_dev=xd, what="unaligned")
    out = torch.empty(n + 1, dtype=DTYPES[dt], device="cuda")[1:]
    y = gpu_dequantize(bbc, p, a, cb, K, n, DTYPES[dt], out=out)
    assert_bits_equal(to_host(y), oracle.kbit_dequantize(p, a, cb, K, n, dt), f"unaligned dequant {dt}")


@pytest.mark.parametrize("K", [2, 3, 4, 5])
@pytest.mark.parametrize("dt", ["f16", "bf16"])
def test_whole_block_path_with_word_aligned_outputs(bbc, K, dt):
    """Aligned 16-bit input (one block per thread) writing packed words and absmax that are
    only 4-byte aligned: the vector stores must fall back, results identical."""
    cb = oracle.normal_float_codebook(K)
    n = 32 * 1024 * 3 + 32 * 5 + 9          # many warp iterations, a partial one, a ragged block
    nb = (n + 31) // 32
    x = synthetic.weights(n, std=0.02, seed=40 + K, dtype=DTYPES[dt], outlier_frac=0.001)
    ref_p, ref_a = oracle.kbit_quantize(to_host(x), dt, K, cb)
    pbuf = torch.zeros(nb * K + 4, dtype=torch.int32, device="cuda")
    abuf = torch.zeros(nb + 4, dtype=torch.float32, device="cuda")
    packed, absmax = pbuf[1:1 + nb * K], abuf[1:1 + nb]
    assert packed.data_ptr() % 8 == 4
    bbc.kbit_quantize(x.cuda(), K, torch.from_numpy(cb).cuda(), absmax=absmax, packed=packed)
    torch.cuda.synchronize()
    assert_bits_equal(to_host(absmax), ref_a, "absmax, word-aligned output")
    assert_bits_equal(to_host(packed), ref_p, "packed, word-aligned output")
    assert int(pbuf[0]) == 0 and int(pbuf[-3:].abs().sum()) == 0


@pytest.mark.parametrize("K", [2, 3, 4, 5])
@pytest.mark.parametrize("dt", ["f16", "bf16", "f32"])
def test_dequant_whole_blocks_with_word_aligned_packed(bbc, K, dt):
    """Aligned output (one block per thread) reading packed words that are only 4-byte
    aligned: the vector word loads must fall back, results identical."""
    rng = np.random.default_rng(60 + K)
    n = 32 * 4096 + 32 * 3 + 21
    nb = (n + 31) // 32
    cb = oracle.normal_float_codebook(K)
    packed = rng.integers(0, 2 ** 32, nb * K, dtype=np.uint64).astype(np.uint32)
    absmax = rng.uniform(0, 3, nb).astype(np.float32)
    ref = oracle.kbit_dequantize(packed, absmax, cb, K, n, dt)
    buf = torch.zeros(nb * K + 1, dtype=torch.int32, device="cuda")
    buf[1:] = torch.from_numpy(packed.view(np.int32)).cuda()
    assert buf[1:].data_ptr() % 8 == 4
    y = bbc.kbit_dequantize(buf[1:], torch.from_numpy(absmax).cuda(), torch.from_numpy(cb).cuda(), K, n,
                            DTYPES[dt])
    torch.cuda.synchronize()
    assert_bits_equal(to_host(y)[:n], ref, f"dequant word-aligned packed K={K} {dt}")


# ---------------------------------------------------------------- exactness corners

def exact_thresholds(cb):
    """T_j: smallest fp32 value whose nearest entry (oracle rule) is >= j; by bisection."""
    T = []
    for j in range(1, cb.size):
        lo, hi = f32_key(-4.0), f32_key(4.0)
        while hi - lo > 1:
            mid = (lo + hi) // 2
            v = float(float_keys_to_f32(np.array([mid]))[0])
            if oracle.nearest_entry(v, cb) >= j:
                hi = mid
            else:
                lo = mid
        T.append(float(float_keys_to_f32(np.array([hi]))[0]))
    return np.array(T, np.float32)


def threshold_blocks(cb, scales, ulps=4):
    """Blocks whose quotients land on every threshold and its fp32 neighbours, for several d."""
    T = exact_thresholds(cb)
    vals = []
    for d in scales:
        d = np.float32(d)
        targets = []
        for t in T:
            k = f32_key(t)
            targets += list(float_keys_to_f32(np.arange(k - ulps, k + ulps + 1)))
        xs = []
        for tq in targets:
            x = np.float32(tq) * d
            for _ in range(8):      # walk x until x / d rounds to the target (IEEE fp32 division)
                q = np.float32(x) / d
                if q == tq:
                    break
                x = np.nextafter(np.float32(x), np.float32(np.inf) if q < tq else np.float32(-np.inf))
            if abs(x) < d:
                xs.append(np.float32(x))
        for i in range(0, len(xs), 31):      # each block: 31 probes plus the absmax itself
            blk = [d] + xs[i:i + 31]
            blk += [np.float32(0.0)] * (32 - len(blk))
            vals += blk
    return np.array(vals, np.float32)


@pytest.mark.parametrize("K", [2, 3, 4, 5])
def test_quotients_on_thresholds(bbc, K):
    cb = oracle.normal_float_codebook(K)
    x = threshold_blocks(cb, [1.0, 0.7373, 3.25e-3, 1234.5, 1e-8, 2.0 ** -20])
    check_quantize(bbc, torch.from_numpy(x), K, cb, what=f"thresholds K{K}")


@pytest.mark.parametrize("K", [2, 3, 4, 5])
@pytest.mark.parametrize("dt", ["bf16", "f16"])
def test_every_16bit_quotient_for_several_absmax(bbc, K, dt):
    """Every value of the 16-bit type in [-d, d] as a numerator, for several block maxima d (the
    block's first element): all quotients these d can produce, those on and beside every
    threshold included. The length is whole warp iterations of 32 blocks, so the aligned
    one-block-per-thread path (8-byte table, sign-bit increment) decides all of them."""
    cb = oracle.normal_float_codebook(K)
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    widen = oracle.bf16_bits_to_f32 if dt == "bf16" else oracle.f16_bits_to_f32
    narrow = oracle.f32_to_bf16_bits if dt == "bf16" else oracle.f32_to_f16_bits
    vals = widen(bits)
    blocks = []
    for d_req in (1.0, 0.7373, 3.25e-3, 1234.5):
        d_bits = narrow(np.array([d_req], np.float32))[0]
        d = widen(np.array([d_bits], np.uint16))[0]
        xs = bits[np.isfinite(vals) & (np.abs(vals) <= d)]
        for i in range(0, xs.size, 31):
            blk = np.zeros(32, np.uint16)
            blk[0] = d_bits
            blk[1:1 + xs[i:i + 31].size] = xs[i:i + 31]
            blocks.append(blk)
    while len(blocks) % 32:
        blocks.append(np.zeros(32, np.uint16))
    x = np.concatenate(blocks)
    xt = torch.from_numpy(x.view(np.int16)).view(DTYPES[dt])
    check_quantize(bbc, xt, K, cb, what=f"every {dt} quotient K{K}")


def test_quotients_on_thresholds_wide_codebook(bbc):
    """Thresholds beyond [-1, 1] and a codebook not symmetric about zero."""
    cb = np.array([-3.0, -1.7, -0.9, -0.2, 0.05, 0.4, 1.1, 2.5], np.float32)
    x = threshold_blocks(cb, [1.0, 0.31])
    check_quantize(bbc, torch.from_numpy(x), 3, cb, what="wide codebook")


def test_special_values_fp32(bbc):
    rng = np.random.default_rng(8)
    blocks = [
        np.zeros(32), -np.zeros(32),
        rng.uniform(-1e-9, 1e-9, 32),                       # under the 1e-8 clamp
        np.r_[1.0, rng.standard_normal(31) * 1e-39],        # subnormal quotients
        rng.standard_normal(32) * 1e-41,                    # subnormal inputs and absmax
        rng.standard_normal(32) * 1e37,                     # 1/d near the subnormal range
        np.r_[3e38, -3.3e38, rng.standard_normal(30)],
        np.r_[np.inf, rng.standard_normal(31)],
        np.r_[-np.inf, np.inf, rng.standard_normal(30)],
        np.r_[np.nan, rng.standard_normal(31)],
        np.full(32, np.nan),
        np.r_[np.nan, np.inf, np.zeros(30)],
        rng.standard_normal(32),
    ]
    x = np.concatenate([np.asarray(b, np.float64) for b in blocks]).astype(np.float32)
    for K in (2, 3, 4, 5):
        check_quantize(bbc, torch.from_numpy(x), K, oracle.normal_float_codebook(K), what=f"special K{K}")


@pytest.mark.parametrize("dt", ["f16", "bf16"])
def test_special_values_half(bbc, dt):
    rng = np.random.default_rng(9)
    x = np.concatenate([
        np.zeros(32), rng.standard_normal(32) * 1e-6, np.r_[np.inf, rng.standard_normal(31)],
        np.r_[np.nan, rng.standard_normal(31)], rng.standard_normal(32) * 6e4 if dt == "f16"
        else rng.standard_normal(32) * 1e38, rng.standard_normal(64)]).astype(np.float32)
    xt = torch.from_numpy(x).to(DTYPES[dt])
    for K in (2, 5):
        check_quantize(bbc, xt, K, oracle.normal_float_codebook(K), what=f"special {dt} K{K}")


PATHOLOGICAL = {
    "unsorted": lambda: np.random.default_rng(1).permutation(oracle.normal_float_codebook(4)),
    "duplicates": lambda: np.array([-1, -.5, -.5, -.25, 0, 0, .1, .2, .3, .3, .4, .5, .6, .7, .9, 1], np.float32),
    "tiny_gaps": lambda: np.linspace(-1e-6, 1e-6, 16).astype(np.float32),
    "near_tie": lambda: np.r_[0.0, 1e-9, np.linspace(0.1, 1, 14)].astype(np.float32),
    "nan_entry": lambda: np.r_[np.nan, oracle.normal_float_codebook(4)[1:]].astype(np.float32),
    "inf_entry": lambda: np.r_[oracle.normal_float_codebook(4)[:-1], np.inf].astype(np.float32),
    "all_zero": lambda: np.zeros(16, np.float32),
    "descending": lambda: oracle.normal_float_codebook(4)[::-1].copy(),
}


@pytest.mark.parametrize("name", sorted(PATHOLOGICAL))
def test_pathological_codebooks(bbc, name):
    cb = PATHOLOGICAL[name]()
    x = synthetic.weights(32 * 300 + 9, seed=4)
    check_quantize(bbc, x, 4, cb, what=name)
    xb = threshold_blocks(oracle.normal_float_codebook(4), [0.5], ulps=2)
    check_quantize(bbc, torch.from_numpy(xb), 4, cb, what=name + " probes")


@pytest.mark.parametrize("K", [2, 3, 4, 5])
@pytest.mark.parametrize("dt", ["f16", "bf16", "f32"])
def test_dequant_random_state(bbc, K, dt):
    """Arbitrary words and absmax values, including zeros, subnormals, overflow, inf and NaN."""
    rng = np.random.default_rng(100 * K + len(dt))
    n = 32 * 5000 + 17
    nb = (n + 31) // 32
    packed = rng.integers(0, 2**32, nb * K, dtype=np.uint64).astype(np.uint32)
    absmax = rng.uniform(0, 3, nb).astype(np.float32)
    specials = np.array([0.0, -0.0, 1e-45, 1e-40, 7e4, 1e30, 3.4e38, np.inf, np.nan, 1.0], np.float32)
    absmax[: specials.size] = specials
    cb = oracle.normal_float_codebook(K)
    check_dequantize(bbc, packed, absmax, cb, K, n, dt, f"random K{K}")


@pytest.mark.parametrize("K", [2, 3, 4])
def test_dequant_long_stream_half_block_path(bbc, K):
    """16-bit outputs of at least 2^26 elements take the half-block path (K <= 4); an odd length
    ends in a ragged half block."""
    rng = np.random.default_rng(7 + K)
    n = (1 << 26) + 37
    nb = (n + 31) // 32
    packed = rng.integers(0, 2**32, nb * K, dtype=np.uint64).astype(np.uint32)
    absmax = rng.uniform(0.01, 0.1, nb).astype(np.float32)
    cb = oracle.normal_float_codebook(K)
    check_dequantize(bbc, packed, absmax, cb, K, n, "bf16", f"long K{K}")


# ---------------------------------------------------------------- contract

def test_no_writes_beyond_outputs_and_inputs_unchanged(bbc):
    K, n = 5, 32 * 77 + 3
    nb = (n + 31) // 32
    x = synthetic.weights(n, seed=12, dtype=torch.bfloat16).cuda()
    x_before = x.clone()
    cb = torch.from_numpy(oracle.normal_float_codebook(K)).cuda()
    cb_before = cb.clone()
    packed = torch.full((nb * K + 64,), 0x5A5A5A5A, dtype=torch.int32, device="cuda")
    absmax = torch.full((nb + 64,), 12345.0, dtype=torch.float32, device="cuda")
    bbc.kbit_quantize(x, K, cb, absmax=absmax, packed=packed)
    out = torch.full((n + 64,), 7.0, dtype=torch.bfloat16, device="cuda")
    bbc.kbit_dequantize(packed, absmax, cb, K, n, torch.bfloat16, out=out)
    torch.cuda.synchronize()
    assert torch.all(packed[nb * K:] == 0x5A5A5A5A)
    assert torch.all(absmax[nb:] == 12345.0)
    assert torch.all(out[n:] == 7.0)
    assert torch.equal(x, x_before) and torch.equal(cb, cb_before)


def test_runs_on_given_stream(bbc):
    K = 3
    cb_np = oracle.normal_float_codebook(K)
    x = synthetic.weights(1 << 16, seed=13)
    s = torch.cuda.Stream()
    xd = x.cuda()
    cb = torch.from_numpy(cb_np).cuda()
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        packed, absmax = bbc.kbit_quantize(xd, K, cb, stream=s)
        y = bbc.kbit_dequantize(packed, absmax, cb, K, xd.numel(), torch.float32, stream=s)
    s.synchronize()
    rp, ra = oracle.kbit_quantize(to_host(x), "f32", K, cb_np)
    assert_bits_equal(to_host(packed), rp, "stream packed")
    assert_bits_equal(to_host(y), oracle.kbit_dequantize(rp, ra, cb_np, K, x.numel(), "f32"), "stream out")


def test_invalid_arguments_raise(bbc):
    from blockwise_bit_codebook_b200 import BBCError
    x = torch.zeros(64, device="cuda")
    cb = torch.zeros(16, device="cuda")
    with pytest.raises(BBCError, match="K must be 2..5"):
        bbc.kbit_quantize(x, 6, cb)
    with pytest.raises(BBCError, match="blocksize must be 32"):
        bbc.kbit_quantize(x, 4, cb, blocksize=64)
    with pytest.raises(BBCError):
        bbc.kbit_dequantize(torch.zeros(8, dtype=torch.int32, device="cuda"), x, cb, 4, 0, torch.float32)
