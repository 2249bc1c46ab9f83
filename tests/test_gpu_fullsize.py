"""Parity at the full c5 size: the 16384 x 16384 bf16 tensor ~ N(0, 0.02) (seed 7, generated on
the device) that bench.py times, through the same calls on whole tensors, so every kernel runs
in the launch configuration the bench measures.

Every k-bit block depends only on its own 32 inputs and every nested inner group (256 outer
blocks of 64) only on its own state, so the oracle recomputes them in ranges: a seeded sample
(plus the first and the last) in the quick tests, and every block and group on all host cores in
the whole-tensor tests. Properties that hold at any size are also checked on the whole outputs
on the device. The nested quantize's offset depends on every outer block, so its whole state is
compared.
"""
import numpy as np
import pytest
import torch

import oracle
from blockwise_bit_codebook_b200 import synthetic
from tests.gpu_util import assert_bits_equal, to_host

pytestmark = pytest.mark.gpu
N = 16384 * 16384
NB = N // 32
BS = 64                                    # nested outer blocksize of the bench
GROUP = BS * 256                           # elements per nested inner group
NF4 = oracle.normal_float_codebook(4)
G8 = synthetic.general8_table()


@pytest.fixture(scope="module")
def bbc():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from blockwise_bit_codebook_b200 import build
    build.build()
    import blockwise_bit_codebook_b200 as m
    m.load_library()
    return m


@pytest.fixture(scope="module")
def x():
    return synthetic.weights(N, std=0.02, seed=7, dtype=torch.bfloat16, device="cuda")


def sample(count, total, seed):
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([[0, total - 1], rng.choice(total, count, replace=False)]))


@pytest.mark.parametrize("K", [3, 5])
def test_c5_kbit_sampled_blocks(bbc, x, K):
    cb = oracle.normal_float_codebook(K)
    cb_dev = torch.from_numpy(cb).cuda()
    packed, absmax = bbc.kbit_quantize(x, K, cb_dev)
    y = bbc.kbit_dequantize(packed, absmax, cb_dev, K, N, torch.bfloat16)
    torch.cuda.synchronize()

    blocks = sample(8192, NB, 100 + K)
    idx = torch.from_numpy(blocks).cuda()
    xb = to_host(x.view(NB, 32)[idx])
    ref_p, ref_a = oracle.kbit_quantize(xb.reshape(-1), "bf16", K, cb)
    assert_bits_equal(to_host(packed.view(NB, K)[idx]).reshape(-1), ref_p, f"c5 packed K={K}")
    assert_bits_equal(to_host(absmax[idx]), ref_a, f"c5 absmax K={K}")
    ref_y = oracle.kbit_dequantize(ref_p, ref_a, cb, K, blocks.size * 32, "bf16")
    assert_bits_equal(to_host(y.view(NB, 32)[idx]).reshape(-1), ref_y, f"c5 dequant K={K} bf16")

    # whole tensor: every block's absmax is its max |x|, and every reconstruction lies within
    # half the widest codebook gap of the block's scale (plus the bf16 rounding of the output)
    xf = x.float().view(NB, 32)
    assert torch.equal(xf.abs().amax(dim=1), absmax[:NB])
    half_gap = float(np.max(np.diff(cb))) / 2
    err = (y.float().view(NB, 32) - xf).abs().amax(dim=1)
    bound = absmax[:NB] * (half_gap * (1 + 2.0 ** -7)) + absmax[:NB] * 2.0 ** -8 + 1e-30
    assert bool((err <= bound).all()), f"K={K}: {int((err > bound).sum())} blocks outside the bound"


def test_c5_nested_dequant_sampled_groups(bbc):
    codes, q, a2, off = synthetic.nested_state(N, BS, seed=3, device="cuda")
    y = bbc.dequantize_4bit_nested(codes, q, torch.from_numpy(G8).cuda(), a2, float(off),
                                   torch.from_numpy(NF4).cuda(), N, BS, torch.bfloat16)
    torch.cuda.synchronize()
    ngroups = N // GROUP
    groups = sample(1024, ngroups, 7)
    idx = torch.from_numpy(groups).cuda()
    # whole inner groups concatenated form a valid nested state of their own
    codes_s = to_host(codes.view(ngroups, GROUP // 2)[idx]).reshape(-1)
    q_s = to_host(q.view(ngroups, 256)[idx]).reshape(-1)
    a2_s = to_host(a2[idx])
    ref = oracle.nested_dequantize(codes_s, q_s, G8, a2_s, float(off), NF4, groups.size * GROUP, BS, 256,
                                   "bf16")
    assert_bits_equal(to_host(y.view(ngroups, GROUP)[idx]).reshape(-1), ref, "c5 nested dequant bf16")


def test_c5_nested_quantize_whole_state(bbc, x):
    codes, q, a2, off = bbc.quantize_4bit_nested(x, BS, torch.from_numpy(NF4).cuda(), torch.from_numpy(G8).cuda())
    torch.cuda.synchronize()
    ref = oracle.quantize_4bit_nested(to_host(x), "bf16", BS, NF4, G8)
    assert_bits_equal(to_host(off), np.array([ref[3]], np.float32), "c5 nested offset")
    assert_bits_equal(to_host(a2)[:ref[2].size], ref[2], "c5 absmax2")
    assert_bits_equal(to_host(q)[:ref[1].size], ref[1], "c5 absmax_q")
    assert_bits_equal(to_host(codes)[:ref[0].size], ref[0], "c5 nested codes")


def _chunks(total, parts):
    step = -(-total // parts)
    return [(a, min(total, a + step)) for a in range(0, total, step)]


def _on_all_cores(fn, total):
    """fn(lo, hi) over contiguous ranges of [0, total) on every host core (the oracle's ctypes
    calls release the interpreter lock)."""
    import os
    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(max_workers=os.cpu_count() or 1) as ex:
        list(ex.map(lambda r: fn(*r), _chunks(total, 4 * (os.cpu_count() or 1))))


@pytest.mark.parametrize("K", [3, 5])
def test_c5_kbit_whole_tensor(bbc, x, K):
    """Every one of the 8,388,608 blocks of the c5 tensor, quantized and dequantized, against the
    oracle bit for bit (ranges of whole blocks on all host cores)."""
    cb = oracle.normal_float_codebook(K)
    cb_dev = torch.from_numpy(cb).cuda()
    packed, absmax = bbc.kbit_quantize(x, K, cb_dev)
    y = bbc.kbit_dequantize(packed, absmax, cb_dev, K, N, torch.bfloat16)
    torch.cuda.synchronize()
    xh = to_host(x)
    got_p, got_a, got_y = to_host(packed)[: NB * K], to_host(absmax)[:NB], to_host(y)[:N]
    bad = []

    def check(lo, hi):          # blocks [lo, hi)
        rp, ra = oracle.kbit_quantize(xh[lo * 32:hi * 32], "bf16", K, cb)
        ry = oracle.kbit_dequantize(rp, ra, cb, K, (hi - lo) * 32, "bf16")
        if not (np.array_equal(got_p[lo * K:hi * K], rp) and np.array_equal(got_a[lo:hi].view(np.uint32),
                                                                              ra.view(np.uint32))
                and np.array_equal(got_y[lo * 32:hi * 32], ry)):
            bad.append((lo, hi))
    _on_all_cores(check, NB)
    assert not bad, f"K={K}: block ranges differing from the oracle: {sorted(bad)[:4]}"


def test_c5_nested_dequant_whole_tensor(bbc):
    """Every inner group of the c5 nested state (16,384 groups of 256 outer blocks of 64) against
    the oracle bit for bit."""
    codes, q, a2, off = synthetic.nested_state(N, BS, seed=3, device="cuda")
    y = bbc.dequantize_4bit_nested(codes, q, torch.from_numpy(G8).cuda(), a2, float(off),
                                   torch.from_numpy(NF4).cuda(), N, BS, torch.bfloat16)
    torch.cuda.synchronize()
    ch, qh, a2h, got = to_host(codes), to_host(q), to_host(a2), to_host(y)[:N]
    ngroups = N // GROUP
    bad = []

    def check(lo, hi):          # inner groups [lo, hi)
        ref = oracle.nested_dequantize(ch[lo * GROUP // 2:hi * GROUP // 2], qh[lo * 256:hi * 256], G8, a2h[lo:hi],
                                       float(off), NF4, (hi - lo) * GROUP, BS, 256, "bf16")
        if not np.array_equal(got[lo * GROUP:hi * GROUP], ref):
            bad.append((lo, hi))
    _on_all_cores(check, ngroups)
    assert not bad, f"group ranges differing from the oracle: {sorted(bad)[:4]}"
