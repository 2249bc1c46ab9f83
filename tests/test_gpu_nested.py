"""GPU parity of the fused nested 4-bit dequant against the oracle (bit-exact)."""
import numpy as np
import pytest
import torch

import oracle
from blockwise_bit_codebook_b200 import synthetic
from tests.gpu_util import DTYPES, assert_bits_equal, to_host
from tests.test_oracle_nested import find_nofma_triples

pytestmark = pytest.mark.gpu

NF4 = None


@pytest.fixture(scope="module")
def bbc():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from blockwise_bit_codebook_b200 import build
    build.build()
    import blockwise_bit_codebook_b200 as m
    m.load_library()
    return m


def tables(fmt):
    code4 = oracle.normal_float_codebook(4) if fmt == "nf4" else synthetic.fp4_table()
    return synthetic.general8_table(), code4


def run_both(bbc, n, bs, dt, fmt, seed=3, all_codes=False, device_gen="cpu", out=None, codes_dev=None):
    codes, q, a2, off = synthetic.nested_state(n, bs, seed=seed, device=device_gen, all_codes=all_codes)
    code2, code4 = tables(fmt)
    ref = oracle.nested_dequantize(to_host(codes), to_host(q), code2, to_host(a2), float(off), code4,
                                   n, bs, 256, dt)
    y = bbc.dequantize_4bit_nested(codes.cuda() if codes_dev is None else codes_dev, q.cuda(),
                                   torch.from_numpy(code2).cuda(), a2.cuda(), float(off),
                                   torch.from_numpy(code4).cuda(), n, bs, DTYPES[dt], out=out)
    torch.cuda.synchronize()
    assert_bits_equal(to_host(y)[:n], ref, f"nested n={n} bs={bs} {fmt} {dt}")
    return y


@pytest.mark.parametrize("dt", ["f16", "bf16", "f32"])
def test_c3_nf4_4096x11008(bbc, dt):
    run_both(bbc, 4096 * 11008, 64, dt, "nf4")


@pytest.mark.parametrize("fmt", ["nf4", "fp4"])
@pytest.mark.parametrize("bs", [32, 64, 128, 256, 1024, 4096])
@pytest.mark.parametrize("dt", ["f16", "bf16", "f32"])
def test_c4_matrix_reduced(bbc, fmt, bs, dt):
    """The C4 case matrix at a size the oracle runs in well under a second: three full
    inner groups at bs=4096 plus a tail of 37 elements; every General8 code occurs."""
    n = 3 * 4096 * 256 + 37
    run_both(bbc, n, bs, dt, fmt, seed=bs, all_codes=True)


@pytest.mark.parametrize("bs", [32, 64, 128, 256, 1024, 4096])
def test_c4_full_size_odd(bbc, bs):
    """The whole C4 matrix at its own size, 8192*8192 + 37 elements (a partial last outer block
    and inner group): both value tables and all three output types, every General8 code present."""
    n = 8192 * 8192 + 37
    codes, q, a2, off = synthetic.nested_state(n, bs, seed=11, device="cuda", all_codes=True)
    hc, hq, ha2 = to_host(codes), to_host(q), to_host(a2)
    out = {dt: torch.empty(n, dtype=DTYPES[dt], device="cuda") for dt in ("f16", "bf16", "f32")}
    for fmt in ("nf4", "fp4"):
        code2, code4 = tables(fmt)
        c2d, c4d = torch.from_numpy(code2).cuda(), torch.from_numpy(code4).cuda()
        for dt in ("f16", "bf16", "f32"):
            ref = oracle.nested_dequantize(hc, hq, code2, ha2, float(off), code4, n, bs, 256, dt)
            y = bbc.dequantize_4bit_nested(codes, q, c2d, a2, float(off), c4d, n, bs, DTYPES[dt], out=out[dt])
            torch.cuda.synchronize()
            assert_bits_equal(to_host(y), ref, f"nested full-size odd n bs={bs} {fmt} {dt}")


@pytest.mark.parametrize("dt", ["f16", "bf16", "f32"])
def test_ragged_sizes(bbc, dt):
    for n in [1, 2, 3, 15, 16, 17, 31, 33, 63, 64, 65, 127, 1000, 4097, 65537, 256 * 64 * 2 + 3]:
        for bs in (32, 64, 4096):
            run_both(bbc, n, bs, dt, "nf4", seed=n + bs)


@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_unaligned_pointers(bbc, dt):
    n, bs = 64 * 300 + 5, 64
    codes, q, a2, off = synthetic.nested_state(n, bs, seed=21)
    code2, code4 = tables("nf4")
    ref = oracle.nested_dequantize(to_host(codes), to_host(q), code2, to_host(a2), float(off), code4,
                                   n, bs, 256, dt)
    cbig = torch.zeros(codes.numel() + 1, dtype=torch.uint8, device="cuda")
    cbig[1:] = codes.cuda()
    out = torch.empty(n + 1, dtype=DTYPES[dt], device="cuda")[1:]
    y = bbc.dequantize_4bit_nested(cbig[1:], q.cuda(), torch.from_numpy(code2).cuda(), a2.cuda(),
                                   float(off), torch.from_numpy(code4).cuda(), n, bs, DTYPES[dt], out=out)
    torch.cuda.synchronize()
    assert_bits_equal(to_host(y), ref, f"unaligned nested {dt}")


@pytest.mark.parametrize("dt", ["f16", "bf16", "f32"])
def test_every_code_pair_and_offsets(bbc, dt):
    """All 256 General8 codes x all 16 value codes, for several inner absmax / offset values."""
    bs = 32
    code2, code4 = tables("nf4")
    codes = np.tile(np.arange(256, dtype=np.uint8), 16)        # 16 bytes per block of 32
    q = np.arange(256, dtype=np.uint8)
    n = 256 * bs
    for a2, off in [(1.0, 0.0), (0.0371, 0.0), (0.0523, 0.0312), (3.5, -0.75), (1e-30, 1e-38)]:
        a2v = np.array([a2], np.float32)
        ref = oracle.nested_dequantize(codes, q, code2, a2v, float(np.float32(off)), code4, n, bs, 256, dt)
        y = bbc.dequantize_4bit_nested(torch.from_numpy(codes).cuda(), torch.from_numpy(q).cuda(),
                                       torch.from_numpy(code2).cuda(), torch.from_numpy(a2v).cuda(),
                                       float(np.float32(off)), torch.from_numpy(code4).cuda(), n, bs,
                                       DTYPES[dt])
        torch.cuda.synchronize()
        assert_bits_equal(to_host(y), ref, f"code sweep {a2} {off} {dt}")


def test_scale_is_not_fused(bbc):
    """Triples where fma(a, b, c) differs from fl(fl(a*b)+c): the kernel must give the latter."""
    for a, b, c, two, fused in find_nofma_triples(16, seed=5):
        code2 = np.full(256, a, np.float32)
        y = bbc.dequantize_4bit_nested(torch.zeros(16, dtype=torch.uint8, device="cuda"),
                                       torch.zeros(1, dtype=torch.uint8, device="cuda"),
                                       torch.from_numpy(code2).cuda(),
                                       torch.tensor([b], dtype=torch.float32, device="cuda"), float(c),
                                       torch.ones(16, dtype=torch.float32, device="cuda"), 32, 32,
                                       torch.float32)
        torch.cuda.synchronize()
        got = y.cpu().numpy()
        assert np.all(got == two) and np.all(got != fused)


def test_no_writes_beyond_n_and_inputs_unchanged(bbc):
    n, bs = 64 * 100 + 7, 64
    codes, q, a2, off = synthetic.nested_state(n, bs, seed=31)
    code2, code4 = tables("fp4")
    cd, qd, a2d = codes.cuda(), q.cuda(), a2.cuda()
    c2d, c4d = torch.from_numpy(code2).cuda(), torch.from_numpy(code4).cuda()
    before = [t.clone() for t in (cd, qd, a2d, c2d, c4d)]
    out = torch.full((n + 40,), -3.0, dtype=torch.float16, device="cuda")
    bbc.dequantize_4bit_nested(cd, qd, c2d, a2d, float(off), c4d, n, bs, torch.float16, out=out)
    torch.cuda.synchronize()
    assert torch.all(out[n:] == -3.0)
    for t, b in zip((cd, qd, a2d, c2d, c4d), before):
        assert torch.equal(t, b)


def test_invalid_arguments_raise(bbc):
    from blockwise_bit_codebook_b200 import BBCError
    z8 = torch.zeros(64, dtype=torch.uint8, device="cuda")
    f = torch.zeros(256, device="cuda")
    with pytest.raises(BBCError, match="power of two"):
        bbc.dequantize_4bit_nested(z8, z8, f, f, 0.0, f, 64, 48, torch.float16)
    with pytest.raises(BBCError, match="blocksize2"):
        bbc.dequantize_4bit_nested(z8, z8, f, f, 0.0, f, 64, 64, torch.float16, blocksize2=128)


@pytest.mark.parametrize("fmt", ["nf4", "fp4"])
@pytest.mark.parametrize("dt", ["f16", "bf16", "f32"])
def test_chain_equals_fused_and_oracle(bbc, fmt, dt):
    """The unfused three-launch chain gives the fused kernel's bits and the oracle's."""
    for n, bs in [(4096 * 4096, 64), (3 * 4096 * 256 + 37, 4096), (64 * 300 + 5, 32)]:
        codes, q, a2, off = synthetic.nested_state(n, bs, seed=n % 1000 + bs, all_codes=True)
        code2, code4 = tables(fmt)
        args = (codes.cuda(), q.cuda(), torch.from_numpy(code2).cuda(), a2.cuda(), float(off),
                torch.from_numpy(code4).cuda(), n, bs, DTYPES[dt])
        ws = torch.full(((n + bs - 1) // bs,), float("nan"), dtype=torch.float32, device="cuda")
        y_chain = bbc.dequantize_4bit_nested_chain(*args, scale_workspace=ws)
        y_fused = bbc.dequantize_4bit_nested(*args)
        torch.cuda.synchronize()
        ref = oracle.nested_dequantize(to_host(codes), to_host(q), code2, to_host(a2), float(off), code4,
                                       n, bs, 256, dt)
        assert_bits_equal(to_host(y_chain)[:n], ref, f"chain n={n} {fmt} {dt}")
        assert_bits_equal(to_host(y_fused)[:n], to_host(y_chain)[:n], f"fused vs chain {dt}")
        # the workspace holds exactly the separately rounded scales
        qn, a2n = to_host(q), to_host(a2)
        sample = np.unique(np.r_[0, 1, (n - 1) // bs, np.random.default_rng(0).integers(0, (n - 1) // bs + 1, 64)])
        want = np.array([oracle.nested_scale(float(code2[qn[b]]), float(a2n[b // 256]), float(off))
                         for b in sample], np.float32)
        assert_bits_equal(to_host(ws)[sample], want, "chain scales")


@pytest.mark.parametrize("dt", ["f16", "bf16", "f32"])
def test_plain_4bit_parity(bbc, dt):
    rng = np.random.default_rng(41)
    code4 = synthetic.fp4_table()
    for n in [1, 3, 31, 32, 33, 1000, 65537, 4096 * 1024 + 7]:
        for bs in (32, 64, 256, 4096):
            nb = (n + bs - 1) // bs
            codes = torch.from_numpy(rng.integers(0, 256, (n + 1) // 2, dtype=np.uint8))
            am = rng.uniform(0, 2, nb).astype(np.float32)
            am[:3] = [0.0, 1e-40, 7e4][: min(3, nb)]
            ref = oracle.dequantize_4bit(codes.numpy(), am, code4, n, bs, dt)
            y = bbc.dequantize_4bit(codes.cuda(), torch.from_numpy(am).cuda(),
                                    torch.from_numpy(code4).cuda(), n, bs, DTYPES[dt])
            torch.cuda.synchronize()
            assert_bits_equal(to_host(y)[:n], ref, f"plain 4-bit n={n} bs={bs} {dt}")


def test_chain_invalid_arguments(bbc):
    from blockwise_bit_codebook_b200 import BBCError
    z8 = torch.zeros(64, dtype=torch.uint8, device="cuda")
    f = torch.zeros(256, device="cuda")
    with pytest.raises(BBCError, match="null pointer"):
        import ctypes as ct
        L = bbc.load_library()
        st = L.dequantize_4bit_nested_chain(ct.c_void_p(z8.data_ptr()), ct.c_void_p(z8.data_ptr()),
                                            ct.c_void_p(f.data_ptr()), ct.c_void_p(f.data_ptr()),
                                            ct.c_float(0.0), ct.c_void_p(f.data_ptr()), 64, 64, 256, 1,
                                            ct.c_void_p(f.data_ptr()), None, None)
        bbc._native._check("dequantize_4bit_nested_chain", st)
    with pytest.raises(BBCError, match="power of two"):
        bbc.dequantize_4bit(z8, f, f, 64, 100, torch.float16)
