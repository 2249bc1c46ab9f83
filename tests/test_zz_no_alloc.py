"""The allocation-free chain entry point (static scratch) against the workspace chain and the
oracle.

Named so that pytest collects it last: it must pass both in a fresh process and after every
other test has run in the same process.
"""
import ctypes as ct

import numpy as np
import pytest
import torch

import oracle
from blockwise_bit_codebook_b200 import synthetic
from tests.gpu_util import DTYPES, assert_bits_equal, to_host

SCRATCH_FLOATS = 1048576     # BBC_NOALLOC_SCRATCH_FLOATS in include/bbc.h


@pytest.fixture(scope="module")
def bbc():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from blockwise_bit_codebook_b200 import build
    build.build()
    import blockwise_bit_codebook_b200 as m
    m.load_library()
    return m


def _p(t):
    return ct.c_void_p(t.data_ptr())


def _free_bytes():
    free, _ = torch.cuda.mem_get_info()
    return free


def _cases():
    # (n, blocksize, fmt, dtype, seed): the first fills the scratch to its limit, the second is
    # ragged and smaller, so it runs over scales the first call left behind.
    return [(SCRATCH_FLOATS * 64, 64, "nf4", "bf16", 5), (3 * 4096 * 256 + 37, 4096, "fp4", "f16", 9)]


@pytest.mark.gpu
def test_noalloc_matches_workspace_chain_two_calls(bbc):
    L = bbc.load_library()
    code2 = torch.from_numpy(synthetic.general8_table()).cuda()
    for call, (n, bs, fmt, dt, seed) in enumerate(_cases()):
        codes, q, a2, off = synthetic.nested_state(n, bs, seed=seed, device="cuda", all_codes=True)
        code4_np = oracle.normal_float_codebook(4) if fmt == "nf4" else synthetic.fp4_table()
        code4 = torch.from_numpy(code4_np).cuda()
        want = bbc.dequantize_4bit_nested_chain(codes, q, code2, a2, float(off), code4, n, bs, DTYPES[dt])
        out = torch.full((n,), float("nan"), dtype=DTYPES[dt], device="cuda")
        torch.cuda.synchronize()
        before, free_before = torch.cuda.memory_allocated(), _free_bytes()
        st = L.dequantize_4bit_nested_chain_noalloc(_p(codes), _p(q), _p(code2), _p(a2), ct.c_float(float(off)),
                                                    _p(code4), n, bs, 256, int(bbc.BBC_F16 if dt == "f16" else
                                                                              bbc.BBC_BF16), _p(out),
                                                    ct.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == 0, bbc.bbc_last_error()
        torch.cuda.synchronize()
        # nothing allocated: neither through torch's allocator nor on the device at all (the
        # driver's free-memory figure is unchanged by the call)
        assert torch.cuda.memory_allocated() == before
        assert _free_bytes() >= free_before
        assert_bits_equal(to_host(out), to_host(want)[:n], f"no-alloc chain, call {call + 1}")
        if n < 1 << 24:
            # the small ragged case also against the oracle, bit for bit
            ref = oracle.nested_dequantize(to_host(codes), to_host(q), synthetic.general8_table(), to_host(a2),
                                           float(off), code4_np, n, bs, 256, dt)
            assert_bits_equal(to_host(out), ref, f"no-alloc chain vs oracle, call {call + 1} {dt}")
        del codes, q, a2, want, out


@pytest.mark.gpu
def test_noalloc_oversize_rejected(bbc):
    from blockwise_bit_codebook_b200 import BBCError
    z8 = torch.zeros(64, dtype=torch.uint8, device="cuda")
    f = torch.zeros(256, device="cuda")
    n = (SCRATCH_FLOATS + 1) * 32          # one outer block past the limit; nothing is read
    with pytest.raises(BBCError, match="static scratch"):
        bbc.dequantize_4bit_nested_chain_noalloc(z8, z8, f, f, 0.0, f, n, 32, torch.float16, out=f)


@pytest.mark.gpu
def test_noalloc_refuses_host_memory(bbc):
    # a pinned host buffer as the output: refused on the host, nothing launched
    L = bbc.load_library()
    n, bs = 4096, 64
    codes, q, a2, off = synthetic.nested_state(n, bs, seed=2, device="cuda")
    code2 = torch.from_numpy(synthetic.general8_table()).cuda()
    code4 = torch.from_numpy(synthetic.fp4_table()).cuda()
    host_out = torch.empty(n, dtype=torch.float16).pin_memory()
    st = L.dequantize_4bit_nested_chain_noalloc(_p(codes), _p(q), _p(code2), _p(a2), ct.c_float(float(off)),
                                                _p(code4), n, bs, 256, int(bbc.BBC_F16), _p(host_out),
                                                ct.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 1 and "host memory" in bbc.bbc_last_error()
