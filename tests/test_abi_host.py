"""Host-only checks of the C ABI (no GPU needed, no kernel launched).

* libbbc.so loads and exports every function declared in include/bbc.h;
* argument validation happens on the host before any CUDA call, so invalid
  calls return their status here without a device;
* bbc_nf_codebook (host code) equals the oracle's normal-float codebook.
"""
import ctypes as ct
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bbc.h")


@pytest.fixture(scope="module")
def lib():
    from blockwise_bit_codebook_b200 import build, load_library
    build.build()
    return load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(\w+)\s*\(", text, flags=re.M)


def test_header_declares_the_boundary():
    names = set(declared_functions())
    assert {"kbit_quantize", "kbit_dequantize", "dequantize_4bit_nested", "dequantize_4bit",
            "dequantize_4bit_nested_chain", "bbc_nf_codebook", "bbc_last_error",
            "kbit_quantize_e4m4", "kbit_dequantize_e4m4", "quantize_4bit", "quantize_4bit_nested",
            "quantize_4bit_nested_workspace_bytes", "linear_4bit_nested", "linear_kbit"} <= names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_exported_symbols_via_nm(lib):
    import subprocess
    from blockwise_bit_codebook_b200 import library_path
    out = subprocess.run(["nm", "-D", "--defined-only", library_path()], capture_output=True,
                         text=True).stdout
    syms = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in declared_functions():
        assert name in syms, name


P = ct.c_void_p
FAKE = P(0x1000)        # never dereferenced: every call below fails validation first


def _q(lib, A=FAKE, dtype=2, n=64, K=4, bs=32, cb=FAKE, am=FAKE, pk=FAKE):
    return lib.kbit_quantize(A, dtype, n, K, bs, cb, am, pk, None)


def _dq(lib, pk=FAKE, am=FAKE, cb=FAKE, K=4, bs=32, n=64, dt=2, out=FAKE):
    return lib.kbit_dequantize(pk, am, cb, K, bs, n, dt, out, None)


def _nd(lib, n=64, bs=64, bs2=256, dt=1, codes=FAKE, out=FAKE):
    return lib.dequantize_4bit_nested(codes, FAKE, FAKE, FAKE, ct.c_float(0.0), FAKE, n, bs, bs2, dt,
                                      out, None)


def test_quantize_validation(lib):
    assert _q(lib, A=None) == 1
    assert _q(lib, cb=None) == 1 and _q(lib, am=None) == 1 and _q(lib, pk=None) == 1
    assert _q(lib, n=0) == 1 and _q(lib, n=-5) == 1
    for K in (0, 1, 6, 8):
        assert _q(lib, K=K) == 1
    assert "K must be 2..5" in lib.bbc_last_error().decode()
    assert _q(lib, dtype=3) == 1 and _q(lib, dtype=-1) == 1
    assert _q(lib, bs=64) == 2 and _q(lib, bs=16) == 2
    assert _q(lib, A=P(0x1001), dtype=0) == 1          # fp16 at an odd address
    assert _q(lib, am=P(0x1002)) == 1


def test_dequantize_validation(lib):
    assert _dq(lib, pk=None) == 1 and _dq(lib, out=None) == 1
    assert _dq(lib, n=0) == 1
    assert _dq(lib, K=6) == 1 and _dq(lib, K=1) == 1
    assert _dq(lib, dt=7) == 1
    assert _dq(lib, bs=128) == 2
    assert _dq(lib, out=P(0x1002), dt=2) == 1           # fp32 output at a 2-byte address
    assert _dq(lib, pk=P(0x1001)) == 1


def test_e4m4_validation(lib):
    q = lambda A=FAKE, dtype=1, n=64, K=4, bs=32, am=FAKE: lib.kbit_quantize_e4m4(  # noqa: E731
        A, dtype, n, K, bs, FAKE, am, FAKE, None)
    d = lambda am=FAKE, K=4, bs=32, n=64, dt=1, out=FAKE: lib.kbit_dequantize_e4m4(  # noqa: E731
        FAKE, am, FAKE, K, bs, n, dt, out, None)
    assert q(A=None) == 1 and q(am=None) == 1 and q(n=0) == 1 and q(K=6) == 1 and q(dtype=4) == 1
    assert "kbit_quantize_e4m4" in lib.bbc_last_error().decode()
    assert q(bs=64) == 2
    assert q(A=P(0x1001)) == 1                           # bf16 input at an odd address
    assert d(am=None) == 1 and d(out=None) == 1 and d(n=-1) == 1 and d(K=1) == 1 and d(dt=3) == 1
    assert d(bs=16) == 2
    assert d(out=P(0x1001), dt=0) == 1
    assert "kbit_dequantize_e4m4" in lib.bbc_last_error().decode()


def test_quantize_4bit_validation(lib):
    q = lambda A=FAKE, dt=1, n=64, bs=64, cb=FAKE, am=FAKE, co=FAKE: lib.quantize_4bit(  # noqa: E731
        A, dt, n, bs, cb, am, co, None)
    assert q(A=None) == 1 and q(co=None) == 1 and q(am=None) == 1 and q(n=0) == 1 and q(dt=3) == 1
    for bs in (0, 16, 48, 8192):
        assert q(bs=bs) == 1
    assert "blocksize" in lib.bbc_last_error().decode()
    assert q(A=P(0x1001), dt=0) == 1 and q(am=P(0x1002)) == 1
    ws = lib.quantize_4bit_nested_workspace_bytes
    assert ws(0, 64) == 0 and ws(100, 48) == 0
    for n in (10 ** 6, 64 * 2048 * 3):                   # 8 and 3 first-level tree nodes
        nbo = (n + 63) // 64
        s1 = (nbo + 2047) // 2048
        # absmax (256-byte padded), then the two node buffers, the first padded to an even count
        assert ws(n, 64) == ((nbo * 4 + 255) // 256) * 256 + (s1 + (s1 & 1) + (s1 + 2047) // 2048) * 8
    nq = lambda ws_ptr=P(0x100000), wsb=1 << 20, bs2=256, n=4096, off=FAKE: lib.quantize_4bit_nested(  # noqa: E731
        FAKE, 1, n, 64, FAKE, FAKE, bs2, FAKE, FAKE, FAKE, off, ws_ptr, wsb, None)
    assert nq(ws_ptr=None) == 1 and nq(off=None) == 1 and nq(n=-1) == 1
    assert nq(bs2=128) == 2
    assert nq(wsb=10) == 1 and "workspace" in lib.bbc_last_error().decode()
    assert nq(ws_ptr=P(0x100010)) == 1                   # workspace not 256-byte aligned


def test_nested_validation(lib):
    assert _nd(lib, codes=None) == 1 and _nd(lib, out=None) == 1
    assert _nd(lib, n=0) == 1
    for bs in (0, 16, 48, 100, 8192):
        assert _nd(lib, bs=bs) == 1
    assert _nd(lib, bs2=128) == 2
    assert _nd(lib, dt=5) == 1
    assert "blocksize2 must be 256" in (lib.bbc_last_error().decode() if _nd(lib, bs2=512) else "")


def test_plain_and_chain_validation(lib):
    assert lib.dequantize_4bit(None, FAKE, FAKE, 64, 64, 1, FAKE, None) == 1
    assert lib.dequantize_4bit(FAKE, FAKE, FAKE, 0, 64, 1, FAKE, None) == 1
    assert lib.dequantize_4bit(FAKE, FAKE, FAKE, 64, 48, 1, FAKE, None) == 1
    assert lib.dequantize_4bit(FAKE, FAKE, FAKE, 64, 64, 9, FAKE, None) == 1
    chain = lambda ws=FAKE, bs=64, bs2=256: lib.dequantize_4bit_nested_chain(  # noqa: E731
        FAKE, FAKE, FAKE, FAKE, ct.c_float(0.0), FAKE, 64, bs, bs2, 1, FAKE, ws, None)
    assert chain(ws=None) == 1
    assert chain(ws=P(0x1002)) == 1
    assert chain(bs=16) == 1
    assert chain(bs2=128) == 2


def test_linear_validation(lib):
    """Both fused linear entries reject bad arguments on the host (the pointers are never read)."""
    lib.linear_kbit.argtypes = [ct.c_void_p, ct.c_int, ct.c_int64, ct.c_int64, ct.c_int64, ct.c_void_p,
                                ct.c_void_p, ct.c_void_p, ct.c_int, ct.c_int, ct.c_void_p, ct.c_void_p]
    kl = lambda X=FAKE, dt=1, M=1, N=16, K=64, pk=FAKE, am=FAKE, cb=FAKE, bits=4, bs=32, Y=FAKE: lib.linear_kbit(  # noqa: E731
        X, dt, M, N, K, pk, am, cb, bits, bs, Y, None)
    assert kl(X=None) == 1 and kl(pk=None) == 1 and kl(Y=None) == 1 and kl(M=0) == 1
    assert kl(bits=1) == 1 and kl(bits=6) == 1 and "bits" in lib.bbc_last_error().decode()
    assert kl(bs=64) == 2 and kl(dt=2) == 2 and kl(M=33) == 2 and kl(N=24) == 2 and kl(K=96) == 2
    assert kl(pk=P(0x100008)) == 1 and kl(X=P(0x100008)) == 1
    assert "16-byte" in lib.bbc_last_error().decode()
    lib.linear_4bit_nested.argtypes = [ct.c_void_p, ct.c_int, ct.c_int64, ct.c_int64, ct.c_int64, ct.c_void_p,
                                       ct.c_void_p, ct.c_void_p, ct.c_void_p, ct.c_float, ct.c_void_p, ct.c_int,
                                       ct.c_int, ct.c_void_p, ct.c_void_p]
    nl = lambda X=FAKE, dt=1, M=1, N=16, K=64, co=FAKE, bs=64, bs2=256: lib.linear_4bit_nested(  # noqa: E731
        X, dt, M, N, K, co, FAKE, FAKE, FAKE, 0.0, FAKE, bs, bs2, FAKE, None)
    assert nl(X=None) == 1 and nl(K=0) == 1 and nl(bs=48) == 1 and nl(co=P(0x100008)) == 1
    assert nl(dt=2) == 2 and nl(M=40) == 2 and nl(K=32) == 2 and nl(bs2=128) == 2


def test_last_error_is_per_thread(lib):
    import threading
    _q(lib, K=9)
    seen = {}

    def other():
        seen["msg"] = lib.bbc_last_error().decode()
    t = threading.Thread(target=other)
    t.start()
    t.join()
    assert seen["msg"] == "" and "K must be" in lib.bbc_last_error().decode()


@pytest.mark.parametrize("K", [1, 2, 3, 4, 5, 6, 7, 8])
def test_nf_codebook_matches_oracle(lib, orc, K):
    from blockwise_bit_codebook_b200 import bbc_nf_codebook
    ours = bbc_nf_codebook(K)
    if K <= 5:
        ref = orc.normal_float_codebook(K)
    else:   # same construction through the oracle module's quantile routine
        from oracle.codebook import unnormalized_quantiles
        q = unnormalized_quantiles(K)
        ref = q / np.abs(q).max()
    assert np.array_equal(ours.view(np.uint32), ref.view(np.uint32))


def test_nf_codebook_rejects_bad_k(lib):
    out = np.empty(512, np.float32)
    assert lib.bbc_nf_codebook(0, out.ctypes.data_as(P)) == 1
    assert lib.bbc_nf_codebook(9, out.ctypes.data_as(P)) == 1
    assert lib.bbc_nf_codebook(4, None) == 1


def test_debug_build_exports_the_same_boundary():
    """libbbc_debug.so (the bounds-guarded build) exports every declared function and says it is
    the debug build; the release library says it is not (no CUDA call is made)."""
    import subprocess
    from blockwise_bit_codebook_b200 import build, load_library
    dbg_path = build.build(debug=True)
    out = subprocess.run(["nm", "-D", "--defined-only", dbg_path], capture_output=True, text=True).stdout
    syms = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in declared_functions():
        assert name in syms, name
    dbg = ct.CDLL(dbg_path)
    assert dbg.bbc_is_debug_build() == 1
    assert load_library().bbc_is_debug_build() == 0


def test_debug_status_rejects_a_null_pointer(lib):
    assert lib.bbc_debug_status(None, 0) == 1


def test_debug_status_without_a_device_reports_a_cuda_error(lib):
    """With no usable device the status read fails cleanly (BBC_ERR_CUDA), it does not crash; on
    a device the release build reports 0."""
    c = ct.c_uint(123)
    st = lib.bbc_debug_status(ct.byref(c), 1)
    assert st in (0, 3), st
    if st == 0:
        assert c.value == 0
