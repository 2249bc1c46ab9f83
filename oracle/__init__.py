"""Plain CPU oracle for blockwise codebook quantization.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package. The library (``blockwise_bit_codebook_b200``) never imports it, and
it never imports the library. Each function cites the passage it follows:

* k-bit codec: bitsandbytes k-bit patch series, tests/test_kbit_quantization.py
  (quantize_kbit_ref, dequantize_kbit_ref, pack_kbit_ref, unpack_kbit_ref) and
  csrc/ops.cu (kQuantizeBlockwise_kbit, kDequantizeBlockwise_kbit).
* E4M4 uint8 absmax: the same series, PATCH 005 "Add vectorized dequant kernel
  and E4M4 uint8 absmax support" (encode_absmax_e4m4, decode_absmax_e4m4 in
  bitsandbytes/functional.py; decode_e4m4_absmax in csrc/ops.cu), and the
  quantize_kbit / dequantize_kbit paths that use it.
* 4-bit quantize, the nested offset and the General8 absmax compression (the
  inverse of the nested dequant): readings built from the k-bit rule and the
  nested decode, since the nested-dequant page does not describe the quantize.
* the dequant fused into its linear consumer (the page's dequantize-plus-linear
  public-path controls): nested_dequantize, then a float64 matmul (a library step).
* nested 4-bit dequant and the plain 4-bit decode of its unfused form: "Fuse
  nested 4-bit scale reconstruction on SM103", Summary and Implementation.

Arrays: fp32 as ``np.float32``; fp16 and bfloat16 as their raw 16-bit patterns
in ``np.uint16`` (numpy has no bfloat16). dtype names are "f16", "bf16", "f32".

Parity status of each function (see the pins in tests/test_oracle_*.py):
every function here is pinned; none is "parity unpinned".
"""
import ctypes as ct
import os

import numpy as np

from . import build as _build
from .codebook import normal_float_codebook, unnormalized_quantiles  # noqa: F401

_DT = {"f16": 0, "bf16": 1, "f32": 2}
KBIT_BLOCKSIZE = 32

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ct.CDLL(path)
        P = ct.c_void_p
        I64 = ct.c_int64
        L.orc_kbit_quantize.argtypes = [P, ct.c_int, I64, ct.c_int, P, P, P, P]
        L.orc_kbit_quantize.restype = ct.c_int
        L.orc_kbit_dequantize.argtypes = [P, P, P, ct.c_int, I64, ct.c_int, P]
        L.orc_kbit_dequantize.restype = ct.c_int
        L.orc_nested_dequantize.argtypes = [P, P, P, P, ct.c_float, P, I64, I64, I64, ct.c_int, P]
        L.orc_nested_dequantize.restype = ct.c_int
        L.orc_dequantize_4bit.argtypes = [P, P, P, I64, I64, ct.c_int, P]
        L.orc_dequantize_4bit.restype = ct.c_int
        L.orc_kbit_pack.argtypes = [P, I64, ct.c_int, P]
        L.orc_kbit_unpack.argtypes = [P, I64, ct.c_int, P]
        L.orc_nearest_entry.argtypes = [ct.c_float, P, ct.c_int]
        L.orc_nearest_entry.restype = ct.c_int
        L.orc_nested_scale.argtypes = [ct.c_float, ct.c_float, ct.c_float]
        L.orc_nested_scale.restype = ct.c_float
        for f in ("orc_f32_to_f16_array", "orc_f32_to_bf16_array"):
            getattr(L, f).argtypes = [P, I64, P]
        L.orc_f16_to_f32_array.argtypes = [P, I64, P]
        L.orc_e4m4_encode.argtypes = [ct.c_float]
        L.orc_e4m4_encode.restype = ct.c_uint8
        L.orc_e4m4_decode.argtypes = [ct.c_uint8]
        L.orc_e4m4_decode.restype = ct.c_float
        L.orc_quantize_4bit.argtypes = [P, ct.c_int, I64, I64, P, P, P]
        L.orc_quantize_4bit.restype = ct.c_int
        L.orc_absmax_offset.argtypes = [P, I64]
        L.orc_absmax_offset.restype = ct.c_float
        L.orc_quantize_absmax_nested.argtypes = [P, I64, ct.c_float, P, I64, P, P]
        L.orc_quantize_absmax_nested.restype = ct.c_int
        L.orc_e4m4_encode_array.argtypes = [P, I64, P]
        L.orc_e4m4_decode_array.argtypes = [P, I64, P]
        _lib = L
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ct.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_blocks(n: int, bs: int = KBIT_BLOCKSIZE) -> int:
    return (n + bs - 1) // bs


def f32_to_f16_bits(x) -> np.ndarray:
    x = _c(x, np.float32).reshape(-1)
    out = np.empty(x.size, np.uint16)
    lib().orc_f32_to_f16_array(_p(x), x.size, _p(out))
    return out


def f32_to_bf16_bits(x) -> np.ndarray:
    x = _c(x, np.float32).reshape(-1)
    out = np.empty(x.size, np.uint16)
    lib().orc_f32_to_bf16_array(_p(x), x.size, _p(out))
    return out


def f16_bits_to_f32(h) -> np.ndarray:
    h = _c(h, np.uint16).reshape(-1)
    out = np.empty(h.size, np.float32)
    lib().orc_f16_to_f32_array(_p(h), h.size, _p(out))
    return out


def bf16_bits_to_f32(h) -> np.ndarray:
    h = _c(h, np.uint16).reshape(-1)
    return (h.astype(np.uint32) << 16).view(np.float32)


def nearest_entry(xn: float, codebook) -> int:
    cb = _c(codebook, np.float32)
    return lib().orc_nearest_entry(ct.c_float(xn), _p(cb), cb.size)


def kbit_pack(idx, K: int) -> np.ndarray:
    idx = _c(idx, np.uint8).reshape(-1)
    n = idx.size
    out = np.empty(num_blocks(n) * K, np.uint32)
    lib().orc_kbit_pack(_p(idx), n, K, _p(out))
    return out


def kbit_unpack(packed, K: int, n: int) -> np.ndarray:
    packed = _c(packed, np.uint32).reshape(-1)
    assert packed.size >= num_blocks(n) * K
    out = np.empty(n, np.uint8)
    lib().orc_kbit_unpack(_p(packed), n, K, _p(out))
    return out


def kbit_quantize(A, dtype: str, K: int, codebook, return_indices: bool = False):
    """Quantize; returns (packed uint32[nb*K], absmax f32[nb]) (+ per-lane indices u8[nb*32]).

    A holds fp32 values for dtype "f32", raw 16-bit patterns for "f16"/"bf16".
    """
    A = _c(A, np.float32 if dtype == "f32" else np.uint16).reshape(-1)
    cb = _c(codebook, np.float32)
    assert cb.size == (1 << K)
    n = A.size
    nb = num_blocks(n)
    absmax = np.empty(nb, np.float32)
    packed = np.empty(nb * K, np.uint32)
    idx = np.empty(nb * KBIT_BLOCKSIZE, np.uint8) if return_indices else None
    rc = lib().orc_kbit_quantize(_p(A), _DT[dtype], n, K, _p(cb), _p(absmax), _p(packed),
                                 _p(idx) if idx is not None else None)
    assert rc == 0
    return (packed, absmax, idx) if return_indices else (packed, absmax)


def kbit_dequantize(packed, absmax, codebook, K: int, n: int, dtype: str) -> np.ndarray:
    """Returns fp32 values ("f32") or raw 16-bit patterns ("f16"/"bf16")."""
    packed = _c(packed, np.uint32).reshape(-1)
    absmax = _c(absmax, np.float32).reshape(-1)
    cb = _c(codebook, np.float32)
    nb = num_blocks(n)
    assert packed.size >= nb * K and absmax.size >= nb and cb.size == (1 << K)
    out = np.empty(n, np.float32 if dtype == "f32" else np.uint16)
    rc = lib().orc_kbit_dequantize(_p(packed), _p(absmax), _p(cb), K, n, _DT[dtype], _p(out))
    assert rc == 0
    return out


def e4m4_encode(absmax) -> np.ndarray:
    """fp32 absmax -> uint8 E4M4 codes (bias 11), the pages' encode_absmax_e4m4 steps."""
    a = _c(absmax, np.float32).reshape(-1)
    out = np.empty(a.size, np.uint8)
    lib().orc_e4m4_encode_array(_p(a), a.size, _p(out))
    return out


def e4m4_decode(codes) -> np.ndarray:
    """uint8 E4M4 codes -> their exact fp32 values (decode_absmax_e4m4)."""
    c = _c(codes, np.uint8).reshape(-1)
    out = np.empty(c.size, np.float32)
    lib().orc_e4m4_decode_array(_p(c), c.size, _p(out))
    return out


def kbit_quantize_e4m4(A, dtype: str, K: int, codebook):
    """quantize_kbit with absmax_format "e4m4": the packed words are those of the fp32-absmax
    quantize (the codes use the exact fp32 absmax); the stored absmax is its E4M4 encoding."""
    packed, absmax = kbit_quantize(A, dtype, K, codebook)
    return packed, e4m4_encode(absmax)


def kbit_dequantize_e4m4(packed, absmax_e4m4, codebook, K: int, n: int, dtype: str) -> np.ndarray:
    """dequantize_kbit with a uint8 E4M4 absmax: decode each block's absmax, then the fp32 path."""
    return kbit_dequantize(packed, e4m4_decode(absmax_e4m4), codebook, K, n, dtype)


def quantize_4bit(A, dtype: str, blocksize: int, code4):
    """Per outer block absmax (fp32) and nibble-packed 4-bit codes (uint8[ceil(n/2)], element 2j
    in the high nibble). A: fp32 values or raw 16-bit patterns."""
    A = _c(A, np.float32 if dtype == "f32" else np.uint16).reshape(-1)
    c4 = _c(code4, np.float32)
    assert c4.size == 16
    n = A.size
    absmax = np.empty((n + blocksize - 1) // blocksize, np.float32)
    codes = np.empty((n + 1) // 2, np.uint8)
    assert lib().orc_quantize_4bit(_p(A), _DT[dtype], n, blocksize, _p(c4), _p(absmax), _p(codes)) == 0
    return codes, absmax


def absmax_offset(absmax) -> np.float32:
    """The nested offset: mean of the outer absmax, a pairwise binary64 sum over the values
    zero-padded to a power of two, divided by the count, rounded once to fp32."""
    a = _c(absmax, np.float32).reshape(-1)
    return np.float32(lib().orc_absmax_offset(_p(a), a.size))


def quantize_absmax_nested(absmax, offset: float, code2, blocksize2: int = 256):
    """General8 codes of the centred outer absmax and the per-group inner absmax."""
    a = _c(absmax, np.float32).reshape(-1)
    c2 = _c(code2, np.float32)
    assert c2.size == 256
    nbi = (a.size + blocksize2 - 1) // blocksize2
    q = np.empty(a.size, np.uint8)
    a2 = np.empty(nbi, np.float32)
    assert lib().orc_quantize_absmax_nested(_p(a), a.size, ct.c_float(offset), _p(c2), blocksize2, _p(q),
                                            _p(a2)) == 0
    return q, a2


def quantize_4bit_nested(A, dtype: str, blocksize: int, code4, code2, blocksize2: int = 256):
    """The nested 4-bit state of A: (codes, absmax_q, absmax2, offset)."""
    codes, absmax = quantize_4bit(A, dtype, blocksize, code4)
    off = absmax_offset(absmax)
    q, a2 = quantize_absmax_nested(absmax, float(off), code2, blocksize2)
    return codes, q, a2, off


def linear_4bit_nested(X, x_dtype: str, N: int, K: int, state, code2, code4, blocksize: int,
                       blocksize2: int = 256):
    """Y = X @ W^T with W[N, K] the nested 4-bit weight dequantized to x_dtype (nested_dequantize
    of the flattened N*K codes, rounded to the activation type as the unfused path materialises
    it). Returns (Y64, S): the float64 product (each product of two 16-bit values is exact in
    binary64; the binary64 sums lose at most K * 2^-53 relative) and S = |X| @ |W|^T, the scale of
    the accumulation error bound. X: [M, K] raw 16-bit patterns of x_dtype."""
    codes, absmax_q, absmax2, offset = state
    Wb = nested_dequantize(codes, absmax_q, code2, absmax2, float(offset), code4, N * K, blocksize,
                           blocksize2, x_dtype)
    widen = f16_bits_to_f32 if x_dtype == "f16" else bf16_bits_to_f32
    W = widen(Wb).astype(np.float64).reshape(N, K)
    Xf = widen(_c(X, np.uint16).reshape(-1)).astype(np.float64).reshape(-1, K)
    return Xf @ W.T, np.abs(Xf) @ np.abs(W).T


def linear_kbit(X, x_dtype: str, N: int, Kin: int, packed, absmax, codebook, K: int):
    """Y = X @ W^T with W[N, Kin] the k-bit weight dequantized to x_dtype (kbit_dequantize of the
    flattened N*Kin codes, as the unfused dequantize-then-linear path materialises it). Returns
    (Y64, S) as linear_4bit_nested. X: [M, Kin] raw 16-bit patterns of x_dtype."""
    Wb = kbit_dequantize(packed, absmax, codebook, K, N * Kin, x_dtype)
    widen = f16_bits_to_f32 if x_dtype == "f16" else bf16_bits_to_f32
    W = widen(Wb).astype(np.float64).reshape(N, Kin)
    Xf = widen(_c(X, np.uint16).reshape(-1)).astype(np.float64).reshape(-1, Kin)
    return Xf @ W.T, np.abs(Xf) @ np.abs(W).T


def nested_scale(code2_val: float, absmax2_val: float, offset: float) -> float:
    """fl(fl(code2 * absmax2) + offset) in fp32, returned as a Python float."""
    return float(np.float32(lib().orc_nested_scale(code2_val, absmax2_val, offset)))


def nested_dequantize(codes, absmax_q, code2, absmax2, offset: float, code4,
                      n: int, blocksize: int, blocksize2: int, dtype: str) -> np.ndarray:
    codes = _c(codes, np.uint8).reshape(-1)
    absmax_q = _c(absmax_q, np.uint8).reshape(-1)
    code2 = _c(code2, np.float32)
    absmax2 = _c(absmax2, np.float32).reshape(-1)
    code4 = _c(code4, np.float32)
    nbo = num_blocks(n, blocksize)
    assert codes.size >= (n + 1) // 2 and absmax_q.size >= nbo
    assert absmax2.size >= num_blocks(nbo, blocksize2) and code2.size == 256 and code4.size == 16
    out = np.empty(n, np.float32 if dtype == "f32" else np.uint16)
    rc = lib().orc_nested_dequantize(_p(codes), _p(absmax_q), _p(code2), _p(absmax2),
                                     ct.c_float(offset), _p(code4), n, blocksize, blocksize2,
                                     _DT[dtype], _p(out))
    assert rc == 0
    return out


def dequantize_4bit(codes, absmax, code4, n: int, blocksize: int, dtype: str) -> np.ndarray:
    """Plain 4-bit decode with an fp32 absmax per block (the last launch of the unfused chain)."""
    codes = _c(codes, np.uint8).reshape(-1)
    absmax = _c(absmax, np.float32).reshape(-1)
    code4 = _c(code4, np.float32)
    assert codes.size >= (n + 1) // 2 and absmax.size >= num_blocks(n, blocksize) and code4.size == 16
    out = np.empty(n, np.float32 if dtype == "f32" else np.uint16)
    rc = lib().orc_dequantize_4bit(_p(codes), _p(absmax), _p(code4), n, blocksize, _DT[dtype], _p(out))
    assert rc == 0
    return out
