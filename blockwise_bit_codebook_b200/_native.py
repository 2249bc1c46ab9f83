"""ctypes binding of libbbc.so (argument marshalling only)."""
import ctypes as ct
import os

import numpy as np

BBC_F16, BBC_BF16, BBC_F32 = 0, 1, 2
_STATUS = {0: "BBC_OK", 1: "BBC_ERR_INVALID", 2: "BBC_ERR_UNSUPPORTED", 3: "BBC_ERR_CUDA"}

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.environ.get("BBC_LIBRARY") or os.path.join(_HERE, "libbbc.so")
_lib = None


class BBCError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn} failed with {_STATUS.get(status, status)}: {msg}")
        self.status = status


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load libbbc.so; raises if it has not been built (there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"{_LIB_PATH} is missing: build it with "
                          "`python -m blockwise_bit_codebook_b200.build`")
    L = ct.CDLL(_LIB_PATH)
    P, I64, I = ct.c_void_p, ct.c_int64, ct.c_int
    L.kbit_quantize.argtypes = [P, I, I64, I, I, P, P, P, P]
    L.kbit_quantize.restype = I
    L.kbit_dequantize.argtypes = [P, P, P, I, I, I64, I, P, P]
    L.kbit_dequantize.restype = I
    L.quantize_4bit.argtypes = [P, I, I64, I, P, P, P, P]
    L.quantize_4bit.restype = I
    L.quantize_4bit_nested_workspace_bytes.argtypes = [I64, I]
    L.quantize_4bit_nested_workspace_bytes.restype = ct.c_size_t
    L.quantize_4bit_nested.argtypes = [P, I, I64, I, P, P, I, P, P, P, P, P, ct.c_size_t, P]
    L.quantize_4bit_nested.restype = I
    L.linear_4bit_nested.argtypes = [P, I, I64, I64, I64, P, P, P, P, ct.c_float, P, I, I, P, P]
    L.linear_4bit_nested.restype = I
    L.linear_kbit.argtypes = [P, I, I64, I64, I64, P, P, P, I, I, P, P]
    L.linear_kbit.restype = I
    L.kbit_quantize_e4m4.argtypes = [P, I, I64, I, I, P, P, P, P]
    L.kbit_quantize_e4m4.restype = I
    L.kbit_dequantize_e4m4.argtypes = [P, P, P, I, I, I64, I, P, P]
    L.kbit_dequantize_e4m4.restype = I
    L.dequantize_4bit_nested.argtypes = [P, P, P, P, ct.c_float, P, I64, I, I, I, P, P]
    L.dequantize_4bit_nested.restype = I
    L.dequantize_4bit.argtypes = [P, P, P, I64, I, I, P, P]
    L.dequantize_4bit.restype = I
    L.dequantize_4bit_nested_chain.argtypes = [P, P, P, P, ct.c_float, P, I64, I, I, I, P, P, P]
    L.dequantize_4bit_nested_chain.restype = I
    L.dequantize_4bit_nested_chain_noalloc.argtypes = [P, P, P, P, ct.c_float, P, I64, I, I, I, P, P]
    L.dequantize_4bit_nested_chain_noalloc.restype = I
    L.bbc_nf_codebook.argtypes = [I, P]
    L.bbc_nf_codebook.restype = I
    L.bbc_wait_timeouts.argtypes = [ct.POINTER(ct.c_uint)]
    L.bbc_wait_timeouts.restype = I
    L.bbc_debug_status.argtypes = [ct.POINTER(ct.c_uint), ct.c_int]
    L.bbc_debug_status.restype = I
    L.bbc_is_debug_build.argtypes = []
    L.bbc_is_debug_build.restype = I
    L.bbc_last_error.argtypes = []
    L.bbc_last_error.restype = ct.c_char_p
    _lib = L
    return L


def bbc_last_error() -> str:
    return load_library().bbc_last_error().decode()


def _check(fn: str, status: int):
    if status != 0:
        raise BBCError(fn, status, bbc_last_error())


def _dt(dtype) -> int:
    import torch
    if isinstance(dtype, int):
        return dtype
    m = {torch.float16: BBC_F16, torch.bfloat16: BBC_BF16, torch.float32: BBC_F32}
    if dtype not in m:
        raise ValueError(f"unsupported dtype {dtype}")
    return m[dtype]


def _torch_dtype(dt: int):
    import torch
    return {BBC_F16: torch.float16, BBC_BF16: torch.bfloat16, BBC_F32: torch.float32}[dt]


def _ptr(t, device=None, name="tensor"):
    """Address of a tensor argument. Every tensor a call passes must be a contiguous CUDA tensor
    on the call's device (the device of its first tensor): anything else raises ValueError here,
    before the library is called, so that no kernel is given a host address or reads a strided
    view as if it were contiguous."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (it is on {t.device})")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, the call's other tensors on {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ct.c_void_p(t.data_ptr())


def _stream(stream, device):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ct.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def kbit_quantize(A, K: int, codebook, absmax=None, packed=None, blocksize: int = 32, stream=None):
    """k-bit quantize a CUDA tensor (any shape, contiguous). Returns (packed, absmax)."""
    import torch
    L = load_library()
    d = A.device
    n = A.numel()
    nb = (n + blocksize - 1) // blocksize if blocksize > 0 else 0
    if absmax is None:
        absmax = torch.empty(max(nb, 1), dtype=torch.float32, device=A.device)
    if packed is None:
        packed = torch.empty(max(nb * K, 1), dtype=torch.int32, device=A.device)
    st = L.kbit_quantize(_ptr(A, d, "A"), _dt(A.dtype), n, K, blocksize, _ptr(codebook, d, "codebook"),
                         _ptr(absmax, d, "absmax"),
                         _ptr(packed, d, "packed"), _stream(stream, A.device))
    _check("kbit_quantize", st)
    return packed, absmax


def kbit_dequantize(packed, absmax, codebook, K: int, n: int, dtype, out=None, blocksize: int = 32,
                    stream=None):
    """Inverse of kbit_quantize; returns a 1-D CUDA tensor of n elements of `dtype`."""
    import torch
    L = load_library()
    d = packed.device
    dt = _dt(dtype)
    if out is None:
        out = torch.empty(max(n, 1), dtype=_torch_dtype(dt), device=packed.device)
    st = L.kbit_dequantize(_ptr(packed, d, "packed"), _ptr(absmax, d, "absmax"), _ptr(codebook, d, "codebook"),
                           K, blocksize, n, dt, _ptr(out, d, "out"),
                           _stream(stream, packed.device))
    _check("kbit_dequantize", st)
    return out


def kbit_quantize_e4m4(A, K: int, codebook, absmax=None, packed=None, blocksize: int = 32, stream=None):
    """kbit_quantize with the per-block absmax stored as one E4M4 byte. Returns (packed, absmax_u8)."""
    import torch
    L = load_library()
    d = A.device
    n = A.numel()
    nb = (n + blocksize - 1) // blocksize if blocksize > 0 else 0
    if absmax is None:
        absmax = torch.empty(max(nb, 1), dtype=torch.uint8, device=A.device)
    if packed is None:
        packed = torch.empty(max(nb * K, 1), dtype=torch.int32, device=A.device)
    st = L.kbit_quantize_e4m4(_ptr(A, d, "A"), _dt(A.dtype), n, K, blocksize, _ptr(codebook, d, "codebook"),
                              _ptr(absmax, d, "absmax"),
                              _ptr(packed, d, "packed"), _stream(stream, A.device))
    _check("kbit_quantize_e4m4", st)
    return packed, absmax


def kbit_dequantize_e4m4(packed, absmax, codebook, K: int, n: int, dtype, out=None, blocksize: int = 32,
                         stream=None):
    """kbit_dequantize with a uint8 E4M4 absmax; returns a 1-D CUDA tensor of n elements of `dtype`."""
    import torch
    L = load_library()
    d = packed.device
    dt = _dt(dtype)
    if out is None:
        out = torch.empty(max(n, 1), dtype=_torch_dtype(dt), device=packed.device)
    st = L.kbit_dequantize_e4m4(_ptr(packed, d, "packed"), _ptr(absmax, d, "absmax"),
                                _ptr(codebook, d, "codebook"), K, blocksize, n, dt, _ptr(out, d, "out"),
                                _stream(stream, packed.device))
    _check("kbit_dequantize_e4m4", st)
    return out


def quantize_4bit(A, blocksize: int, code4, absmax=None, codes=None, stream=None):
    """4-bit codes (uint8[ceil(n/2)], element 2j high nibble) and fp32 absmax per outer block."""
    import torch
    L = load_library()
    d = A.device
    n = A.numel()
    nbo = (n + blocksize - 1) // blocksize if blocksize > 0 else 1
    if absmax is None:
        absmax = torch.empty(max(nbo, 1), dtype=torch.float32, device=A.device)
    if codes is None:
        codes = torch.empty(max((n + 1) // 2, 1), dtype=torch.uint8, device=A.device)
    st = L.quantize_4bit(_ptr(A, d, "A"), _dt(A.dtype), n, blocksize, _ptr(code4, d, "code4"),
                         _ptr(absmax, d, "absmax"), _ptr(codes, d, "codes"),
                         _stream(stream, A.device))
    _check("quantize_4bit", st)
    return codes, absmax


def quantize_4bit_nested_workspace_bytes(n: int, blocksize: int) -> int:
    return int(load_library().quantize_4bit_nested_workspace_bytes(n, blocksize))


def quantize_4bit_nested(A, blocksize: int, code4, code2, blocksize2: int = 256, workspace=None,
                         out=None, stream=None):
    """The nested 4-bit state of A: (codes, absmax_q, absmax2, offset) with offset a 1-element
    CUDA tensor. `out` may hold preallocated (codes, absmax_q, absmax2, offset)."""
    import torch
    L = load_library()
    d = A.device
    n = A.numel()
    nbo = (n + blocksize - 1) // blocksize if blocksize > 0 else 1
    nbi = (nbo + blocksize2 - 1) // blocksize2 if blocksize2 > 0 else 1
    if out is None:
        out = (torch.empty(max((n + 1) // 2, 1), dtype=torch.uint8, device=A.device),
               torch.empty(max(nbo, 1), dtype=torch.uint8, device=A.device),
               torch.empty(max(nbi, 1), dtype=torch.float32, device=A.device),
               torch.empty(1, dtype=torch.float32, device=A.device))
    codes, absmax_q, absmax2, offset = out
    wsb = quantize_4bit_nested_workspace_bytes(n, blocksize) if n > 0 else 0
    if workspace is None:
        workspace = torch.empty(max(wsb, 1), dtype=torch.uint8, device=A.device)
    st = L.quantize_4bit_nested(_ptr(A, d, "A"), _dt(A.dtype), n, blocksize, _ptr(code4, d, "code4"),
                                _ptr(code2, d, "code2"), blocksize2, _ptr(codes, d, "codes"),
                                _ptr(absmax_q, d, "absmax_q"), _ptr(absmax2, d, "absmax2"),
                                _ptr(offset, d, "offset"), _ptr(workspace, d, "workspace"),
                                workspace.numel() * workspace.element_size(), _stream(stream, A.device))
    _check("quantize_4bit_nested", st)
    return codes, absmax_q, absmax2, offset


def linear_4bit_nested(X, codes, absmax_q, code2, absmax2, offset: float, code4, N: int, blocksize: int,
                       blocksize2: int = 256, out=None, stream=None):
    """Y = X @ W^T for X [M, K] (fp16/bf16) and W [N, K] the nested 4-bit weight, decoded on the
    fly (never materialised; M > 32 on the tensor cores, N % 128 == 0). Returns Y [M, N] in X's
    dtype."""
    import torch
    L = load_library()
    d = X.device
    M, K = X.shape
    if out is None:
        out = torch.empty((M, N), dtype=X.dtype, device=X.device)
    st = L.linear_4bit_nested(_ptr(X, d, "X"), _dt(X.dtype), M, N, K, _ptr(codes, d, "codes"),
                              _ptr(absmax_q, d, "absmax_q"), _ptr(code2, d, "code2"), _ptr(absmax2, d, "absmax2"),
                              ct.c_float(offset), _ptr(code4, d, "code4"), blocksize, blocksize2,
                              _ptr(out, d, "out"), _stream(stream, X.device))
    _check("linear_4bit_nested", st)
    return out


def linear_kbit(X, packed, absmax, codebook, K: int, N: int, blocksize: int = 32, out=None, stream=None):
    """Y = X @ W^T for X [M, Kin] (fp16/bf16) and W [N, Kin] the k-bit weight of kbit_quantize
    (K bits, blocksize 32), decoded on the fly (M > 32 on the tensor cores, N % 128 == 0).
    Returns Y [M, N] in X's dtype."""
    import torch
    L = load_library()
    d = X.device
    M, Kin = X.shape
    if out is None:
        out = torch.empty((M, N), dtype=X.dtype, device=X.device)
    st = L.linear_kbit(_ptr(X, d, "X"), _dt(X.dtype), M, N, Kin, _ptr(packed, d, "packed"),
                       _ptr(absmax, d, "absmax"), _ptr(codebook, d, "codebook"), K, blocksize,
                       _ptr(out, d, "out"), _stream(stream, X.device))
    _check("linear_kbit", st)
    return out


def dequantize_4bit_nested(codes, absmax_q, code2, absmax2, offset: float, code4, n: int,
                           blocksize: int, dtype, out=None, blocksize2: int = 256, stream=None):
    """Nested NF4/FP4 dequant; returns a 1-D CUDA tensor of n elements of `dtype`."""
    import torch
    L = load_library()
    d = codes.device
    dt = _dt(dtype)
    if out is None:
        out = torch.empty(max(n, 1), dtype=_torch_dtype(dt), device=codes.device)
    st = L.dequantize_4bit_nested(_ptr(codes, d, "codes"), _ptr(absmax_q, d, "absmax_q"),
                                  _ptr(code2, d, "code2"), _ptr(absmax2, d, "absmax2"),
                                  ct.c_float(offset), _ptr(code4, d, "code4"), n, blocksize, blocksize2, dt,
                                  _ptr(out, d, "out"), _stream(stream, codes.device))
    _check("dequantize_4bit_nested", st)
    return out


def dequantize_4bit(codes, absmax, code4, n: int, blocksize: int, dtype, out=None, stream=None):
    """Plain NF4/FP4 decode with an fp32 absmax per block; returns n elements of `dtype`."""
    import torch
    L = load_library()
    d = codes.device
    dt = _dt(dtype)
    if out is None:
        out = torch.empty(max(n, 1), dtype=_torch_dtype(dt), device=codes.device)
    st = L.dequantize_4bit(_ptr(codes, d, "codes"), _ptr(absmax, d, "absmax"), _ptr(code4, d, "code4"), n,
                           blocksize, dt, _ptr(out, d, "out"),
                           _stream(stream, codes.device))
    _check("dequantize_4bit", st)
    return out


def dequantize_4bit_nested_chain(codes, absmax_q, code2, absmax2, offset: float, code4, n: int,
                                 blocksize: int, dtype, out=None, scale_workspace=None,
                                 blocksize2: int = 256, stream=None):
    """The unfused three-launch form of dequantize_4bit_nested (same result)."""
    import torch
    L = load_library()
    d = codes.device
    dt = _dt(dtype)
    if out is None:
        out = torch.empty(max(n, 1), dtype=_torch_dtype(dt), device=codes.device)
    if scale_workspace is None:
        scale_workspace = torch.empty(max((n + blocksize - 1) // blocksize, 1), dtype=torch.float32,
                                      device=codes.device)
    st = L.dequantize_4bit_nested_chain(_ptr(codes, d, "codes"), _ptr(absmax_q, d, "absmax_q"),
                                        _ptr(code2, d, "code2"), _ptr(absmax2, d, "absmax2"),
                                        ct.c_float(offset), _ptr(code4, d, "code4"), n, blocksize, blocksize2, dt,
                                        _ptr(out, d, "out"), _ptr(scale_workspace, d, "scale_workspace"),
                                        _stream(stream, codes.device))
    _check("dequantize_4bit_nested_chain", st)
    return out


def dequantize_4bit_nested_chain_noalloc(codes, absmax_q, code2, absmax2, offset: float, code4, n: int,
                                         blocksize: int, dtype, out=None, blocksize2: int = 256,
                                         stream=None):
    """The three-launch chain with its scale tensor in the library's fixed scratch.

    For callers that cannot allocate device memory: nothing is allocated by the call (pass
    `out` to allocate nothing here either). At most BBC_NOALLOC_SCRATCH_FLOATS outer blocks;
    calls that can overlap on the GPU share the scratch and race.
    """
    import torch
    L = load_library()
    d = codes.device
    dt = _dt(dtype)
    if out is None:
        out = torch.empty(max(n, 1), dtype=_torch_dtype(dt), device=codes.device)
    st = L.dequantize_4bit_nested_chain_noalloc(_ptr(codes, d, "codes"), _ptr(absmax_q, d, "absmax_q"),
                                                _ptr(code2, d, "code2"), _ptr(absmax2, d, "absmax2"),
                                                ct.c_float(offset), _ptr(code4, d, "code4"), n, blocksize, blocksize2,
                                                dt, _ptr(out, d, "out"), _stream(stream, codes.device))
    _check("dequantize_4bit_nested_chain_noalloc", st)
    return out


def bbc_wait_timeouts() -> int:
    """Bounded in-kernel waits that gave up on the current device since the last call (the
    count is reset); 0 when every wait completed."""
    L = load_library()
    c = ct.c_uint(0)
    _check("bbc_wait_timeouts", L.bbc_wait_timeouts(ct.byref(c)))
    return int(c.value)


def bbc_debug_status(reset: bool = False) -> int:
    """Bits of the debug build's bounds guards that failed on the current device (0 in a release
    build); `reset` clears them after reading."""
    L = load_library()
    c = ct.c_uint(0)
    _check("bbc_debug_status", L.bbc_debug_status(ct.byref(c), 1 if reset else 0))
    return int(c.value)


def bbc_is_debug_build() -> bool:
    """True when the loaded library was compiled with the bounds guards."""
    return bool(load_library().bbc_is_debug_build())


def bbc_nf_codebook(K: int) -> np.ndarray:
    """Host-side normal-float codebook (2^K fp32 values, ascending, max |c| = 1)."""
    L = load_library()
    out = np.empty(1 << K, np.float32)
    _check("bbc_nf_codebook", L.bbc_nf_codebook(K, out.ctypes.data_as(ct.c_void_p)))
    return out
