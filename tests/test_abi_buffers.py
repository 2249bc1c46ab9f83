"""The C ABI's buffer checks and the binding's tensor checks, on the host (no kernel launched).

After the scalar arguments pass, every entry point checks its buffers before any launch: an
output that overlaps an input or another output, and a pointer that is not memory of the
current device, return BBC_ERR_INVALID. The overlap test is host arithmetic; on a machine
without a GPU the device-memory test cannot succeed, so such calls fail there with
BBC_ERR_INVALID too. The Python binding refuses CPU, non-contiguous and other-device tensors
with ValueError before it calls the library.
"""
import ctypes as ct

import pytest

P = ct.c_void_p
INVALID = 1


@pytest.fixture(scope="module")
def lib():
    from blockwise_bit_codebook_b200 import build, load_library
    build.build()
    return load_library()


def _err(lib):
    return lib.bbc_last_error().decode()


# distinct, aligned, non-overlapping addresses for a call whose other arguments are valid
A, CB, AM, PK, OUT = (P(0x10000000 + i * 0x1000000) for i in range(5))


def test_quantize_output_overlapping_input(lib):
    n = 4096
    # packed starts inside A (n bf16 = 8 KB)
    assert lib.kbit_quantize(A, 1, n, 4, 32, CB, AM, P(A.value + 4096), None) == INVALID
    assert "overlaps input A" in _err(lib)
    # absmax inside the codebook
    assert lib.kbit_quantize(A, 1, n, 4, 32, CB, P(CB.value + 32), PK, None) == INVALID
    assert "overlaps input codebook" in _err(lib)
    # the two outputs overlap each other
    assert lib.kbit_quantize(A, 1, n, 4, 32, CB, AM, P(AM.value + 64), None) == INVALID
    assert "outputs absmax and packed overlap" in _err(lib)


def test_adjacent_buffers_do_not_overlap(lib):
    n = 4096
    # packed right after A's last byte: not an overlap, so the call reaches the device-memory check
    st = lib.kbit_quantize(A, 1, n, 4, 32, CB, AM, P(A.value + n * 2), None)
    assert st == INVALID and "overlap" not in _err(lib)


def test_dequant_and_nested_overlaps(lib):
    n = 1 << 14
    assert lib.kbit_dequantize(PK, AM, CB, 3, 32, n, 2, P(PK.value + 16), None) == INVALID
    assert "output out overlaps input packed" in _err(lib)
    st = lib.dequantize_4bit_nested(A, AM, CB, PK, ct.c_float(0.0), P(OUT.value - 16), n, 64, 256, 1, OUT, None)
    assert st == INVALID and "overlaps input code4" in _err(lib)
    st = lib.dequantize_4bit_nested_chain(A, AM, CB, PK, ct.c_float(0.0), CB, n, 64, 256, 1, OUT,
                                          P(OUT.value + 1024), None)
    assert st == INVALID and "outputs out and scale_workspace overlap" in _err(lib)


def test_linear_output_overlapping_weight(lib):
    st = lib.linear_kbit(A, 1, 1, 64, 64, PK, AM, CB, 4, 32, P(PK.value + 64), None)
    assert st == INVALID and "output Y overlaps input packed" in _err(lib)


def test_pointer_that_is_not_device_memory(lib):
    # valid, non-overlapping arguments at addresses that are no CUDA allocation: refused before
    # any launch, whether or not this machine has a GPU
    assert lib.kbit_quantize(A, 1, 4096, 4, 32, CB, AM, PK, None) == INVALID
    msg = _err(lib)
    assert "device memory" in msg or "host memory" in msg or "not memory the CUDA runtime knows" in msg


class _FakeTensor:
    """Just enough of a tensor for the binding's argument checks."""

    def __init__(self, is_cuda=True, device="cuda:0", contiguous=True):
        import torch
        self.is_cuda, self.device, self._c = is_cuda, torch.device(device), contiguous

    def is_contiguous(self):
        return self._c

    def data_ptr(self):
        return 0x1000


def test_binding_refuses_cpu_strided_and_other_device_tensors():
    import torch

    from blockwise_bit_codebook_b200 import _native
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        _native._ptr(torch.zeros(4), torch.device("cuda:0"), "A")
    with pytest.raises(ValueError, match="must be contiguous"):
        _native._ptr(_FakeTensor(contiguous=False), torch.device("cuda:0"), "A")
    with pytest.raises(ValueError, match="is on cuda:1"):
        _native._ptr(_FakeTensor(device="cuda:1"), torch.device("cuda:0"), "codebook")
    assert _native._ptr(_FakeTensor(), torch.device("cuda:0"), "A").value == 0x1000


def test_binding_refuses_a_cpu_input_before_calling():
    import torch

    import blockwise_bit_codebook_b200 as bbc
    with pytest.raises(ValueError, match="A must be a CUDA tensor"):
        bbc.kbit_quantize(torch.zeros(64, dtype=torch.bfloat16), 4, torch.zeros(16))
