"""Helpers shared by the GPU parity tests (host-side marshalling only)."""
import numpy as np
import torch

DTYPES = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}


def dtname(dtype) -> str:
    return {torch.float16: "f16", torch.bfloat16: "bf16", torch.float32: "f32"}[dtype]


def to_host(t: torch.Tensor) -> np.ndarray:
    """fp32 -> float32 array; fp16/bf16 -> raw uint16 patterns (the oracle's input form)."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.float32:
        return t.numpy().copy()
    if t.dtype in (torch.float16, torch.bfloat16):
        return t.view(torch.int16).numpy().view(np.uint16).copy()
    if t.dtype == torch.int32:
        return t.numpy().view(np.uint32).copy()
    return t.numpy().copy()


def assert_bits_equal(got: np.ndarray, ref: np.ndarray, what: str = ""):
    """Exact equality of bit patterns; a NaN matches any NaN of the same format."""
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    if got.dtype == np.float32:
        g, r = got.view(np.uint32), ref.view(np.uint32)
        gn, rn = np.isnan(got), np.isnan(ref)
    elif got.dtype == np.uint16 and what.endswith("f16"):
        g, r = got, ref
        gn = ((got & 0x7C00) == 0x7C00) & ((got & 0x3FF) != 0)
        rn = ((ref & 0x7C00) == 0x7C00) & ((ref & 0x3FF) != 0)
    elif got.dtype == np.uint16:
        g, r = got, ref
        gn = ((got & 0x7F80) == 0x7F80) & ((got & 0x7F) != 0)
        rn = ((ref & 0x7F80) == 0x7F80) & ((ref & 0x7F) != 0)
    else:
        g, r = got, ref
        gn = rn = np.zeros(got.shape, bool)
    assert np.array_equal(gn, rn), f"{what}: NaN positions differ"
    bad = np.flatnonzero((g != r) & ~gn)
    assert bad.size == 0, f"{what}: {bad.size} mismatches, first at {bad[:8]}: got {g[bad[:8]]} ref {r[bad[:8]]}"


def float_keys_to_f32(keys: np.ndarray) -> np.ndarray:
    keys = keys.astype(np.int64)
    bits = np.where(keys >= 0, keys, (-(keys + 1)) | 0x80000000).astype(np.uint32)
    return bits.view(np.float32)


def f32_key(v) -> int:
    b = int(np.float32(v).view(np.uint32))
    return b if b < 0x80000000 else -(b & 0x7FFFFFFF) - 1
