"""Blockwise bit-codebook quantization on NVIDIA B200 (sm_100a).

Thin Python binding of the C ABI in include/bbc.h (libbbc.so, built in-tree by
``python -m blockwise_bit_codebook_b200.build``). The functions carry the C
names and only marshal arguments: every step of every operation runs in the
library's CUDA kernels. torch is used for device memory and streams only.

    kbit_quantize(A, K, codebook)                       -> (packed, absmax)
    kbit_dequantize(packed, absmax, codebook, K, n, dtype) -> out
    kbit_quantize_e4m4 / kbit_dequantize_e4m4   the same with a uint8 E4M4 absmax
    dequantize_4bit_nested(codes, absmax_q, code2, absmax2, offset, code4,
                           n, blocksize, dtype)         -> out
    dequantize_4bit(codes, absmax, code4, n, blocksize, dtype)  -> out
    quantize_4bit(A, blocksize, code4)                  -> (codes, absmax)
    quantize_4bit_nested(A, blocksize, code4, code2)    -> (codes, absmax_q, absmax2, offset)
    dequantize_4bit_nested_chain(...)   the unfused three-launch form (same result)
    bbc_nf_codebook(K)                                  -> np.float32[2^K] (host)

There is no CPU fallback: if libbbc.so is missing or a call fails, an
exception is raised.
"""
from ._native import (  # noqa: F401
    BBC_BF16,
    BBC_F16,
    BBC_F32,
    BBCError,
    bbc_last_error,
    bbc_nf_codebook,
    bbc_wait_timeouts,
    bbc_debug_status,
    bbc_is_debug_build,
    dequantize_4bit,
    dequantize_4bit_nested,
    dequantize_4bit_nested_chain,
    dequantize_4bit_nested_chain_noalloc,
    kbit_dequantize,
    kbit_dequantize_e4m4,
    kbit_quantize,
    kbit_quantize_e4m4,
    quantize_4bit,
    quantize_4bit_nested,
    quantize_4bit_nested_workspace_bytes,
    library_path,
    linear_4bit_nested,
    linear_kbit,
    load_library,
)
