"""Seeded synthetic inputs with the shapes and value distributions of the workloads.

This module generates data only; it holds none of the method's arithmetic and
is shared by the tests, the benchmark and the smoke check. Every draw is a
seeded torch generator on the requested device (CPU generation and CUDA
generation give different, individually reproducible streams).

Workloads (sizes from the k-bit patch series' tests and the nested-dequant
pull request's benchmark shapes):
  * k-bit weights: N(0, std) fp32, optionally with a seeded fraction of
    entries scaled by 20 as outliers, then cast to fp16/bf16/fp32;
  * nested 4-bit state: uniform random code bytes (all 16 nibbles occur),
    uniform General8 absmax codes (or a seeded permutation of i mod 256 so all
    256 codes occur), inner absmax ~ U(0.01, 0.1) fp32, offset ~ N(0.03, 0.005).

The NF4, FP4 and General8 tables of bitsandbytes are not printed on the pages,
so the nested path takes them as inputs; the tables here are documented
synthetic stand-ins (the NF4 stand-in is the library's own 16-entry
normal-float codebook, from bbc_nf_codebook or the oracle).
"""
import numpy as np
import torch


def _gen(seed: int, device) -> torch.Generator:
    return torch.Generator(device=torch.device(device)).manual_seed(int(seed))


def weights(n: int, std: float = 1.0, seed: int = 0, dtype=torch.float32, device="cpu",
            outlier_frac: float = 0.0, outlier_scale: float = 20.0, outlier_seed: int = 2):
    """N(0, std) values in fp32, a seeded fraction scaled by outlier_scale, cast to dtype."""
    x = torch.randn(n, generator=_gen(seed, device), device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    if outlier_frac > 0:
        k = int(round(n * outlier_frac))
        idx = torch.randperm(n, generator=_gen(outlier_seed, device), device=device)[:k]
        x[idx] *= outlier_scale
    return x.to(dtype)


def fp4_table() -> np.ndarray:
    """Stand-in FP4 value table: sign-magnitude, codes 0..7 = +{0, 1/12, 1/6, 1/4, 1/3, 1/2, 2/3, 1},
    codes 8..15 the same magnitudes negated (code 8 is -0.0)."""
    mags = np.array([0.0, 1 / 12, 1 / 6, 1 / 4, 1 / 3, 1 / 2, 2 / 3, 1.0], np.float64)
    return np.concatenate([mags, -mags]).astype(np.float32)


def general8_table() -> np.ndarray:
    """Stand-in General8 code table: 256 ascending fp32 values t^3, t = (i - 127.5) / 127.5,
    spanning [-1, 1] over several binades."""
    t = (np.arange(256, dtype=np.float64) - 127.5) / 127.5
    return (np.sign(t) * np.abs(t) ** 3).astype(np.float32)


def nested_state(n: int, blocksize: int, seed: int = 3, device="cpu", all_codes: bool = False,
                 blocksize2: int = 256):
    """Codes, General8 absmax codes, inner absmax and offset for an n-element nested 4-bit tensor."""
    nbytes = (n + 1) // 2
    nbo = (n + blocksize - 1) // blocksize
    nbi = (nbo + blocksize2 - 1) // blocksize2
    codes = torch.randint(0, 256, (nbytes,), generator=_gen(seed, device), device=device,
                          dtype=torch.uint8)
    if all_codes:
        perm = torch.randperm(nbo, generator=_gen(seed + 1, device), device=device)
        absmax_q = (perm % 256).to(torch.uint8)
    else:
        absmax_q = torch.randint(0, 256, (nbo,), generator=_gen(seed + 1, device), device=device,
                                 dtype=torch.uint8)
    absmax2 = torch.rand(nbi, generator=_gen(seed + 2, device), device=device,
                         dtype=torch.float32) * 0.09 + 0.01
    offset = float(torch.randn(1, generator=_gen(seed + 3, "cpu"), dtype=torch.float32)[0] * 0.005 + 0.03)
    return codes, absmax_q, absmax2, np.float32(offset)


def kbit_state(n: int, K: int, seed: int = 5, device="cpu"):
    """A k-bit weight state for n elements (blocksize 32): uniformly random bit-plane words, so
    every index 0 .. 2^K - 1 occurs, and per-block absmax ~ U(0.01, 0.1)."""
    nb = (n + 31) // 32
    packed = torch.randint(-2 ** 31, 2 ** 31, (nb * K,), generator=_gen(seed, device), device=device,
                           dtype=torch.int64).to(torch.int32)
    absmax = torch.rand(nb, generator=_gen(seed + 1, device), device=device, dtype=torch.float32) * 0.09 + 0.01
    return packed, absmax
