"""Normal-float codebook, as the k-bit pages define it (test infrastructure only).

Source: bitsandbytes k-bit patch series, tests/test_kbit_quantization.py and
bitsandbytes/functional.py, create_normal_float_codebook. For n = 2^k levels the
pages take the standard-normal quantile at the n bin midpoints
(levels from 0.5/n to 1 - 0.5/n, evenly spaced, in fp32), evaluated in float64,
rounded to fp32, then divide the fp32 vector by its largest magnitude (in fp32).

The evenly spaced fp32 levels are exactly (2i+1)/(2n) for n a power of two, so
they are formed here directly. The quantile function is scipy's norm.ppf, the
library routine the pages name.
"""
import numpy as np
from scipy.stats import norm


def normal_float_codebook(k: int) -> np.ndarray:
    n = 1 << k
    levels = (2.0 * np.arange(n, dtype=np.float64) + 1.0) / (2.0 * n)   # exact in fp32 and fp64
    levels32 = levels.astype(np.float32)
    q = norm.ppf(levels32.astype(np.float64)).astype(np.float32)
    return q / np.abs(q).max()


def unnormalized_quantiles(k: int) -> np.ndarray:
    """The fp32 quantiles before the division by the largest magnitude."""
    n = 1 << k
    levels = (2.0 * np.arange(n, dtype=np.float64) + 1.0) / (2.0 * n)
    return norm.ppf(levels).astype(np.float32)
