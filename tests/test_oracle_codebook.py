"""Pins for the normal-float codebook (k-bit patch series, create_normal_float_codebook).

Checked against what the pages fix (size, ascending order, largest magnitude 1,
near-symmetry, |mean| < 0.1: TestCodebook in tests/test_kbit_quantization.py)
and against the closed form of the normal CDF: Phi(v) = erfc(-v / sqrt 2) / 2
from the C library, which is independent of the quantile routine used.
"""
import math

import numpy as np
import pytest


@pytest.mark.parametrize("k", [2, 3, 4, 5])
def test_codebook_properties(orc, k):
    cb = orc.normal_float_codebook(k)
    assert cb.dtype == np.float32 and cb.size == (1 << k)
    assert np.all(np.diff(cb) > 0)                      # strictly ascending
    assert np.abs(cb).max() == np.float32(1.0)          # x / x == 1 exactly in IEEE
    assert np.abs(cb + cb[::-1]).max() <= 1e-6          # symmetric about 0
    assert abs(float(cb.mean())) < 0.1


@pytest.mark.parametrize("k", [2, 3, 4, 5])
def test_quantiles_invert_the_normal_cdf(orc, k):
    n = 1 << k
    q = orc.unnormalized_quantiles(k).astype(np.float64)
    for i in range(n):
        level = (2 * i + 1) / (2 * n)
        phi = 0.5 * math.erfc(-q[i] / math.sqrt(2.0))
        dens = math.exp(-0.5 * q[i] ** 2) / math.sqrt(2 * math.pi)
        # q[i] is the float64 quantile rounded to fp32: |Phi(q) - level| <= density * half-ulp
        tol = dens * abs(q[i]) * 2.0 ** -24 + 1e-15
        assert abs(phi - level) <= tol, (k, i, phi, level)


@pytest.mark.parametrize("k", [2, 3, 4, 5])
def test_normalisation_is_one_fp32_division(orc, k):
    q = orc.unnormalized_quantiles(k)
    cb = orc.normal_float_codebook(k)
    m = np.float32(np.abs(q).max())
    from tests.exact import rn_div
    for i in range(q.size):
        assert cb[i] == rn_div(q[i], m)
