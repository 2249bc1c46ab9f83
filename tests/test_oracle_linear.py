"""Pins of the oracle's dequant-plus-linear references (the nested-dequant page's public-path
controls: a quantized weight dequantized, then a linear layer), for the nested 4-bit and the
k-bit weight. The dequants are pinned elsewhere; here the float64 matmul step is checked against
exact rational dot products on small shapes."""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from blockwise_bit_codebook_b200 import synthetic


def test_linear_matches_exact_rationals():
    M, N, K, bs = 3, 16, 128, 64
    x = synthetic.weights(M * K, std=1.0, seed=1).numpy()
    xb = oracle.f32_to_bf16_bits(x).reshape(M, K)
    w = synthetic.weights(N * K, std=0.02, seed=2).numpy()
    nf4, g8 = oracle.normal_float_codebook(4), synthetic.general8_table()
    state = oracle.quantize_4bit_nested(w, "f32", bs, nf4, g8)
    Y, S = oracle.linear_4bit_nested(xb, "bf16", N, K, state, g8, nf4, bs)
    Wb = oracle.nested_dequantize(state[0], state[1], g8, state[2], float(state[3]), nf4, N * K, bs, 256, "bf16")
    W = oracle.bf16_bits_to_f32(Wb).reshape(N, K)
    X = oracle.bf16_bits_to_f32(xb.reshape(-1)).reshape(M, K)
    for m in range(M):
        for n in range(N):
            exact = sum(Fraction(float(X[m, k])) * Fraction(float(W[n, k])) for k in range(K))
            assert abs(Fraction(float(Y[m, n])) - exact) <= Fraction(K, 2 ** 53) * Fraction(float(S[m, n]))
            assert S[m, n] == float(sum(abs(Fraction(float(X[m, k])) * Fraction(float(W[n, k]))) for k in range(K)))


@pytest.mark.parametrize("K", [2, 3, 4, 5])
def test_linear_kbit_matches_exact_rationals(K):
    M, N, Kin = 2, 16, 96
    x = synthetic.weights(M * Kin, std=1.0, seed=10 + K).numpy()
    xb = oracle.f32_to_f16_bits(x).reshape(M, Kin)
    w = synthetic.weights(N * Kin, std=0.02, seed=20 + K, outlier_frac=0.01).numpy()
    cb = oracle.normal_float_codebook(K)
    packed, absmax = oracle.kbit_quantize(w, "f32", K, cb)
    Y, S = oracle.linear_kbit(xb, "f16", N, Kin, packed, absmax, cb, K)
    W = oracle.f16_bits_to_f32(oracle.kbit_dequantize(packed, absmax, cb, K, N * Kin, "f16")).reshape(N, Kin)
    X = oracle.f16_bits_to_f32(xb.reshape(-1)).reshape(M, Kin)
    # the weight is the k-bit reconstruction codebook[idx] * absmax, rounded to fp16
    idx = oracle.kbit_unpack(packed, K, N * Kin).reshape(N, Kin)
    am = np.repeat(absmax, 32)[:N * Kin].reshape(N, Kin)
    assert np.array_equal(W, (cb[idx] * am).astype(np.float32).astype(np.float16).astype(np.float32))
    for m in range(M):
        for n in range(N):
            exact = sum(Fraction(float(X[m, k])) * Fraction(float(W[n, k])) for k in range(Kin))
            assert abs(Fraction(float(Y[m, n])) - exact) <= Fraction(Kin, 2 ** 53) * Fraction(float(S[m, n]))
