"""Pins of the oracle's dequant-plus-linear reference (the nested-dequant page's public-path
controls: 4-bit weight dequantized, then a linear layer). The dequant is pinned elsewhere; here
the float64 matmul step is checked against exact rational dot products on small shapes."""
from fractions import Fraction

import numpy as np

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
