"""GPU parity of the fused dequant + linear layers (nested 4-bit and k-bit weights) against the
float64 oracle.

The fused kernel accumulates in fp32 on the tensor cores, so it is not bit-exact; the tolerance
comes from the arithmetic: every product of two 16-bit values is exact, the K additions in fp32
lose at most 2 K 2^-24 sum|x w| (twice the RN bound, allowing for the tensor core's internal
accumulation), and the result is rounded once to the activation type (half an ulp)."""
import numpy as np
import pytest
import torch

import oracle
from blockwise_bit_codebook_b200 import synthetic
from tests.gpu_util import DTYPES, to_host

pytestmark = pytest.mark.gpu
NF4 = oracle.normal_float_codebook(4)
G8 = synthetic.general8_table()


@pytest.fixture(scope="module")
def bbc():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from blockwise_bit_codebook_b200 import build
    build.build()
    import blockwise_bit_codebook_b200 as m
    m.load_library()
    return m


def run_case(bbc, M, N, K, bs, dt, seed=0):
    codes, q, a2, off = synthetic.nested_state(N * K, bs, seed=seed)
    x = synthetic.weights(M * K, std=1.0, seed=seed + 100, dtype=DTYPES[dt]).reshape(M, K)
    Y64, S = oracle.linear_4bit_nested(to_host(x), dt, N, K, (to_host(codes), to_host(q), to_host(a2), off),
                                       G8, NF4, bs)
    y = bbc.linear_4bit_nested(x.cuda(), codes.cuda(), q.cuda(), torch.from_numpy(G8).cuda(), a2.cuda(),
                               float(off), torch.from_numpy(NF4).cuda(), N, bs)
    torch.cuda.synchronize()
    got = y.float().cpu().numpy().astype(np.float64)
    acc_err = 2 * K * 2.0 ** -24 * S
    half_ulp = (2.0 ** -8 if dt == "bf16" else 2.0 ** -11) * (np.abs(Y64) + acc_err)
    err = np.abs(got - Y64)
    bound = acc_err + half_ulp + 1e-30
    assert np.all(err <= bound), (M, N, K, bs, dt, float(np.max(err / bound)))
    return float(np.max(err / bound))


@pytest.mark.parametrize("dt", ["bf16", "f16"])
@pytest.mark.parametrize("M,N", [(1, 4096), (8, 4096), (32, 4096), (32, 11008)])
def test_public_path_control_shapes(bbc, M, N, dt):
    """The page's dequantize-plus-linear controls: M = 1, 8, 32; N = 4096 / 11008; K = 4096."""
    run_case(bbc, M, N, 4096, 64, dt, seed=M)


@pytest.mark.parametrize("dt", ["bf16", "f16"])
def test_ragged_m_and_blocksizes(bbc, dt):
    # (8, 32, 8192, 64): X too large to stage in shared memory, read from global memory instead
    for M, N, K, bs in [(3, 64, 640, 64), (9, 256, 1024, 32), (17, 128, 4096, 4096), (31, 48, 192, 128),
                        (2, 16, 64, 32), (8, 32, 8192, 64), (16, 64, 2048, 256),
                        # K % 128 == 64: a 64-wide window ends every row (staged X, X from L2)
                        (1, 272, 4160, 64), (8, 48, 4160, 32), (24, 32, 1088, 128)]:
        run_case(bbc, M, N, K, bs, dt, seed=M + N)


def run_kbit_case(bbc, M, N, Kin, K, dt, seed=0):
    packed, absmax = synthetic.kbit_state(N * Kin, K, seed=seed)
    cb = oracle.normal_float_codebook(K)
    x = synthetic.weights(M * Kin, std=1.0, seed=seed + 100, dtype=DTYPES[dt]).reshape(M, Kin)
    Y64, S = oracle.linear_kbit(to_host(x), dt, N, Kin, to_host(packed), to_host(absmax), cb, K)
    y = bbc.linear_kbit(x.cuda(), packed.cuda(), absmax.cuda(), torch.from_numpy(cb).cuda(), K, N)
    torch.cuda.synchronize()
    got = y.float().cpu().numpy().astype(np.float64)
    acc_err = 2 * Kin * 2.0 ** -24 * S
    half_ulp = (2.0 ** -8 if dt == "bf16" else 2.0 ** -11) * (np.abs(Y64) + acc_err)
    bound = acc_err + half_ulp + 1e-30
    assert np.all(np.abs(got - Y64) <= bound), (M, N, Kin, K, dt, float(np.max(np.abs(got - Y64) / bound)))


@pytest.mark.parametrize("K", [2, 3, 4, 5])
@pytest.mark.parametrize("M", [1, 8, 32])
def test_kbit_control_shapes(bbc, M, K):
    """The public-path control shapes (N = K = 4096) with a k-bit weight, every code width."""
    run_kbit_case(bbc, M, 4096, 4096, K, "bf16", seed=M * 10 + K)


@pytest.mark.parametrize("dt", ["bf16", "f16"])
def test_kbit_ragged_shapes(bbc, dt):
    # staged X with 128-wide windows, X from L2 with 64-wide windows, 64-wide row tails, n-tiles 1..4
    cases = [(3, 64, 640), (9, 256, 1024), (17, 128, 4096), (31, 48, 192), (2, 16, 64), (8, 32, 8192),
             (1, 272, 4160), (8, 48, 4160), (24, 32, 1088), (16, 64, 2048)]
    for i, (M, N, Kin) in enumerate(cases):
        run_kbit_case(bbc, M, N, Kin, 2 + i % 4, dt, seed=i)


def test_invalid_arguments(bbc):
    from blockwise_bit_codebook_b200 import BBCError
    x = torch.zeros(33, 64, dtype=torch.bfloat16, device="cuda")
    z8 = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    f = torch.zeros(256, device="cuda")
    with pytest.raises(BBCError, match="N % 128"):           # M > 32: the tensor-core path
        bbc.linear_4bit_nested(x, z8, z8, f, f, 0.0, f, 16, 64)
    with pytest.raises(BBCError, match="N % 16"):
        bbc.linear_4bit_nested(x[:4], z8, z8, f, f, 0.0, f, 24, 64)
    with pytest.raises(BBCError, match="K % 64"):
        bbc.linear_4bit_nested(x[:4, :48].contiguous(), z8, z8, f, f, 0.0, f, 16, 64)
    with pytest.raises(BBCError, match="aligned"):
        bbc.linear_4bit_nested(x[:4], z8[1:], z8, f, f, 0.0, f, 16, 64)
    with pytest.raises(BBCError, match="aligned"):
        bbc.linear_4bit_nested(x[:4], z8[8:], z8, f, f, 0.0, f, 16, 64)
    with pytest.raises(BBCError, match="fp16 or bf16"):
        bbc.linear_4bit_nested(x[:4].float(), z8, z8, f, f, 0.0, f, 16, 64)


def test_kbit_invalid_arguments(bbc):
    from blockwise_bit_codebook_b200 import BBCError
    x = torch.zeros(4, 64, dtype=torch.bfloat16, device="cuda")
    pk = torch.zeros(4096, dtype=torch.int32, device="cuda")
    f = torch.zeros(256, device="cuda")
    with pytest.raises(BBCError, match="bits"):
        bbc.linear_kbit(x, pk, f, f, 6, 16)
    with pytest.raises(BBCError, match="N % 128"):
        bbc.linear_kbit(torch.zeros(33, 64, dtype=torch.bfloat16, device="cuda"), pk, f, f, 4, 16)
    with pytest.raises(BBCError, match="aligned"):
        bbc.linear_kbit(x, pk[2:], f, f, 4, 16)
    with pytest.raises(BBCError, match="blocksize"):
        bbc.linear_kbit(x, pk, f, f, 4, 16, blocksize=64)
