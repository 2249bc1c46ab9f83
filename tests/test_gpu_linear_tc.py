"""GPU parity of the fused dequant + linear layers for M > 32 (the tensor-core path: tcgen05 with
accumulators in tensor memory, weight tiles decoded into shared memory, activation tiles by TMA,
K split over a thread-block cluster when there are few output tiles) against the float64 oracle,
within the same derived bound as the M <= 32 path (exact 16-bit products, fp32 sums: at most
2 K 2^-24 sum|x w|, then one rounding to the activation type). Every call must also leave the
device's count of bounded waits that gave up at zero."""
import pytest
import torch

from tests.test_gpu_linear import bbc, run_case, run_kbit_case  # noqa: F401

pytestmark = pytest.mark.gpu


def _no_timeouts(bbc):
    assert bbc.bbc_wait_timeouts() == 0


@pytest.mark.parametrize("M,N,K,bs,dt", [
    (33, 128, 64, 64, "bf16"),          # one K stage, one tile: no split
    (64, 256, 512, 32, "f16"),          # 64-row activation tiles, two outer blocks per stage
    (100, 384, 1024, 128, "bf16"),      # ragged M inside a 128-row tile
    (128, 4096, 4096, 64, "bf16"),      # K split over a cluster
    (256, 4096, 4096, 64, "bf16"),      # 256-row tiles, the cluster split of the headline shape
    (300, 1024, 2048, 4096, "f16"),     # two activation tiles, the second mostly past M
    (64, 11008, 4096, 64, "bf16"),      # the N = 11008 control shape at M = 64
    (200, 128, 8192, 64, "bf16"),       # a single output tile: eight CTAs share K
    (300, 4096, 4096, 64, "bf16"),      # 2 x 32 output tiles: K split over a pair of CTAs
    (256, 11008, 4096, 64, "f16"),      # 86 row tiles of 256 activations: no split
])
def test_nested_tensor_core_path(bbc, M, N, K, bs, dt):
    run_case(bbc, M, N, K, bs, dt, seed=M + K)
    _no_timeouts(bbc)


@pytest.mark.parametrize("bits", [2, 3, 4, 5])
@pytest.mark.parametrize("M,N,K,dt", [(64, 256, 1024, "bf16"), (130, 512, 2048, "f16"), (256, 4096, 4096, "bf16")])
def test_kbit_tensor_core_path(bbc, M, N, K, dt, bits):
    run_kbit_case(bbc, M, N, K, bits, dt, seed=M * 7 + bits)
    _no_timeouts(bbc)


def test_tensor_core_path_is_deterministic(bbc):
    from blockwise_bit_codebook_b200 import synthetic
    import oracle
    M, N, K, bs = 256, 2048, 4096, 64
    codes, q, a2, off = (t.cuda() if hasattr(t, "cuda") else t for t in synthetic.nested_state(N * K, bs, seed=4))
    x = synthetic.weights(M * K, std=1.0, seed=9, dtype=torch.bfloat16, device="cuda").reshape(M, K)
    g8 = torch.from_numpy(synthetic.general8_table()).cuda()
    nf4 = torch.from_numpy(oracle.normal_float_codebook(4)).cuda()
    ys = [bbc.linear_4bit_nested(x, codes, q, g8, a2, float(off), nf4, N, bs) for _ in range(3)]
    torch.cuda.synchronize()
    for y in ys[1:]:
        assert torch.equal(y.view(torch.int16), ys[0].view(torch.int16))
    _no_timeouts(bbc)
