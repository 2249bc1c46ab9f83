"""Multi-rank host logic on CPU (gloo, world size 2): sharding needs no collective.

Each rank quantizes its own block-aligned shard with the CPU oracle; the
gathered shards must equal the whole-tensor result bit for bit, and the
benchmark's max-over-ranks timing reduction must return the largest value.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from blockwise_bit_codebook_b200.dist import kbit_shard, nested_shard, shard_range


def test_shard_ranges_cover_and_align():
    for n in [1, 31, 32, 33, 1000, 32 * 1000 + 7, 10**6 + 3]:
        for world in [1, 2, 3, 4, 8]:
            rs = [kbit_shard(n, r, world) for r in range(world)]
            assert rs[0][0] == 0 and rs[-1][1] == n
            for (a0, a1), (b0, b1) in zip(rs, rs[1:]):
                assert a1 == b0
            for a0, a1 in rs:
                assert a0 <= a1
                if a0 < a1:                      # empty shards sit at n
                    assert a0 % 32 == 0
                    assert a1 % 32 == 0 or a1 == n
    s0, s1 = nested_shard(8192 * 8192 + 37, 64, 1, 2)
    assert s0 % (64 * 256) == 0
    with pytest.raises(ValueError):
        shard_range(10, 2, 2, 4)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, n, K, result_dir):
    import torch
    import torch.distributed as dist

    import oracle
    from blockwise_bit_codebook_b200 import synthetic
    from blockwise_bit_codebook_b200.dist import kbit_shard, max_over_ranks

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x = synthetic.weights(n, std=0.02, seed=1).numpy()
        cb = oracle.normal_float_codebook(K)
        s0, s1 = kbit_shard(n, rank, world)
        packed, absmax = oracle.kbit_quantize(x[s0:s1], "f32", K, cb)
        np.save(os.path.join(result_dir, f"packed{rank}.npy"), packed)
        np.save(os.path.join(result_dir, f"absmax{rank}.npy"), absmax)
        m = max_over_ranks(float(rank + 1) * 1.5)
        np.save(os.path.join(result_dir, f"max{rank}.npy"), np.array([m]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo(tmp_path):
    import oracle
    from blockwise_bit_codebook_b200 import synthetic
    world, n, K = 2, 32 * 4099 + 13, 4
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, n, K, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    x = synthetic.weights(n, std=0.02, seed=1).numpy()
    ref_p, ref_a = oracle.kbit_quantize(x, "f32", K, oracle.normal_float_codebook(K))
    got_p = np.concatenate([np.load(tmp_path / f"packed{r}.npy") for r in range(world)])
    got_a = np.concatenate([np.load(tmp_path / f"absmax{r}.npy") for r in range(world)])
    assert np.array_equal(got_p, ref_p) and np.array_equal(got_a, ref_a)
    for r in range(world):
        assert np.load(tmp_path / f"max{r}.npy")[0] == 3.0
