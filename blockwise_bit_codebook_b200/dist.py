"""Multi-GPU plumbing for the codec: sharding without any data-path collective.

Both operations are blockwise, so a tensor splits across ranks into
independent contiguous ranges; each rank runs the unchanged single-GPU calls
on its range and no data crosses between GPUs:

  * k-bit: ranges are whole 32-element blocks; rank r's packed words and
    absmax values are exactly the slice [start/32 * K, stop/32 * K) and
    [start/32, stop/32) of the whole-tensor outputs;
  * nested 4-bit: ranges are whole inner groups (256 outer blocks), so each
    rank reads only its own slice of absmax_q and absmax2.

The only cross-rank step is timing: the benchmark takes the maximum elapsed
time over ranks (an all-reduce of one number, off the data path).
"""
from typing import Tuple


def shard_range(n: int, rank: int, world: int, align: int) -> Tuple[int, int]:
    """Contiguous [start, stop) of n elements for `rank`, boundaries multiples of `align`.

    Units of `align` elements are dealt as evenly as possible (the first ranks get
    one extra unit); the last rank also takes the ragged tail.
    """
    if world < 1 or not (0 <= rank < world):
        raise ValueError(f"bad rank {rank} of {world}")
    if align < 1:
        raise ValueError("align must be >= 1")
    units = (n + align - 1) // align
    base, extra = divmod(units, world)
    u0 = rank * base + min(rank, extra)
    u1 = u0 + base + (1 if rank < extra else 0)
    return min(n, u0 * align), min(n, u1 * align)


def kbit_shard(n: int, rank: int, world: int) -> Tuple[int, int]:
    """Element range of a k-bit shard: whole 32-element blocks."""
    return shard_range(n, rank, world, 32)


def nested_shard(n: int, blocksize: int, rank: int, world: int, blocksize2: int = 256) -> Tuple[int, int]:
    """Element range of a nested 4-bit shard: whole inner groups (blocksize * blocksize2 elements)."""
    return shard_range(n, rank, world, blocksize * blocksize2)


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of `value` over all ranks of the default process group (identity without one)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
