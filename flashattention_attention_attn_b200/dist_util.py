"""Helpers for running the path on several GPUs, one process per GPU.

The path shards without any exchange: prefill heads (by kv-head group) and
batches are independent, and so are decode sequences.  The benchmark runs
weak-scaling replicas (every rank its own seeded batch) and reduces only
its timings.
"""

from __future__ import annotations


def rank_seed(base: int, rank: int) -> int:
    """Seed of rank `rank`'s batch: distinct per rank, equal to `base` on rank 0."""
    return base + 100 * rank


def shard_range(n: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous share [lo, hi) of n units for `rank` (sizes differ by <= 1)."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    q, r = divmod(n, world)
    lo = rank * q + min(rank, r)
    return lo, lo + q + (1 if rank < r else 0)


def kv_head_shard(Hq: int, Hkv: int, world: int, rank: int):
    """(kv heads, q heads) of a head-sharded prefill: whole GQA groups stay together."""
    klo, khi = shard_range(Hkv, world, rank)
    g = Hq // Hkv
    return (klo, khi), (klo * g, khi * g)


def max_over_ranks(values, device=None):
    """Element-wise max of a list of floats over all ranks (identity without a group)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()
