"""Helpers for running the path on several GPUs, one process per GPU.

The path shards without any exchange: prefill heads (by kv-head group) and
batches are independent, and so are decode sequences.  The benchmark runs
weak-scaling replicas (every rank its own seeded batch) and reduces only
its timings.

One partition does need an exchange: a context-parallel decode, where every
rank holds part of each sequence's cached tokens.  Each rank attends the
(replicated) query to its own tokens (paged_attn_decode_partial), the ranks
all-gather the fp32 partials (o, lse) in one collective, and every rank
merges them (attn_lse_merge).  The exchange is B * Hq * (d + 1) fp32 per
rank.
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


def context_shard(block_table, seq_lens, world: int, rank: int, block_size: int = 16):
    """Rank `rank`'s share of a context-parallel decode.

    Sequence b of L_b tokens (clamped to what its table row can name) has
    nb_b = ceil(L_b / block_size) logical blocks; the rank takes the
    contiguous blocks [lo_b, hi_b) = shard_range(nb_b, world, rank), so every
    rank holds about nb_b / world of them.  Returns (table [B, W] int32 with
    the block ids of the share in order, -1 past it; lens [B] int32 = tokens
    of the share; lo [B] int64 = first logical block), on the table's device.
    The shares of all ranks cover every position of every sequence once.
    """
    import torch

    B, max_blocks = block_table.shape
    dev = block_table.device
    L = seq_lens.to(device=dev, dtype=torch.int64).clamp(0, max_blocks * block_size)
    nb = (L + block_size - 1) // block_size
    q, r = nb // world, nb % world
    lo = rank * q + torch.clamp(r, max=rank)
    hi = lo + q + (r > rank).to(torch.int64)
    width = max(int((hi - lo).max()) if B > 0 else 0, 1)
    cols = lo[:, None] + torch.arange(width, device=dev)[None, :]
    inside = cols < hi[:, None]
    ids = block_table.gather(1, cols.clamp(max=max_blocks - 1))
    table = torch.where(inside, ids, torch.full_like(ids, -1)).to(torch.int32).contiguous()
    lens = (torch.minimum(L, hi * block_size) - lo * block_size).clamp(min=0).to(torch.int32).contiguous()
    return table, lens, lo


def gather_partials(o_part, lse_part, group=None):
    """All-gather every rank's partial (o [B, Hq, d], lse [B, Hq]) in one
    collective; returns ([R, B, Hq, d], [R, B, Hq]) in rank order."""
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    flat = torch.cat([o_part.reshape(-1), lse_part.reshape(-1)])
    bufs = [torch.empty_like(flat) for _ in range(world)]
    dist.all_gather(bufs, flat, group=group)
    allp = torch.stack(bufs)
    n = o_part.numel()
    return (allp[:, :n].reshape(world, *o_part.shape).contiguous(),
            allp[:, n:].reshape(world, *lse_part.shape).contiguous())


def context_parallel_decode(q, k_cache, v_cache, block_table, seq_lens, num_blocks: int, group=None,
                            num_splits: int = 0):
    """Context-parallel decode: q [B, Hq, d] bf16 replicated on every rank;
    k_cache / v_cache [num_blocks, block_size, Hkv, d] this rank's pool (the
    library takes 16-token blocks), block_table /
    seq_lens this rank's share of every sequence (for instance from
    context_shard).  Returns O [B, Hq, d] bf16, the same on every rank."""
    import torch
    import torch.distributed as dist

    from . import _binding

    B, Hq, d = q.shape
    block_size, Hkv = k_cache.shape[1], k_cache.shape[2]
    o_part = torch.empty(B, Hq, d, device=q.device, dtype=torch.float32)
    lse_part = torch.empty(B, Hq, device=q.device, dtype=torch.float32)
    _binding.paged_attn_decode_partial(q, k_cache, v_cache, block_table, seq_lens, B, Hq, Hkv, d, block_size,
                                       block_table.shape[1], num_blocks, num_splits, o_part, lse_part)
    parts_o, parts_lse = gather_partials(o_part, lse_part, group)
    o = torch.empty(B, Hq, d, device=q.device, dtype=torch.bfloat16)
    _binding.attn_lse_merge(parts_o, parts_lse, dist.get_world_size(group), B, Hq, d, o)
    return o
