"""The N>1 path on CPU: two gloo ranks (127.0.0.1).

Checks the pieces the multi-GPU benchmark relies on: per-rank batches are
distinct, timings reduce to their maximum over ranks, and the natural
partitions of the path (kv-head groups for prefill, sequences for decode)
reproduce the unsharded result exactly when gathered (computed with the
oracle, so no GPU is needed)."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from flashattention_attention_attn_b200 import dist_util, inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle import fp64_attention as orc
        f64 = lambda t: t.to(torch.float64).numpy()  # noqa: E731

        # 1. timings: max over ranks
        got = dist_util.max_over_ranks([1.0 + rank, 10.0 - rank])
        assert got == [float(world), 10.0], got

        # 2. weak-scaling batches differ per rank
        spec = inputs.PrefillSpec(B=1, Hq=8, Hkv=2, T=40, S=40, d=16, causal=True, seed=21)
        q, _, _ = inputs.make_prefill(spec, seed=dist_util.rank_seed(spec.seed, rank))
        allq = [torch.empty_like(q) for _ in range(world)]
        dist.all_gather(allq, q)
        assert not torch.equal(allq[0], allq[1])

        # 3. head-sharded prefill gathers to the unsharded result
        q, k, v = inputs.make_prefill(spec)
        (klo, khi), (qlo, qhi) = dist_util.kv_head_shard(spec.Hq, spec.Hkv, world, rank)
        O, L = orc.attention(f64(q[:, :, qlo:qhi]), f64(k[:, :, klo:khi]), f64(v[:, :, klo:khi]), spec.scale, True)
        parts = [None] * world
        dist.all_gather_object(parts, (qlo, qhi, O, L))

        # 4. sequence-sharded decode gathers to the unsharded result
        dspec = inputs.DecodeSpec(B=5, Hq=8, Hkv=2, d=16, block_size=16, max_blocks=6, ctx_lo=1, ctx_hi=96,
                                  seed=22)
        inp = inputs.make_paged(dspec)
        lo, hi = dist_util.shard_range(dspec.B, world, rank)
        Od, Ld = orc.paged_decode(f64(inp.q[lo:hi]), f64(inp.k_cache), f64(inp.v_cache),
                                  inp.block_table[lo:hi].numpy(), inp.seq_lens[lo:hi].numpy(), 16, dspec.scale)
        dparts = [None] * world
        dist.all_gather_object(dparts, (lo, hi, Od, Ld))

        if rank == 0:
            Of, Lf = orc.attention(f64(q), f64(k), f64(v), spec.scale, True)
            for qlo_, qhi_, O_, L_ in parts:
                np.testing.assert_array_equal(O_, Of[:, :, qlo_:qhi_])
                np.testing.assert_array_equal(L_, Lf[:, qlo_:qhi_])
            Odf, Ldf = orc.paged_decode(f64(inp.q), f64(inp.k_cache), f64(inp.v_cache), inp.block_table.numpy(),
                                        inp.seq_lens.numpy(), 16, dspec.scale)
            for lo_, hi_, O_, L_ in dparts:
                np.testing.assert_array_equal(O_, Odf[lo_:hi_])
                np.testing.assert_array_equal(L_, Ldf[lo_:hi_])
            open(os.path.join(out_dir, "ok"), "w").write("ok")
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    mp.spawn(_worker, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True)
    assert (tmp_path / "ok").exists()


@pytest.mark.parametrize("n,world", [(0, 2), (5, 2), (8, 3), (3, 4), (128, 8)])
def test_shard_range_partitions(n, world):
    spans = [dist_util.shard_range(n, world, r) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == n
    for (a, b), (c, _) in zip(spans, spans[1:]):
        assert b == c and b >= a
    sizes = [b - a for a, b in spans]
    assert max(sizes) - min(sizes) <= 1
