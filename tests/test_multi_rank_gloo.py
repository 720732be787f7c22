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

        # 5. context-parallel decode: every rank attends to its share of every
        #    sequence, the partials are all-gathered (one collective) and merged
        cinp = inputs.make_paged(inputs.DecodeSpec(B=4, Hq=8, Hkv=2, d=16, block_size=16, max_blocks=9, ctx_lo=0,
                                                   ctx_hi=140, seed=23))
        ctab, clens, _ = dist_util.context_shard(cinp.block_table, cinp.seq_lens, world, rank)
        Oc, Lc = orc.paged_decode(f64(cinp.q), f64(cinp.k_cache), f64(cinp.v_cache), ctab.numpy(), clens.numpy(),
                                  16, 0.25)
        po, pl = dist_util.gather_partials(torch.from_numpy(Oc), torch.from_numpy(Lc))
        assert po.shape == (world,) + Oc.shape and pl.shape == (world,) + Lc.shape
        np.testing.assert_array_equal(po[rank].numpy(), Oc)
        Om, Lm = orc.merge_partials(po.numpy(), pl.numpy())
        Ofull, Lfull = orc.paged_decode(f64(cinp.q), f64(cinp.k_cache), f64(cinp.v_cache),
                                        cinp.block_table.numpy(), cinp.seq_lens.numpy(), 16, 0.25)
        np.testing.assert_allclose(Om, Ofull, rtol=0, atol=1e-12)
        np.testing.assert_allclose(Lm, Lfull, rtol=0, atol=1e-12)

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


@pytest.mark.parametrize("world", [1, 2, 3, 5, 8])
def test_context_shares_cover_every_position_once(world):
    lens = torch.tensor([0, 1, 15, 16, 17, 100, 160, 144, 999], dtype=torch.int32)  # 999: past the row, clamped
    table = torch.arange(9 * 10, dtype=torch.int32).reshape(9, 10) * 7 + 3
    seen = {b: [] for b in range(len(lens))}
    for r in range(world):
        t, n, lo = dist_util.context_shard(table, lens, world, r)
        assert t.dtype == torch.int32 and n.dtype == torch.int32 and t.shape[0] == len(lens)
        for b in range(len(lens)):
            nb = (int(n[b]) + 15) // 16
            assert torch.all(t[b, nb:] == -1)
            for p in range(int(n[b])):  # local position p is global position lo*16 + p
                g = int(lo[b]) * 16 + p
                assert int(t[b, p // 16]) == int(table[b, g // 16]) and p % 16 == g % 16
                seen[b].append(g)
    for b in range(len(lens)):
        L = min(int(lens[b]), 160)
        assert sorted(seen[b]) == list(range(L)), b
