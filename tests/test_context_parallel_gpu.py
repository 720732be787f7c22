"""Context-parallel decode on the CUDA path: paged_attn_decode_partial over a
share of every sequence's cached tokens and attn_lse_merge of the shares.

A multi-GPU run gives each rank one share and all-gathers the partials
before the merge.  Here the ranks are independent launches on one GPU, each
over its own share (from dist_util.context_shard); their partials are
stacked as the all-gather would stack them and merged.  The partials and
the merged output are compared with the fp64 oracle (the oracle's merge of
its own partials is pinned in test_oracle_pins.py; the all-gather itself
runs on two gloo ranks in test_multi_rank_gloo.py)."""

import math
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch

from flashattention_attention_attn_b200 import dist_util, inputs
from oracle import fp64_attention as orc
from tests._parity import check_close, f64, oracle_decode, run_decode

pytestmark = pytest.mark.gpu


class _Dev:
    """The inputs of a decode, on the GPU once."""

    def __init__(self, inp):
        self.inp = inp
        self.q, self.k, self.v = inp.q.cuda(), inp.k_cache.cuda(), inp.v_cache.cuda()
        self.B, self.Hq, self.d = inp.q.shape
        self.Hkv = inp.k_cache.shape[2]
        self.pool = inp.k_cache.shape[0]


def run_partial(dev, table, lens, num_splits=0):
    import flashattention_attention_attn_b200 as fa
    o = torch.full((dev.B, dev.Hq, dev.d), float("nan"), device="cuda", dtype=torch.float32)
    lse = torch.full((dev.B, dev.Hq), float("nan"), device="cuda", dtype=torch.float32)
    fa.paged_attn_decode_partial(dev.q, dev.k, dev.v, table.cuda(), lens.cuda(), dev.B, dev.Hq, dev.Hkv, dev.d, 16,
                                 table.shape[1], dev.pool, num_splits, o, lse)
    torch.cuda.synchronize()
    assert fa.attn_read_device_status(clear=True) == 0
    return o, lse


def run_merge(parts_o, parts_lse):
    import flashattention_attention_attn_b200 as fa
    R, B, Hq, d = parts_o.shape
    o = torch.full((B, Hq, d), float("nan"), device="cuda", dtype=torch.bfloat16)
    fa.attn_lse_merge(parts_o.cuda().contiguous(), parts_lse.cuda().contiguous(), R, B, Hq, d, o)
    torch.cuda.synchronize()
    return o.cpu()


def oracle_share(inp, table, lens):
    d = inp.q.shape[-1]
    return orc.paged_decode(f64(inp.q), f64(inp.k_cache), f64(inp.v_cache), table.numpy(), lens.numpy(), 16,
                            1.0 / math.sqrt(d))


@pytest.mark.parametrize("splits", [1, 7, 0])
def test_partial_over_all_keys_rounds_to_the_decode(splits):
    """One share holding everything: o_part is the decode's output before its
    bf16 rounding (same kernels, same split count), lse the oracle's."""
    inp = inputs.make_paged(inputs.WORKLOADS["paged_decode_b64"])
    dev = _Dev(inp)
    o, lse = run_partial(dev, inp.block_table, inp.seq_lens, splits)
    assert torch.equal(o.to(torch.bfloat16).cpu(), run_decode(inp, num_splits=splits))
    O, L = oracle_decode(inp)
    check_close(f64(o), O, f64(lse), L, what=f"all keys, splits={splits}")


@pytest.mark.parametrize("d,splits", [(128, 1), (128, 3), (128, 0), (64, 1), (64, 0)])
def test_partial_edges_agree_with_oracle(d, splits):
    lens = [0, 1, 15, 16, 17, 300, 0, 640]
    spec = inputs.DecodeSpec(B=len(lens), Hq=16, Hkv=4, d=d, block_size=16, max_blocks=40, ctx_lo=0, ctx_hi=0,
                             seed=81)
    inp = inputs.make_paged(spec, seq_lens=lens)
    o, lse = run_partial(_Dev(inp), inp.block_table, inp.seq_lens, splits)
    O, L = oracle_decode(inp)
    check_close(f64(o), O, f64(lse), L, what=f"edges d={d} splits={splits}")
    for b in (0, 6):  # no key: o = 0 exactly, lse = -inf
        assert torch.all(o[b] == 0) and torch.all(torch.isneginf(lse[b]))


@pytest.mark.parametrize("world", [2, 3, 4])
def test_emulated_ranks_merge_to_the_full_decode(world):
    inp = inputs.make_paged(inputs.WORKLOADS["paged_decode_b64"])
    dev = _Dev(inp)
    po, pl = [], []
    for rank in range(world):
        table, lens, _ = dist_util.context_shard(inp.block_table, inp.seq_lens, world, rank)
        o, lse = run_partial(dev, table, lens)
        if rank == world - 1:  # one share against the oracle on that share
            Os, Ls = oracle_share(inp, table, lens)
            check_close(f64(o), Os, f64(lse), Ls, what=f"share {rank} of {world}")
        po.append(o)
        pl.append(lse)
    out = run_merge(torch.stack(po), torch.stack(pl))
    O, _ = oracle_decode(inp)
    check_close(f64(out), O, what=f"merged over {world} shares")


def test_emulated_ranks_long_context_131k():
    """One 131,072-token sequence over 4 shares of 2048 blocks each."""
    inp = inputs.make_paged(inputs.WORKLOADS["long_decode_131k"])
    dev = _Dev(inp)
    po, pl = [], []
    for rank in range(4):
        table, lens, lo = dist_util.context_shard(inp.block_table, inp.seq_lens, 4, rank)
        assert int(lens[0]) == 32768 and int(lo[0]) == 2048 * rank
        o, lse = run_partial(dev, table, lens)
        po.append(o)
        pl.append(lse)
    out = run_merge(torch.stack(po), torch.stack(pl))
    O, _ = oracle_decode(inp)
    check_close(f64(out), O, what="131k over 4 shares")


@pytest.mark.parametrize("R,d", [(1, 128), (2, 64), (9, 128), (40, 128), (300, 128), (300, 64)])
def test_merge_of_given_partials_agrees_with_oracle(R, d):
    """attn_lse_merge on partials drawn directly: lse spread over 16 nats,
    some -inf, rows where every part is -inf; 300 parts take the widest
    merge through two rounds."""
    g = torch.Generator().manual_seed(82 + R + d)
    B, Hq = 3, 8
    po = torch.randn(R, B, Hq, d, generator=g)
    pl = torch.rand(R, B, Hq, generator=g) * 16.0 - 8.0
    pl[torch.rand(R, B, Hq, generator=g) < 0.25] = -math.inf
    pl[:, 1, 2] = -math.inf  # no key in any part
    pl[0, 2, :] = pl[:, 2, :].max(dim=0).values + 3.0  # a dominant part
    out = run_merge(po, pl)
    O, L = orc.merge_partials(po.double().numpy(), pl.double().numpy())
    check_close(f64(out), O, what=f"merge R={R} d={d}")
    assert torch.all(out[1, 2] == 0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_context_parallel_decode_in_a_one_rank_group():
    """dist_util.context_parallel_decode end to end (partial, all-gather over
    NCCL, merge) in a process group of one rank."""
    code = f"""
import os, sys, datetime
sys.path.insert(0, {os.getcwd()!r})
import torch, torch.distributed as dist
from flashattention_attention_attn_b200 import dist_util, inputs
from tests._parity import check_close, f64, oracle_decode
os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT="{_free_port()}")
torch.cuda.set_device(0)
dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60))
try:
    spec = inputs.DecodeSpec(B=6, Hq=32, Hkv=8, d=128, block_size=16, max_blocks=64, ctx_lo=0, ctx_hi=1024, seed=83)
    inp = inputs.make_paged(spec)
    table, lens, _ = dist_util.context_shard(inp.block_table.cuda(), inp.seq_lens.cuda(), 1, 0)
    o = dist_util.context_parallel_decode(inp.q.cuda(), inp.k_cache.cuda(), inp.v_cache.cuda(), table, lens,
                                          inp.k_cache.shape[0])
    torch.cuda.synchronize()
    O, _ = oracle_decode(inp)
    check_close(f64(o), O, what="context_parallel_decode")
    print("ok")
finally:
    dist.destroy_process_group()
"""
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout[-2000:] + r.stderr[-2000:]
