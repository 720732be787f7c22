"""The natural partitions of the path, run on the CUDA path of one GPU.

A multi-GPU run would give each rank one share: a group of whole kv heads
(with their query heads) of a prefill, or a range of sequences of a decode
or of a packed batch.  Here every share is launched on its own slice and the
gathered outputs must equal the unsharded launch bit for bit: no result of
the kernels may depend on the heads or sequences around it.  (The same
partitions are checked with the oracle on two gloo ranks in
test_multi_rank_gloo.py.)"""

import pytest
import torch

from flashattention_attention_attn_b200 import dist_util, inputs
from tests._parity import run_decode, run_decode_fp8, run_prefill, run_varlen

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world", [2, 4])
def test_kv_head_shards_equal_unsharded_prefill(world):
    spec = inputs.PrefillSpec(B=2, Hq=32, Hkv=8, T=700, S=700, d=128, causal=True, seed=71)
    q, k, v = inputs.make_prefill(spec)
    o_full, lse_full = run_prefill(q, k, v, True, spec.scale)
    for rank in range(world):
        (klo, khi), (qlo, qhi) = dist_util.kv_head_shard(spec.Hq, spec.Hkv, world, rank)
        o, lse = run_prefill(q[:, :, qlo:qhi].contiguous(), k[:, :, klo:khi].contiguous(),
                             v[:, :, klo:khi].contiguous(), True, spec.scale)
        assert torch.equal(o, o_full[:, :, qlo:qhi]), f"rank {rank}: O differs"
        assert torch.equal(lse, lse_full[:, qlo:qhi]), f"rank {rank}: LSE differs"


@pytest.mark.parametrize("world", [2, 3])
def test_batch_shards_equal_unsharded_prefill(world):
    spec = inputs.PrefillSpec(B=5, Hq=8, Hkv=2, T=300, S=300, d=64, causal=True, seed=72)
    q, k, v = inputs.make_prefill(spec)
    o_full, lse_full = run_prefill(q, k, v, True, spec.scale)
    for rank in range(world):
        lo, hi = dist_util.shard_range(spec.B, world, rank)
        o, lse = run_prefill(q[lo:hi], k[lo:hi], v[lo:hi], True, spec.scale)
        assert torch.equal(o, o_full[lo:hi]) and torch.equal(lse, lse_full[lo:hi]), f"rank {rank}"


def _slice_paged(inp, lo, hi):
    return inputs.PagedInputs(q=inp.q[lo:hi].contiguous(), k_cache=inp.k_cache, v_cache=inp.v_cache,
                              block_table=inp.block_table[lo:hi].contiguous(),
                              seq_lens=inp.seq_lens[lo:hi].contiguous(), block_size=inp.block_size)


@pytest.mark.parametrize("world,splits", [(2, 7), (4, 1), (3, 5)])
def test_sequence_shards_equal_unsharded_decode(world, splits):
    inp = inputs.make_paged(inputs.WORKLOADS["paged_decode_b64"])
    o_full = run_decode(inp, num_splits=splits)
    for rank in range(world):
        lo, hi = dist_util.shard_range(inp.q.shape[0], world, rank)
        o = run_decode(_slice_paged(inp, lo, hi), num_splits=splits)
        assert torch.equal(o, o_full[lo:hi]), f"rank {rank}: O differs"


def test_sequence_shards_equal_unsharded_decode_fp8():
    spec = inputs.DecodeSpec(B=12, Hq=32, Hkv=8, d=128, block_size=16, max_blocks=80, ctx_lo=1, ctx_hi=1280,
                             seed=73)
    inp = inputs.make_paged_fp8(spec)
    o_full = run_decode_fp8(inp, num_splits=4)
    for rank in range(2):
        lo, hi = dist_util.shard_range(spec.B, 2, rank)
        part = inputs.PagedInputsFp8(q=inp.q[lo:hi].contiguous(), k_cache=inp.k_cache, v_cache=inp.v_cache,
                                     block_table=inp.block_table[lo:hi].contiguous(),
                                     seq_lens=inp.seq_lens[lo:hi].contiguous(), block_size=inp.block_size,
                                     k_scale=inp.k_scale, v_scale=inp.v_scale)
        assert torch.equal(run_decode_fp8(part, num_splits=4), o_full[lo:hi]), f"rank {rank}: O differs"


def test_sequence_shards_equal_unsharded_varlen():
    spec = inputs.VARLEN_WORKLOADS["varlen_prefill_16seq"]
    inp = inputs.make_varlen(spec)
    o_full, lse_full = run_varlen(inp, True, spec.scale)
    for rank in range(2):
        lo, hi = dist_util.shard_range(spec.B, 2, rank)
        q0, q1 = int(inp.cu_q[lo]), int(inp.cu_q[hi])
        k0, k1 = int(inp.cu_k[lo]), int(inp.cu_k[hi])
        part = inputs.VarlenInputs(q=inp.q[q0:q1].contiguous(), k=inp.k[k0:k1].contiguous(),
                                   v=inp.v[k0:k1].contiguous(), cu_q=(inp.cu_q[lo:hi + 1] - q0).contiguous(),
                                   cu_k=(inp.cu_k[lo:hi + 1] - k0).contiguous())
        o, lse = run_varlen(part, True, spec.scale)
        assert torch.equal(o, o_full[q0:q1]), f"rank {rank}: O differs"
        assert torch.equal(lse, lse_full[:, q0:q1]), f"rank {rank}: LSE differs"
