"""Parity of the sm_100a paged decode (paged_attn_decode through the C ABI)
with the fp64 oracle, split invariance and block-table bit-exactness."""

import pytest
import torch

from flashattention_attention_attn_b200 import inputs
from tests._parity import check_close, f64, oracle_decode, run_decode

pytestmark = pytest.mark.gpu


def test_paged_decode_workload_b64():
    inp = inputs.make_paged(inputs.WORKLOADS["paged_decode_b64"])
    o = run_decode(inp)
    O, _ = oracle_decode(inp)
    check_close(f64(o), O, what="paged_decode_b64")


def test_long_decode_workload_131k():
    inp = inputs.make_paged(inputs.WORKLOADS["long_decode_131k"])
    o = run_decode(inp)
    O, _ = oracle_decode(inp)
    check_close(f64(o), O, what="long_decode_131k")


@pytest.mark.parametrize("splits", [1, 2, 7, 0])
def test_split_counts_agree_with_oracle(splits):
    spec = inputs.DecodeSpec(B=6, Hq=32, Hkv=8, d=128, block_size=16, max_blocks=40, ctx_lo=1, ctx_hi=640,
                             seed=11)
    inp = inputs.make_paged(spec)
    o = run_decode(inp, num_splits=splits)
    O, _ = oracle_decode(inp)
    check_close(f64(o), O, what=f"splits={splits}")


@pytest.mark.parametrize("splits", [1, 5, 0])
def test_block_permutation_is_bit_exact(splits):
    spec = inputs.DecodeSpec(B=8, Hq=32, Hkv=8, d=128, block_size=16, max_blocks=64, ctx_lo=100, ctx_hi=1024,
                             seed=12, extra_pool_blocks=9)
    a = inputs.make_paged(spec)
    b = inputs.permute_pool(a, seed=99)
    assert not torch.equal(a.block_table, b.block_table)
    oa = run_decode(a, num_splits=splits)
    ob = run_decode(b, num_splits=splits)
    assert torch.equal(oa, ob)


@pytest.mark.parametrize("Hq,Hkv,d", [(32, 8, 64), (8, 8, 128), (16, 2, 128), (24, 6, 128), (8, 1, 64),
                                      (12, 12, 128)])
def test_head_layouts(Hq, Hkv, d):
    spec = inputs.DecodeSpec(B=3, Hq=Hq, Hkv=Hkv, d=d, block_size=16, max_blocks=20, ctx_lo=1, ctx_hi=320,
                             seed=13 + Hq + Hkv)
    inp = inputs.make_paged(spec)
    o = run_decode(inp)
    O, _ = oracle_decode(inp)
    check_close(f64(o), O, what=f"Hq{Hq} Hkv{Hkv} d{d}")


def test_edge_lengths():
    """Empty sequence, one token, exactly one block, one past a block, full table."""
    lens = [0, 1, 16, 17, 31, 32 * 16]
    spec = inputs.DecodeSpec(B=len(lens), Hq=32, Hkv=8, d=128, block_size=16, max_blocks=32, ctx_lo=0,
                             ctx_hi=0, seed=14)
    inp = inputs.make_paged(spec, seq_lens=lens)
    for splits in (1, 3, 0):
        o = run_decode(inp, num_splits=splits)
        O, _ = oracle_decode(inp)
        check_close(f64(o), O, what=f"edge splits={splits}")
        assert torch.all(o[0] == 0)


def test_garbage_past_sequence_end_is_ignored():
    """Slots of the last block past seq_len hold NaN: the result is unchanged."""
    lens = [5, 23, 40]
    spec = inputs.DecodeSpec(B=3, Hq=32, Hkv=8, d=128, block_size=16, max_blocks=4, ctx_lo=0, ctx_hi=0,
                             seed=15)
    inp = inputs.make_paged(spec, seq_lens=lens)
    ref = run_decode(inp)
    for b, L in enumerate(lens):
        last = int(inp.block_table[b, (L - 1) // 16])
        inp.k_cache[last, L % 16 or 16:] = float("nan")
        inp.v_cache[last, L % 16 or 16:] = float("nan")
    o = run_decode(inp)
    assert torch.equal(o, ref)
    O, _ = oracle_decode(inp)
    check_close(f64(o), O, what="nan tail")


@pytest.mark.parametrize("splits,max_blocks", [(9, 128), (17, 128), (33, 128), (65, 128), (128, 128),
                                               (129, 320), (320, 320)])
def test_many_splits_every_combine_shape(splits, max_blocks):
    """Split counts that select 1, 2, 4, 8, 16 and 32 warps per merged row;
    320 splits take a 32-warp row through two rounds of 8 splits per warp."""
    lens = [0, 5, 700, 2047, 16 * max_blocks, 1300, 16, 33]
    spec = inputs.DecodeSpec(B=len(lens), Hq=32, Hkv=8, d=128, block_size=16, max_blocks=max_blocks, ctx_lo=0,
                             ctx_hi=0, seed=16)
    inp = inputs.make_paged(spec, seq_lens=lens)
    o = run_decode(inp, num_splits=splits)
    O, _ = oracle_decode(inp)
    check_close(f64(o), O, what=f"splits={splits}")
    assert torch.all(o[0] == 0)
