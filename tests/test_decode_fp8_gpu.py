"""Parity of paged_attn_decode_fp8 (e4m3 KV cache, per-tensor scales) with
the fp64 oracle evaluated on the exactly decoded cache."""

import pytest
import torch

from flashattention_attention_attn_b200 import inputs
from tests._parity import check_close, f64, oracle_decode_fp8, run_decode_fp8

pytestmark = pytest.mark.gpu


def test_fp8_workload_b64():
    inp = inputs.make_paged_fp8(inputs.WORKLOADS["paged_decode_b64"])
    O, _ = oracle_decode_fp8(inp)
    check_close(f64(run_decode_fp8(inp)), O, what="fp8 paged_decode_b64")


def test_fp8_long_context():
    inp = inputs.make_paged_fp8(inputs.WORKLOADS["long_decode_131k"], k_scale=0.5, v_scale=2.0)
    O, _ = oracle_decode_fp8(inp)
    check_close(f64(run_decode_fp8(inp)), O, what="fp8 long_decode_131k")


@pytest.mark.parametrize("Hq,Hkv,splits", [(32, 8, 1), (32, 8, 7), (8, 8, 0), (16, 2, 3), (24, 6, 0), (8, 1, 2)])
def test_fp8_heads_and_splits(Hq, Hkv, splits):
    lens = [0, 1, 15, 16, 17, 200, 511]
    spec = inputs.DecodeSpec(B=len(lens), Hq=Hq, Hkv=Hkv, d=128, block_size=16, max_blocks=32, ctx_lo=0, ctx_hi=0,
                             seed=70 + Hq + Hkv)
    inp = inputs.make_paged_fp8(spec, seq_lens=lens)
    o = run_decode_fp8(inp, num_splits=splits)
    O, _ = oracle_decode_fp8(inp)
    check_close(f64(o), O, what=f"fp8 Hq{Hq} Hkv{Hkv} splits{splits}")
    assert torch.all(o[0] == 0)


def test_fp8_permutation_bit_exact_and_nan_tail():
    lens = [37, 300, 1000, 16]
    spec = inputs.DecodeSpec(B=4, Hq=32, Hkv=8, d=128, block_size=16, max_blocks=64, ctx_lo=0, ctx_hi=0, seed=75,
                             extra_pool_blocks=5)
    a = inputs.make_paged_fp8(spec, seq_lens=lens)
    oa = run_decode_fp8(a, num_splits=4)
    pb = inputs.permute_pool(inputs.PagedInputs(q=a.q, k_cache=a.k_cache, v_cache=a.v_cache,
                                                block_table=a.block_table, seq_lens=a.seq_lens, block_size=16), 9)
    b = inputs.PagedInputsFp8(q=a.q, k_cache=pb.k_cache, v_cache=pb.v_cache, block_table=pb.block_table,
                              seq_lens=a.seq_lens, block_size=16, k_scale=a.k_scale, v_scale=a.v_scale)
    assert torch.equal(run_decode_fp8(b, num_splits=4), oa)
    for i, L in enumerate(lens):  # e4m3 NaN (0x7f) in the slots past each sequence end
        last = int(b.block_table[i, (L - 1) // 16])
        b.k_cache[last, L % 16 or 16:] = 0x7F
        b.v_cache[last, L % 16 or 16:] = 0x7F
    assert torch.equal(run_decode_fp8(b, num_splits=4), oa)
