"""Parity of attn_fwd_varlen (packed sequences, no padding) with the fp64
oracle, and bit-identity with attn_fwd for a single sequence."""

import pytest
import torch

from flashattention_attention_attn_b200 import inputs
from tests._parity import check_close, f64, oracle_varlen, run_prefill, run_varlen

pytestmark = pytest.mark.gpu


def _spec(B, Hq=32, Hkv=8, d=128, causal=True, seed=0):
    return inputs.VarlenSpec(B=B, Hq=Hq, Hkv=Hkv, d=d, len_lo=1, len_hi=1, causal=causal, seed=seed)


@pytest.mark.parametrize("causal", [True, False])
def test_ragged_self_attention(causal):
    lens = [1, 127, 128, 129, 300, 513, 0, 1000, 256, 40]
    spec = _spec(len(lens), causal=causal, seed=30)
    inp = inputs.make_varlen(spec, q_lens=lens)
    o, lse = run_varlen(inp, causal, spec.scale)
    O, L = oracle_varlen(inp, causal, spec.scale)
    check_close(f64(o), O, lse.numpy(), L, what=f"varlen causal={causal}")


def test_chunked_queries_longer_keys_and_rows_without_keys():
    q_lens = [64, 200, 130, 5, 300]
    k_lens = [500, 200, 1000, 2, 100]  # T < S (bottom-right), T == S, T > S (leading rows see nothing)
    spec = _spec(len(q_lens), Hq=16, Hkv=4, seed=31)
    inp = inputs.make_varlen(spec, q_lens=q_lens, k_lens=k_lens)
    o, lse = run_varlen(inp, True, spec.scale)
    O, L = oracle_varlen(inp, True, spec.scale)
    check_close(f64(o), O, lse.numpy(), L, what="varlen chunked")


@pytest.mark.parametrize("B", [32, 40])
def test_many_sequences_both_grids(B):
    # up to 32 sequences: one CTA per (head, 256-row query block that exists);
    # more: the full grid, whose CTAs past a sequence's end exit at once
    g = torch.Generator().manual_seed(34 + B)
    lens = [int(x) for x in torch.randint(0, 600, (B,), generator=g)]
    lens[0], lens[5], lens[-1] = 0, 256, 257
    spec = _spec(B, Hq=8, Hkv=2, seed=34 + B)
    inp = inputs.make_varlen(spec, q_lens=lens)
    o, lse = run_varlen(inp, True, spec.scale)
    O, L = oracle_varlen(inp, True, spec.scale)
    check_close(f64(o), O, lse.numpy(), L, what=f"varlen B={B}")
    # a max_seqlen_q above the true maximum changes nothing
    o2, lse2 = run_varlen(inp, True, spec.scale, max_q=inp.max_q + 700)
    assert torch.equal(o, o2) and torch.equal(lse, lse2)


def test_head_dim_64_mha():
    lens = [77, 260, 129]
    spec = _spec(len(lens), Hq=8, Hkv=8, d=64, seed=32)
    inp = inputs.make_varlen(spec, q_lens=lens)
    o, lse = run_varlen(inp, True, spec.scale)
    O, L = oracle_varlen(inp, True, spec.scale)
    check_close(f64(o), O, lse.numpy(), L, what="varlen d64")


def test_varlen_workload():
    spec = inputs.VARLEN_WORKLOADS["varlen_prefill_16seq"]
    inp = inputs.make_varlen(spec)
    o, lse = run_varlen(inp, True, spec.scale)
    O, L = oracle_varlen(inp, True, spec.scale)
    check_close(f64(o), O, lse.numpy(), L, what="varlen_prefill_16seq")


def test_single_sequence_matches_dense_bit_for_bit():
    spec = inputs.PrefillSpec(B=1, Hq=8, Hkv=2, T=700, S=700, d=128, causal=True, seed=33)
    q, k, v = inputs.make_prefill(spec)
    od, ld = run_prefill(q, k, v, True, spec.scale)
    inp = inputs.VarlenInputs(q=q[0].contiguous(), k=k[0].contiguous(), v=v[0].contiguous(),
                              cu_q=torch.tensor([0, 700], dtype=torch.int32),
                              cu_k=torch.tensor([0, 700], dtype=torch.int32))
    ov, lv = run_varlen(inp, True, spec.scale)
    assert torch.equal(ov, od[0]) and torch.equal(lv, ld[0])
