"""Parity of paged_attn_prefill (chunked prefill against the paged cache)
with the fp64 oracle; block-table bit-exactness; garbage past the end."""

import pytest
import torch

from flashattention_attention_attn_b200 import inputs
from tests._parity import check_close, f64, oracle_chunked, run_chunked

pytestmark = pytest.mark.gpu


def _spec(B, Hq=32, Hkv=8, d=128, max_blocks=64, seed=0):
    return inputs.ChunkedSpec(B=B, Hq=Hq, Hkv=Hkv, d=d, block_size=16, max_blocks=max_blocks, ctx_lo=1, ctx_hi=1,
                              q_lo=1, q_hi=1, seed=seed)


@pytest.mark.parametrize("causal", [True, False])
def test_ragged_chunks(causal):
    ctx = [1, 17, 128, 300, 1000, 777, 129, 40]
    ql = [1, 17, 100, 64, 300, 777, 1, 39]
    spec = _spec(len(ctx), seed=40)
    inp = inputs.make_chunked(spec, ctx_lens=ctx, q_lens=ql)
    o, lse = run_chunked(inp, causal, spec.scale)
    O, L = oracle_chunked(inp, causal, spec.scale)
    check_close(f64(o), O, lse.numpy(), L, what=f"chunked causal={causal}")


def test_d64_gqa8():
    ctx, ql = [200, 513, 90], [200, 130, 2]
    spec = _spec(3, Hq=16, Hkv=2, d=64, seed=41)
    inp = inputs.make_chunked(spec, ctx_lens=ctx, q_lens=ql)
    o, lse = run_chunked(inp, True, spec.scale)
    O, L = oracle_chunked(inp, True, spec.scale)
    check_close(f64(o), O, lse.numpy(), L, what="chunked d64")


@pytest.mark.parametrize("B", [32, 33])
def test_many_sequences_both_grids(B):
    g = torch.Generator().manual_seed(43 + B)
    ctx = [int(x) for x in torch.randint(1, 700, (B,), generator=g)]
    ql = [min(c, int(x)) for c, x in zip(ctx, torch.randint(1, 400, (B,), generator=g))]
    ctx[-1], ql[-1] = 600, 300
    spec = _spec(B, Hq=8, Hkv=2, seed=43 + B)
    inp = inputs.make_chunked(spec, ctx_lens=ctx, q_lens=ql)
    o, lse = run_chunked(inp, True, spec.scale)
    O, L = oracle_chunked(inp, True, spec.scale)
    check_close(f64(o), O, lse.numpy(), L, what=f"chunked B={B}")


def test_block_permutation_bit_exact_and_nan_tail():
    ctx, ql = [250, 333, 1000], [90, 333, 257]
    spec = _spec(3, seed=42)
    a = inputs.make_chunked(spec, ctx_lens=ctx, q_lens=ql)
    oa, la = run_chunked(a, True, spec.scale)
    b = inputs.ChunkedInputs(q=a.q, cu_q=a.cu_q, cache=inputs.permute_pool(a.cache, seed=7))
    ob, lb = run_chunked(b, True, spec.scale)
    assert torch.equal(oa, ob) and torch.equal(la, lb)
    # slots past each sequence end in its last block hold NaN: nothing changes
    for i, L in enumerate(ctx):
        last = int(b.cache.block_table[i, (L - 1) // 16])
        b.cache.k_cache[last, L % 16 or 16:] = float("nan")
        b.cache.v_cache[last, L % 16 or 16:] = float("nan")
    oc, lc = run_chunked(b, True, spec.scale)
    assert torch.equal(oa, oc) and torch.equal(la, lc)


def test_chunked_workload():
    spec = inputs.CHUNKED_WORKLOADS["chunked_prefill_paged"]
    inp = inputs.make_chunked(spec)
    o, lse = run_chunked(inp, True, spec.scale)
    O, L = oracle_chunked(inp, True, spec.scale)
    check_close(f64(o), O, lse.numpy(), L, what="chunked_prefill_paged")
