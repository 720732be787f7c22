"""The torch custom-op wrappers: fake (meta) shapes on CPU, and on the GPU
results that match the fp64 oracle and are identical to the direct
binding's, inside torch.compile without a graph break (aot_eager backend:
no code generation around the ops)."""

import pytest
import torch

from flashattention_attention_attn_b200 import inputs
import flashattention_attention_attn_b200.torch_ops  # noqa: F401  (registers torch.ops.fa_b200)
from tests._parity import (check_close, f64, oracle_chunked, oracle_decode, oracle_decode_fp8, oracle_prefill,
                           oracle_varlen)


def test_fake_shapes_without_running_anything():
    from torch._subclasses.fake_tensor import FakeTensorMode
    with FakeTensorMode():
        q = torch.empty(2, 300, 32, 128, dtype=torch.bfloat16)
        k = torch.empty(2, 400, 8, 128, dtype=torch.bfloat16)
        o, lse = torch.ops.fa_b200.attn_fwd(q, k, k, True, 0.088)
        assert o.shape == q.shape and o.dtype == torch.bfloat16
        assert lse.shape == (2, 32, 300) and lse.dtype == torch.float32
        qd = torch.empty(5, 32, 128, dtype=torch.bfloat16)
        kc = torch.empty(40, 16, 8, 128, dtype=torch.bfloat16)
        bt = torch.empty(5, 8, dtype=torch.int32)
        od = torch.ops.fa_b200.paged_attn_decode(qd, kc, kc, bt, torch.empty(5, dtype=torch.int32), 0)
        assert od.shape == qd.shape
        # packed and paged prefill: o like q, lse [Hq, total_q]
        qp = torch.empty(700, 32, 128, dtype=torch.bfloat16)
        kp = torch.empty(900, 8, 128, dtype=torch.bfloat16)
        cu = torch.empty(4, dtype=torch.int32)
        o, lse = torch.ops.fa_b200.attn_fwd_varlen(qp, kp, kp, cu, cu, 300, True, 0.088)
        assert o.shape == qp.shape and lse.shape == (32, 700) and lse.dtype == torch.float32
        o, lse = torch.ops.fa_b200.paged_attn_prefill(qp, kc, kc, torch.empty(3, 8, dtype=torch.int32),
                                                      torch.empty(3, dtype=torch.int32), cu, 300, True, 0.088)
        assert o.shape == qp.shape and lse.shape == (32, 700)
        k8 = torch.empty(40, 16, 8, 128, dtype=torch.uint8)
        od = torch.ops.fa_b200.paged_attn_decode_fp8(qd, k8, k8, bt, torch.empty(5, dtype=torch.int32), 0, 0.5, 2.0)
        assert od.shape == qd.shape and od.dtype == torch.bfloat16
        # context-parallel halves: fp32 partials, then the merge of R of them
        op, lp = torch.ops.fa_b200.paged_attn_decode_partial(qd, kc, kc, bt, torch.empty(5, dtype=torch.int32), 0)
        assert op.shape == qd.shape and op.dtype == torch.float32 and lp.shape == (5, 32) and lp.dtype == torch.float32
        om = torch.ops.fa_b200.attn_lse_merge(torch.empty(3, 5, 32, 128), torch.empty(3, 5, 32))
        assert om.shape == (5, 32, 128) and om.dtype == torch.bfloat16


@pytest.mark.gpu
def test_ops_match_the_oracle_and_compile_without_graph_break():
    import flashattention_attention_attn_b200 as fa
    ps = inputs.PrefillSpec(B=1, Hq=8, Hkv=2, T=200, S=200, d=128, causal=True, seed=60)
    q, k, v = [t.cuda() for t in inputs.make_prefill(ps)]
    ds = inputs.DecodeSpec(B=3, Hq=32, Hkv=8, d=128, block_size=16, max_blocks=16, ctx_lo=10, ctx_hi=250, seed=61)
    d = inputs.make_paged(ds)
    dq, kc, vc, bt, sl = d.q.cuda(), d.k_cache.cuda(), d.v_cache.cuda(), d.block_table.cuda(), d.seq_lens.cuda()

    o_ref = torch.empty_like(q)
    lse_ref = torch.empty(1, 8, 200, device="cuda")
    fa.attn_fwd(q, k, v, o_ref, lse_ref, 1, 8, 2, 200, 200, 128, True, ps.scale)
    od_ref = torch.empty_like(dq)
    fa.paged_attn_decode(dq, kc, vc, bt, sl, 3, 32, 8, 128, 16, 16, 0, od_ref)

    def f(q, k, v, dq, kc, vc, bt, sl):
        o, lse = torch.ops.fa_b200.attn_fwd(q, k, v, True, ps.scale)
        od = torch.ops.fa_b200.paged_attn_decode(dq, kc, vc, bt, sl, 0)
        return o, lse, od

    g = torch.compile(f, backend="aot_eager", fullgraph=True)
    o, lse, od = g(q, k, v, dq, kc, vc, bt, sl)
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref) and torch.equal(od, od_ref)
    O, L = oracle_prefill(q.cpu(), k.cpu(), v.cpu(), True, ps.scale)
    check_close(f64(o), O, f64(lse), L, what="torch op attn_fwd")
    Od, _ = oracle_decode(d)
    check_close(f64(od), Od, what="torch op paged_attn_decode")


@pytest.mark.gpu
def test_packed_chunked_and_fp8_ops_match_the_oracle_and_the_binding():
    from tests._parity import run_chunked, run_decode_fp8, run_varlen
    vs = inputs.VarlenSpec(B=3, Hq=8, Hkv=2, d=128, len_lo=1, len_hi=1, causal=True, seed=62)
    vin = inputs.make_varlen(vs, q_lens=[5, 130, 300])
    o_ref, lse_ref = run_varlen(vin, True, vs.scale)
    o, lse = torch.ops.fa_b200.attn_fwd_varlen(vin.q.cuda(), vin.k.cuda(), vin.v.cuda(), vin.cu_q.cuda(),
                                               vin.cu_k.cuda(), vin.max_q, True, vs.scale)
    assert torch.equal(o.cpu(), o_ref) and torch.equal(lse.cpu(), lse_ref)
    O, L = oracle_varlen(vin, True, vs.scale)
    check_close(f64(o), O, f64(lse), L, what="torch op attn_fwd_varlen")

    cs = inputs.ChunkedSpec(B=2, Hq=8, Hkv=2, d=128, block_size=16, max_blocks=32, ctx_lo=1, ctx_hi=1, q_lo=1, q_hi=1,
                            seed=63)
    cin = inputs.make_chunked(cs, ctx_lens=[300, 77], q_lens=[100, 77])
    o_ref, lse_ref = run_chunked(cin, True, cs.scale)
    c = cin.cache
    o, lse = torch.ops.fa_b200.paged_attn_prefill(cin.q.cuda(), c.k_cache.cuda(), c.v_cache.cuda(),
                                                  c.block_table.cuda(), c.seq_lens.cuda(), cin.cu_q.cuda(),
                                                  cin.max_q, True, cs.scale)
    assert torch.equal(o.cpu(), o_ref) and torch.equal(lse.cpu(), lse_ref)
    O, L = oracle_chunked(cin, True, cs.scale)
    check_close(f64(o), O, f64(lse), L, what="torch op paged_attn_prefill")

    ds = inputs.DecodeSpec(B=3, Hq=32, Hkv=8, d=128, block_size=16, max_blocks=16, ctx_lo=10, ctx_hi=250, seed=64)
    din = inputs.make_paged_fp8(ds)
    od_ref = run_decode_fp8(din, num_splits=0)
    od = torch.ops.fa_b200.paged_attn_decode_fp8(din.q.cuda(), din.k_cache.cuda(), din.v_cache.cuda(),
                                                 din.block_table.cuda(), din.seq_lens.cuda(), 0, din.k_scale,
                                                 din.v_scale)
    assert torch.equal(od.cpu(), od_ref)
    check_close(f64(od), oracle_decode_fp8(din)[0], what="torch op paged_attn_decode_fp8")


@pytest.mark.gpu
def test_context_parallel_ops_match_the_binding_and_the_oracle():
    """Two shares of every sequence decoded with the partial op and merged
    with the merge op inside torch.compile: identical to the direct binding
    calls, and within the tolerance of the oracle's full decode."""
    import flashattention_attention_attn_b200 as fa
    from flashattention_attention_attn_b200 import dist_util
    ds = inputs.DecodeSpec(B=4, Hq=32, Hkv=8, d=128, block_size=16, max_blocks=40, ctx_lo=0, ctx_hi=640, seed=65)
    d = inputs.make_paged(ds)
    dq, kc, vc = d.q.cuda(), d.k_cache.cuda(), d.v_cache.cuda()
    shares = [dist_util.context_shard(d.block_table.cuda(), d.seq_lens.cuda(), 2, r)[:2] for r in range(2)]

    def f(dq, kc, vc, t0, l0, t1, l1):
        o0, s0 = torch.ops.fa_b200.paged_attn_decode_partial(dq, kc, vc, t0, l0, 0)
        o1, s1 = torch.ops.fa_b200.paged_attn_decode_partial(dq, kc, vc, t1, l1, 0)
        return torch.ops.fa_b200.attn_lse_merge(torch.stack([o0, o1]), torch.stack([s0, s1]))

    g = torch.compile(f, backend="aot_eager", fullgraph=True)
    o = g(dq, kc, vc, *shares[0], *shares[1])
    po = torch.empty(2, 4, 32, 128, device="cuda")
    pl = torch.empty(2, 4, 32, device="cuda")
    for r, (t, n) in enumerate(shares):
        fa.paged_attn_decode_partial(dq, kc, vc, t, n, 4, 32, 8, 128, 16, t.shape[1], kc.shape[0], 0, po[r], pl[r])
    o_ref = torch.empty(4, 32, 128, device="cuda", dtype=torch.bfloat16)
    fa.attn_lse_merge(po, pl, 2, 4, 32, 128, o_ref)
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref)
    check_close(f64(o), oracle_decode(d)[0], what="torch ops context-parallel decode")
