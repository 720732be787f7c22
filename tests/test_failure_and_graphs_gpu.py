"""Failure detection without a GPU fault, and CUDA-graph capture.

* A bounded wait that runs out (a barrier nothing arrives on) records
  ATTN_DEVSTATUS_TIMEOUT and returns; the context stays usable and the next
  attention call is correct.
* attn_fwd and paged_attn_decode are stream-ordered and allocation-safe
  under capture: captured once into a CUDA graph and replayed, they give the
  same bits as direct calls.
* Issued on two streams at once (the decode forked off and joined back, as
  the benchmark step does), they give the same bits as on one stream.
"""

import time

import pytest
import torch

import flashattention_attention_attn_b200 as fa
from flashattention_attention_attn_b200 import inputs
from tests._parity import check_close, f64, oracle_decode, run_decode

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_context_survives():
    assert fa.attn_read_device_status(clear=True) == 0
    t0 = time.perf_counter()
    fa.attn_selftest_bounded_wait()
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    assert fa.attn_read_device_status(clear=True) & 1  # ATTN_DEVSTATUS_TIMEOUT
    assert fa.attn_read_device_status(clear=True) == 0  # cleared
    assert waited < 30.0
    # the context is still usable: a regular call works and is correct
    spec = inputs.DecodeSpec(B=2, Hq=32, Hkv=8, d=128, block_size=16, max_blocks=8, ctx_lo=20, ctx_hi=120, seed=17)
    inp = inputs.make_paged(spec)
    O, _ = oracle_decode(inp)
    check_close(f64(run_decode(inp)), O, what="after timeout")


def test_graph_capture_replays_bit_identically():
    ps = inputs.PrefillSpec(B=1, Hq=8, Hkv=2, T=300, S=300, d=128, causal=True, seed=18)
    q, k, v = [t.cuda() for t in inputs.make_prefill(ps)]
    ds = inputs.DecodeSpec(B=4, Hq=32, Hkv=8, d=128, block_size=16, max_blocks=32, ctx_lo=50, ctx_hi=512, seed=19)
    dinp = inputs.make_paged(ds)
    dq, kc, vc = dinp.q.cuda(), dinp.k_cache.cuda(), dinp.v_cache.cuda()
    bt, sl = dinp.block_table.cuda(), dinp.seq_lens.cuda()
    o = torch.empty_like(q)
    lse = torch.empty(1, 8, 300, device="cuda")
    od = torch.empty(4, 32, 128, device="cuda", dtype=torch.bfloat16)

    def step(stream):
        fa.attn_fwd(q, k, v, o, lse, 1, 8, 2, 300, 300, 128, True, ps.scale, stream)
        fa.paged_attn_decode(dq, kc, vc, bt, sl, 4, 32, 8, 128, 16, 32, 5, od, stream)

    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        step(s)  # first call on the device outside capture (one-time set-up)
    torch.cuda.synchronize()
    ref_o, ref_lse, ref_od = o.clone(), lse.clone(), od.clone()
    o.zero_(); lse.zero_(); od.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step(s)
    for _ in range(3):
        o.zero_(); od.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(o, ref_o) and torch.equal(lse, ref_lse) and torch.equal(od, ref_od)
    assert fa.attn_read_device_status(clear=True) == 0
    del g


def test_prefill_and_decode_on_two_streams_match_one_stream():
    # The benchmark step runs the two ops concurrently: the decode forks onto
    # a second stream and joins back.  The results are those of one stream.
    ps = inputs.PrefillSpec(B=2, Hq=32, Hkv=8, T=512, S=512, d=128, causal=True, seed=20)
    q, k, v = [t.cuda() for t in inputs.make_prefill(ps)]
    ds = inputs.DecodeSpec(B=16, Hq=32, Hkv=8, d=128, block_size=16, max_blocks=64, ctx_lo=100, ctx_hi=1024, seed=21)
    dinp = inputs.make_paged(ds)
    dq, kc, vc = dinp.q.cuda(), dinp.k_cache.cuda(), dinp.v_cache.cuda()
    bt, sl = dinp.block_table.cuda(), dinp.seq_lens.cuda()
    o = torch.empty_like(q)
    lse = torch.empty(2, 32, 512, device="cuda")
    od = torch.empty(16, 32, 128, device="cuda", dtype=torch.bfloat16)
    main = torch.cuda.current_stream()
    side = torch.cuda.Stream()
    fork, join = torch.cuda.Event(), torch.cuda.Event()

    def prefill(st):
        fa.attn_fwd(q, k, v, o, lse, 2, 32, 8, 512, 512, 128, True, ps.scale, st)

    def decode(st):
        fa.paged_attn_decode(dq, kc, vc, bt, sl, 16, 32, 8, 128, 16, 64, 0, od, st)

    prefill(main)
    decode(main)
    torch.cuda.synchronize()
    ref_o, ref_lse, ref_od = o.clone(), lse.clone(), od.clone()
    o.zero_(); lse.zero_(); od.zero_()
    for _ in range(20):
        fork.record(main)
        side.wait_event(fork)
        prefill(main)
        decode(side)
        join.record(side)
        main.wait_event(join)
    torch.cuda.synchronize()
    assert torch.equal(o, ref_o) and torch.equal(lse, ref_lse) and torch.equal(od, ref_od)
    assert fa.attn_read_device_status(clear=True) == 0
