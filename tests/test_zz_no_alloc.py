"""paged_attn_decode_noalloc: the decode entry point for callers that cannot
allocate device memory during a call (a server that has already given all
free memory to its KV-cache pool, code that must not re-enter an allocator).
Its split partials live in a fixed scratch array compiled into the library.

Checked through the C ABI: on two calls in a row with different inputs (so
that contents left in the shared scratch by one call cannot leak into the
next), its output is bit-identical to paged_attn_decode's (the same kernels
on the same inputs) and matches the fp64 oracle; and in a fresh process,
repeated calls change the device's free memory by nothing.  This file is
collected last."""

import os
import subprocess
import sys
import textwrap

import pytest
import torch

import flashattention_attention_attn_b200 as fa
from flashattention_attention_attn_b200 import inputs
from tests._parity import check_close, f64, oracle_decode

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(fn, inp, num_splits):
    B, Hq, d = inp.q.shape
    Hkv = inp.k_cache.shape[2]
    o = torch.full((B, Hq, d), float("nan"), device="cuda", dtype=torch.bfloat16)
    fn(inp.q.cuda(), inp.k_cache.cuda(), inp.v_cache.cuda(), inp.block_table.cuda(), inp.seq_lens.cuda(),
       B, Hq, Hkv, d, inp.block_size, inp.block_table.shape[1], num_splits, o)
    torch.cuda.synchronize()
    assert fa.attn_read_device_status(clear=True) == 0
    return o.cpu()


CASES = {
    # name: (workload, num_splits); each case runs with two seeds in a row
    "b64_7_splits": (inputs.WORKLOADS["paged_decode_b64"], 7),
    "b64_one_split": (inputs.WORKLOADS["paged_decode_b64"], 1),
    "d64_auto": (inputs.DecodeSpec(B=9, Hq=16, Hkv=4, d=64, block_size=16, max_blocks=40, ctx_lo=1, ctx_hi=640,
                                   seed=90), 0),
    "long_131k_auto": (inputs.WORKLOADS["long_decode_131k"], 0),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_noalloc_equals_regular_entry_point_on_two_calls(case):
    spec, num_splits = CASES[case]
    for seed in (spec.seed + 1, spec.seed + 2):
        inp = inputs.make_paged(spec, seed=seed)
        want = _run(fa.paged_attn_decode, inp, num_splits)
        got = _run(fa.paged_attn_decode_noalloc, inp, num_splits)
        assert torch.equal(got, want), f"{case}: no-alloc output differs from paged_attn_decode"
        O, _ = oracle_decode(inp)
        check_close(f64(got), O, what=f"noalloc {case} seed {seed}")


def test_noalloc_rejects_partials_beyond_the_scratch_size():
    spec = inputs.DecodeSpec(B=64, Hq=32, Hkv=8, d=128, block_size=16, max_blocks=256, ctx_lo=16, ctx_hi=64,
                             seed=3)
    inp = inputs.make_paged(spec)
    with pytest.raises(fa.AttnError) as err:  # 256 splits * 64 * 32 rows * 129 floats > 16 MiB
        _run(fa.paged_attn_decode_noalloc, inp, 256)
    assert err.value.status == -2


def test_noalloc_calls_allocate_no_device_memory():
    # a fresh process that calls only the no-alloc entry point: after the
    # first call (which loads the kernels and the scratch array), further
    # calls leave the device's free memory unchanged
    code = textwrap.dedent(f"""
        import sys
        sys.path.insert(0, {ROOT!r})
        import torch
        import flashattention_attention_attn_b200 as fa
        from flashattention_attention_attn_b200 import inputs
        spec = inputs.WORKLOADS["paged_decode_b64"]
        inp = inputs.make_paged(spec)
        args = [t.cuda() for t in (inp.q, inp.k_cache, inp.v_cache, inp.block_table, inp.seq_lens)]
        o = torch.empty(spec.B, spec.Hq, spec.d, device="cuda", dtype=torch.bfloat16)
        def call():
            fa.paged_attn_decode_noalloc(*args, spec.B, spec.Hq, spec.Hkv, spec.d, 16, inp.block_table.shape[1], 7, o)
            torch.cuda.synchronize()
        call()
        free0 = torch.cuda.mem_get_info()[0]
        for _ in range(5):
            call()
        free1 = torch.cuda.mem_get_info()[0]
        assert fa.attn_read_device_status(clear=True) == 0
        print("free bytes", free0, free1)
        sys.exit(0 if free1 == free0 else 1)
    """)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
