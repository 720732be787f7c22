"""paged_attn_decode_noalloc: the decode entry point for callers that cannot
allocate device memory during a call (a server that has already given all
free memory to its KV-cache pool, code that must not re-enter an allocator).
Its split partials live in a fixed scratch array compiled into the library.
Checked through the C ABI against the regular entry point, on two calls in a
row with different inputs, so that contents left in the shared scratch by
one call cannot leak into the next."""

import pytest
import torch

import flashattention_attention_attn_b200 as fa
from flashattention_attention_attn_b200 import inputs
from tests._parity import check_close, f64

pytestmark = pytest.mark.gpu


def _run(fn, inp, num_splits):
    B, Hq, d = inp.q.shape
    Hkv = inp.k_cache.shape[2]
    o = torch.full((B, Hq, d), float("nan"), device="cuda", dtype=torch.bfloat16)
    fn(inp.q.cuda(), inp.k_cache.cuda(), inp.v_cache.cuda(), inp.block_table.cuda(), inp.seq_lens.cuda(),
       B, Hq, Hkv, d, inp.block_size, inp.block_table.shape[1], num_splits, o)
    torch.cuda.synchronize()
    assert fa.attn_read_device_status(clear=True) == 0
    return o.cpu()


@pytest.mark.parametrize("num_splits", [0, 7])
def test_noalloc_matches_regular_entry_point_on_two_calls(num_splits):
    spec = inputs.WORKLOADS["paged_decode_b64"]
    first = inputs.make_paged(spec, seed=spec.seed + 1)
    second = inputs.make_paged(spec, seed=spec.seed + 2)
    want = [_run(fa.paged_attn_decode, x, num_splits) for x in (first, second)]
    got = [_run(fa.paged_attn_decode_noalloc, x, num_splits) for x in (first, second)]
    for g, w in zip(got, want):
        check_close(f64(g), f64(w), what=f"noalloc vs regular, num_splits={num_splits}")


def test_noalloc_rejects_partials_beyond_the_scratch_size():
    spec = inputs.DecodeSpec(B=64, Hq=32, Hkv=8, d=128, block_size=16, max_blocks=256, ctx_lo=16, ctx_hi=64,
                             seed=3)
    inp = inputs.make_paged(spec)
    with pytest.raises(fa.AttnError) as err:  # 256 splits * 64 * 32 rows * 129 floats > 16 MiB
        _run(fa.paged_attn_decode_noalloc, inp, 256)
    assert err.value.status == -2
