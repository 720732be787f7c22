"""Block-table safety of the paged entry points, on the GPU, against the fp64
oracle.  Every position is translated through the block table ("De
aandachtskernel moet dan elke positie via deze tabel vertalen", page "Snelle
attention-kernels en operatorfusie versnellen AI-modellen", section
"FlashAttention-type aandacht en gepagineerde aandacht"); these tests feed
tables that name blocks outside the declared pool and lengths beyond the
table row, and check that such entries are masked (the oracle's reading),
that the device status word says so, and that valid inputs raise no bit.

Every input is built so that every access stays inside allocated memory even
if the checks were missing: the "outside" ids lie in the allocated pool
beyond the size the call declares (or are negative, which a TMA load turns
into zero fill), and tables are padded with valid ids past their last row.
"""

import pytest
import torch

import flashattention_attention_attn_b200 as fa
from flashattention_attention_attn_b200 import inputs
from oracle import fp64_attention as orc
from tests._parity import check_close, f64

pytestmark = pytest.mark.gpu

BAD_BLOCK = 0x2
BAD_SEQLEN = 0x4


def _status():
    torch.cuda.synchronize()
    return fa.attn_read_device_status(clear=True)


def _decode_checked(inp, table, lens, num_blocks, num_splits, max_blocks=None, fp8=False):
    B, Hq, d = inp.q.shape
    Hkv = inp.k_cache.shape[2]
    max_blocks = table.shape[1] if max_blocks is None else max_blocks
    o = torch.full((B, Hq, d), float("nan"), device="cuda", dtype=torch.bfloat16)
    args = (inp.q.cuda(), inp.k_cache.cuda(), inp.v_cache.cuda(), table.cuda(), lens.cuda(), B, Hq, Hkv, d, 16,
            max_blocks)
    if fp8:
        if num_blocks is None:
            fa.paged_attn_decode_fp8(*args, num_splits, inp.k_scale, inp.v_scale, o)
        else:
            fa.paged_attn_decode_fp8_checked(*args, num_blocks, num_splits, inp.k_scale, inp.v_scale, o)
    elif num_blocks is None:
        fa.paged_attn_decode(*args, num_splits, o)
    else:
        fa.paged_attn_decode_checked(*args, num_blocks, num_splits, o)
    return o.cpu(), _status()


def _half_pool_case(seed, B=12, d=128, fp8=False):
    """A decode batch whose pool is twice the size the call will declare:
    about half of every table row names blocks past the declared size, and
    one sequence has every block there."""
    spec = inputs.DecodeSpec(B=B, Hq=32, Hkv=8, d=d, block_size=16, max_blocks=40, ctx_lo=1, ctx_hi=640, seed=seed)
    inp = inputs.make_paged_fp8(spec) if fp8 else inputs.make_paged(spec)
    pool = inp.k_cache.shape[0]
    declared = pool // 2
    table = inp.block_table.clone()
    n3 = (int(inp.seq_lens[3]) + 15) // 16
    big = torch.arange(declared, pool, dtype=torch.int32)
    table[3, :n3] = big[:n3]  # sequence 3: all of its blocks outside the declared pool
    assert ((table >= declared) & (table < pool)).any() and n3 > 0
    return inp, table, declared


@pytest.mark.parametrize("num_splits", [1, 3, 0])
@pytest.mark.parametrize("d", [128, 64])
def test_decode_masks_blocks_outside_the_declared_pool(num_splits, d):
    inp, table, declared = _half_pool_case(70 + d, d=d)
    o, st = _decode_checked(inp, table, inp.seq_lens, declared, num_splits)
    assert st & BAD_BLOCK and not st & BAD_SEQLEN
    O, _ = orc.paged_decode(f64(inp.q), f64(inp.k_cache), f64(inp.v_cache), table.numpy(), inp.seq_lens.numpy(), 16,
                            inp.q.shape[-1] ** -0.5, num_blocks=declared)
    check_close(f64(o), O, what=f"checked decode d={d} splits={num_splits}")
    assert torch.all(o[3] == 0)  # no key inside the pool: O = 0


def test_decode_with_the_true_pool_size_equals_the_unchecked_call():
    spec = inputs.WORKLOADS["paged_decode_b64"]
    inp = inputs.make_paged(spec)
    want, st0 = _decode_checked(inp, inp.block_table, inp.seq_lens, None, 0)
    got, st1 = _decode_checked(inp, inp.block_table, inp.seq_lens, inp.k_cache.shape[0], 0)
    assert st0 == 0 and st1 == 0
    assert torch.equal(got, want)


def test_unchecked_decode_masks_negative_ids():
    # without a pool size, an id below 0 is still never loaded
    spec = inputs.DecodeSpec(B=6, Hq=32, Hkv=8, d=128, block_size=16, max_blocks=20, ctx_lo=40, ctx_hi=320, seed=75)
    inp = inputs.make_paged(spec)
    table = inp.block_table.clone()
    table[0, 0] = -1
    table[2, 1] = -7
    table[5, :2] = -3
    o, st = _decode_checked(inp, table, inp.seq_lens, None, 2)
    assert st & BAD_BLOCK
    O, _ = orc.paged_decode(f64(inp.q), f64(inp.k_cache), f64(inp.v_cache), table.numpy(), inp.seq_lens.numpy(), 16,
                            128 ** -0.5, num_blocks=inp.k_cache.shape[0])
    check_close(f64(o), O, what="unchecked decode, negative ids")


@pytest.mark.parametrize("num_splits", [1, 7])
def test_decode_clamps_lengths_beyond_the_table_row(num_splits):
    # the table is [B, max_blocks] of valid ids followed by padding of valid
    # ids, so that even an unclamped read would stay inside it
    B, max_blocks = 8, 24
    spec = inputs.DecodeSpec(B=B, Hq=32, Hkv=8, d=128, block_size=16, max_blocks=max_blocks, ctx_lo=1, ctx_hi=384,
                             seed=76)
    inp = inputs.make_paged(spec)
    pool = inp.k_cache.shape[0]
    g = torch.Generator().manual_seed(77)
    flat = torch.randint(0, pool, (B * max_blocks + 70000,), generator=g, dtype=torch.int32)
    table = flat[:B * max_blocks].view(B, max_blocks)
    lens = inp.seq_lens.clone()
    lens[1] = max_blocks * 16 + 5
    lens[4] = 10 ** 6
    lens[6] = -30
    o = torch.full((B, 32, 128), float("nan"), device="cuda", dtype=torch.bfloat16)
    fa.paged_attn_decode(inp.q.cuda(), inp.k_cache.cuda(), inp.v_cache.cuda(), flat.cuda(), lens.cuda(), B, 32, 8,
                         128, 16, max_blocks, num_splits, o)
    st = _status()
    assert st & BAD_SEQLEN and not st & BAD_BLOCK
    O, _ = orc.paged_decode(f64(inp.q), f64(inp.k_cache), f64(inp.v_cache), table.numpy(), lens.numpy(), 16,
                            128 ** -0.5)
    check_close(f64(o.cpu()), O, what=f"decode, clamped lengths, splits={num_splits}")
    assert torch.all(o[6].cpu() == 0)


def test_fp8_decode_masks_blocks_outside_the_declared_pool():
    inp, table, declared = _half_pool_case(78, fp8=True)
    o, st = _decode_checked(inp, table, inp.seq_lens, declared, 0, fp8=True)
    assert st & BAD_BLOCK
    K = inp.k_scale * orc.decode_e4m3(inp.k_cache.numpy())
    V = inp.v_scale * orc.decode_e4m3(inp.v_cache.numpy())
    O, _ = orc.paged_decode(f64(inp.q), K, V, table.numpy(), inp.seq_lens.numpy(), 16, 128 ** -0.5,
                            num_blocks=declared)
    check_close(f64(o), O, what="checked FP8 decode")
    assert torch.all(o[3] == 0)


def _chunked_checked(cin, table, lens, num_blocks, causal=True, max_blocks=None):
    total_q, Hq, d = cin.q.shape
    c = cin.cache
    Hkv = c.k_cache.shape[2]
    B = cin.cu_q.numel() - 1
    o = torch.full((total_q, Hq, d), float("nan"), device="cuda", dtype=torch.bfloat16)
    lse = torch.full((Hq, total_q), float("nan"), device="cuda", dtype=torch.float32)
    max_blocks = table.shape[1] if max_blocks is None else max_blocks
    args = (cin.q.cuda(), c.k_cache.cuda(), c.v_cache.cuda(), table.cuda(), lens.cuda(), cin.cu_q.cuda(), B, Hq, Hkv,
            d, 16, max_blocks)
    scale = d ** -0.5
    if num_blocks is None:
        fa.paged_attn_prefill(*args, cin.max_q, total_q, causal, scale, o, lse)
    else:
        fa.paged_attn_prefill_checked(*args, num_blocks, cin.max_q, total_q, causal, scale, o, lse)
    return o.cpu(), lse.cpu(), _status()


@pytest.mark.parametrize("causal", [True, False])
def test_chunked_prefill_masks_blocks_outside_the_declared_pool(causal):
    ctx, ql = [700, 300, 129, 520, 64], [300, 300, 40, 200, 64]
    spec = inputs.ChunkedSpec(B=5, Hq=8, Hkv=2, d=128, block_size=16, max_blocks=48, ctx_lo=1, ctx_hi=1, q_lo=1,
                              q_hi=1, seed=79)
    cin = inputs.make_chunked(spec, ctx_lens=ctx, q_lens=ql)
    c = cin.cache
    pool = c.k_cache.shape[0]
    declared = pool // 2
    table = c.block_table.clone()
    table[4, :4] = torch.arange(declared, declared + 4, dtype=torch.int32)  # sequence 4 sees no key at all
    table[1, 3] = -2
    o, lse, st = _chunked_checked(cin, table, c.seq_lens, declared, causal)
    assert st & BAD_BLOCK and not st & BAD_SEQLEN
    O, L = orc.paged_prefill(f64(cin.q), f64(c.k_cache), f64(c.v_cache), table.numpy(), c.seq_lens.numpy(),
                             cin.cu_q.numpy(), 16, 128 ** -0.5, causal, num_blocks=declared)
    check_close(f64(o), O, lse.numpy(), L, what=f"checked chunked prefill causal={causal}")
    r0, r1 = int(cin.cu_q[4]), int(cin.cu_q[5])
    assert torch.all(o[r0:r1] == 0) and torch.all(torch.isneginf(lse[:, r0:r1]))


def test_chunked_prefill_clamps_lengths_and_masks_negative_ids_unchecked():
    B, max_blocks = 4, 20
    ctx, ql = [200, 300, 100, 90], [100, 64, 100, 90]
    spec = inputs.ChunkedSpec(B=B, Hq=8, Hkv=2, d=64, block_size=16, max_blocks=max_blocks, ctx_lo=1, ctx_hi=1,
                              q_lo=1, q_hi=1, seed=80)
    cin = inputs.make_chunked(spec, ctx_lens=ctx, q_lens=ql)
    c = cin.cache
    pool = c.k_cache.shape[0]
    g = torch.Generator().manual_seed(81)
    flat = torch.randint(0, pool, (B * max_blocks + 70000,), generator=g, dtype=torch.int32)
    table = flat[:B * max_blocks].view(B, max_blocks)
    table[0, 2] = -1
    lens = c.seq_lens.clone()
    lens[1] = 10 ** 6   # clamped to 320 positions: its 64 rows sit at 256..319
    lens[3] = -5        # clamped to 0: every row sees nothing
    o, lse, st = _chunked_checked(cin, flat, lens, None, max_blocks=max_blocks)
    assert st & BAD_BLOCK and st & BAD_SEQLEN
    O, L = orc.paged_prefill(f64(cin.q), f64(c.k_cache), f64(c.v_cache), table.numpy(), lens.numpy(),
                             cin.cu_q.numpy(), 16, 64 ** -0.5, True, num_blocks=pool)
    check_close(f64(o), O, lse.numpy(), L, what="chunked prefill, clamped lengths and a negative id")


def test_valid_inputs_raise_no_status_bit():
    spec = inputs.ChunkedSpec(B=3, Hq=8, Hkv=2, d=128, block_size=16, max_blocks=40, ctx_lo=1, ctx_hi=1, q_lo=1,
                              q_hi=1, seed=82)
    cin = inputs.make_chunked(spec, ctx_lens=[640, 17, 300], q_lens=[200, 17, 1])
    c = cin.cache
    o0, l0, st0 = _chunked_checked(cin, c.block_table, c.seq_lens, None)
    o1, l1, st1 = _chunked_checked(cin, c.block_table, c.seq_lens, c.k_cache.shape[0])
    assert st0 == 0 and st1 == 0
    assert torch.equal(o0, o1) and torch.equal(l0, l1)
