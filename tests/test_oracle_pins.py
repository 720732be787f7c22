"""Pins for the fp64 oracle: each test checks it against something other
than itself (closed forms, brute force, invariants the pages fix, a library
routine), so that a dropped term, a wrong sign or index, or a transposed
operand in the oracle fails at least one of them."""

import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import fp64_attention as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_form_cases.json")


def _val(s):
    s = str(s).strip()
    if "ln(" in s:
        coef, _, rest = s.partition("ln(")
        c = float(Fraction(coef.rstrip("*"))) if coef.strip() else 1.0
        return c * math.log(float(Fraction(rest.rstrip(")"))))
    return float(Fraction(s))


def _arr(x):
    if isinstance(x, list):
        return np.array([_arr(e) for e in x], dtype=np.float64)
    return _val(x)


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


@pytest.mark.parametrize("case", _golden()["prefill"], ids=lambda c: c["name"])
def test_golden_prefill_closed_forms(case):
    q = _arr(case["q"])[None]
    k = _arr(case["k"])[None]
    v = _arr(case["v"])[None]
    O, LSE = orc.attention(q, k, v, _val(case["scale"]), case["causal"])
    np.testing.assert_allclose(O[0], _arr(case["O"]), rtol=0, atol=1e-12)
    np.testing.assert_allclose(LSE[0], _arr(case["LSE"]), rtol=0, atol=1e-12)


@pytest.mark.parametrize("case", _golden()["paged"], ids=lambda c: c["name"])
def test_golden_paged_closed_forms(case):
    O, LSE = orc.paged_decode(_arr(case["q"]), _arr(case["k_cache"]), _arr(case["v_cache"]),
                              np.array(case["block_table"]), np.array(case["seq_lens"]),
                              case["block_size"], _val(case["scale"]))
    np.testing.assert_allclose(O, _arr(case["O"]), rtol=0, atol=1e-12)
    np.testing.assert_allclose(LSE, _arr(case["LSE"]), rtol=0, atol=1e-12)


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _brute_force(q, k, v, scale, causal):
    """Independent naive evaluation with Python floats and math.exp."""
    B, T, Hq, d = q.shape
    S, Hkv = k.shape[1], k.shape[2]
    g = Hq // Hkv
    O = np.zeros((B, T, Hq, d))
    L = np.full((B, Hq, T), -math.inf)
    for b in range(B):
        for h in range(Hq):
            for i in range(T):
                js = [j for j in range(S) if (not causal) or j <= i + S - T]
                if not js:
                    continue
                sc = [scale * sum(float(q[b, i, h, c]) * float(k[b, j, h // g, c]) for c in range(d)) for j in js]
                mx = max(sc)
                w = [math.exp(x - mx) for x in sc]
                tot = sum(w)
                for c in range(d):
                    O[b, i, h, c] = sum(wj * float(v[b, j, h // g, c]) for wj, j in zip(w, js)) / tot
                L[b, h, i] = mx + math.log(tot)
    return O, L


@pytest.mark.parametrize("T,S,causal", [(1, 1, True), (5, 5, True), (3, 7, True), (6, 4, True),
                                        (4, 6, False), (8, 8, False)])
def test_brute_force_tiny(T, S, causal):
    q = _rand((2, T, 4, 8), 1)
    k = _rand((2, S, 2, 8), 2)
    v = _rand((2, S, 2, 8), 3)
    O, L = orc.attention(q, k, v, 0.3, causal)
    Ob, Lb = _brute_force(q, k, v, 0.3, causal)
    np.testing.assert_allclose(O, Ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L, Lb, rtol=0, atol=1e-12)


def test_softmax_rows_sum_to_one_and_respect_mask():
    s = _rand((64, 40), 4) * 10
    counts = np.random.default_rng(5).integers(1, 41, 64)
    P, m, l = orc.softmax_rows(s, counts)
    np.testing.assert_allclose(P.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    for r in range(64):
        assert np.all(P[r, counts[r]:] == 0)
        assert m[r] == s[r, :counts[r]].max()
    assert np.all(P >= 0)


def test_uniform_scores_give_running_mean():
    B, T, H, d = 1, 33, 3, 16
    q = np.zeros((B, T, H, d))
    k = _rand((B, T, H, d), 6)
    v = _rand((B, T, H, d), 7)
    O, L = orc.attention(q, k, v, 0.125, causal=True)
    cummean = np.cumsum(v, axis=1) / np.arange(1, T + 1)[None, :, None, None]
    np.testing.assert_allclose(O, cummean, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L, np.broadcast_to(np.log(np.arange(1, T + 1)), (B, H, T)), atol=1e-12)


def test_single_key_returns_its_value():
    q = _rand((2, 5, 4, 8), 8)
    k = _rand((2, 1, 2, 8), 9)
    v = _rand((2, 1, 2, 8), 10)
    O, L = orc.attention(q, k, v, 0.7, causal=False)
    for h in range(4):
        np.testing.assert_array_equal(O[:, :, h], np.broadcast_to(v[:, 0:1, h // 2], (2, 5, 8)))
        dot = np.einsum("btc,bc->bt", q[:, :, h], k[:, 0, h // 2])
        np.testing.assert_allclose(L[:, h], 0.7 * dot, rtol=0, atol=1e-12)


def test_causal_row0_is_first_value_row():
    q = _rand((2, 9, 8, 4), 11) * 5
    k = _rand((2, 9, 2, 4), 12) * 5
    v = _rand((2, 9, 2, 4), 13)
    O, _ = orc.attention(q, k, v, 1.0, causal=True)
    for h in range(8):
        np.testing.assert_array_equal(O[:, 0, h], v[:, 0, h // 4])


def test_shift_of_all_keys_leaves_output_and_shifts_lse():
    q = _rand((1, 12, 4, 8), 14)
    k = _rand((1, 12, 2, 8), 15)
    v = _rand((1, 12, 2, 8), 16)
    u = _rand((8,), 17)
    O1, L1 = orc.attention(q, k, v, 0.4, causal=True)
    O2, L2 = orc.attention(q, k + u, v, 0.4, causal=True)
    np.testing.assert_allclose(O2, O1, rtol=0, atol=1e-12)
    shift = 0.4 * np.einsum("bthc,c->bht", q, u)
    np.testing.assert_allclose(L2, L1 + shift, rtol=0, atol=1e-11)


def test_gqa_equals_mha_with_repeated_heads():
    q = _rand((2, 10, 8, 8), 18)
    k = _rand((2, 10, 2, 8), 19)
    v = _rand((2, 10, 2, 8), 20)
    O1, L1 = orc.attention(q, k, v, 0.35, causal=True)
    kr = np.repeat(k, 4, axis=2)  # head h -> kv head h // 4
    vr = np.repeat(v, 4, axis=2)
    O2, L2 = orc.attention(q, kr, vr, 0.35, causal=True)
    np.testing.assert_array_equal(O1, O2)
    np.testing.assert_array_equal(L1, L2)


@pytest.mark.parametrize("causal", [True, False])
def test_matches_torch_sdpa_fp64(causal):
    """PyTorch's scaled_dot_product_attention (named on the page as the
    library form of the same computation), fp64 on the CPU, K/V expanded."""
    B, T, Hq, Hkv, d = 2, 37, 8, 2, 16
    q = _rand((B, T, Hq, d), 21)
    k = _rand((B, T, Hkv, d), 22)
    v = _rand((B, T, Hkv, d), 23)
    O, _ = orc.attention(q, k, v, 0.25, causal)
    tq = torch.from_numpy(q).permute(0, 2, 1, 3)
    tk = torch.from_numpy(np.repeat(k, Hq // Hkv, axis=2)).permute(0, 2, 1, 3)
    tv = torch.from_numpy(np.repeat(v, Hq // Hkv, axis=2)).permute(0, 2, 1, 3)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=0.25)
    np.testing.assert_allclose(O, ref.permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-12)


def test_bottom_right_rows_equal_tail_of_square_prefill():
    """Reading: with T < S, causal rows are the last T rows of a T' = S prefill."""
    S, T = 20, 6
    qfull = _rand((1, S, 4, 8), 24)
    k = _rand((1, S, 2, 8), 25)
    v = _rand((1, S, 2, 8), 26)
    Of, Lf = orc.attention(qfull, k, v, 0.3, causal=True)
    Ot, Lt = orc.attention(qfull[:, S - T:], k, v, 0.3, causal=True)
    np.testing.assert_array_equal(Ot, Of[:, S - T:])
    np.testing.assert_array_equal(Lt, Lf[:, :, S - T:])


def test_empty_key_set_gives_zero_and_minus_inf():
    q = _rand((1, 4, 2, 8), 27)
    k = np.zeros((1, 0, 2, 8))
    O, L = orc.attention(q, k, k, 0.3, causal=True)
    assert np.all(O == 0) and np.all(np.isneginf(L))
    # T > S bottom-right: the first T - S rows see nothing
    k = _rand((1, 2, 2, 8), 28)
    O, L = orc.attention(q, k, k, 0.3, causal=True)
    assert np.all(O[:, :2] == 0) and np.all(np.isneginf(L[:, :, :2]))
    assert np.all(np.isfinite(L[:, :, 2:]))


def _paged_case(seed, B=5, Hq=8, Hkv=2, d=8, bs=4, max_blocks=9, extra=3):
    rng = np.random.default_rng(seed)
    lens = rng.integers(0, bs * max_blocks + 1, B)
    lens[0] = bs * max_blocks  # one full row
    lens[1] = 0                # one empty sequence
    nblk = [(int(L) + bs - 1) // bs for L in lens]
    pool = sum(nblk) + extra
    perm = rng.permutation(pool)
    table = -np.ones((B, max_blocks), dtype=np.int32)
    at = 0
    for b, n in enumerate(nblk):
        table[b, :n] = perm[at:at + n]
        at += n
    q = rng.standard_normal((B, Hq, d))
    kc = rng.standard_normal((pool, bs, Hkv, d))
    vc = rng.standard_normal((pool, bs, Hkv, d))
    return q, kc, vc, table, lens, bs


def test_paged_result_invariant_under_block_permutation():
    q, kc, vc, table, lens, bs = _paged_case(29)
    O1, L1 = orc.paged_decode(q, kc, vc, table, lens, bs, 0.3)
    perm = np.random.default_rng(30).permutation(kc.shape[0])
    kc2 = np.empty_like(kc)
    vc2 = np.empty_like(vc)
    kc2[perm] = kc
    vc2[perm] = vc
    t2 = np.where(table >= 0, perm[np.maximum(table, 0)], -1)
    O2, L2 = orc.paged_decode(q, kc2, vc2, t2, lens, bs, 0.3)
    np.testing.assert_array_equal(O1, O2)
    np.testing.assert_array_equal(L1, L2)


def test_paged_decode_equals_last_row_of_causal_prefill():
    q, kc, vc, table, lens, bs = _paged_case(31)
    O, L = orc.paged_decode(q, kc, vc, table, lens, bs, 0.3)
    for b in range(len(lens)):
        n = int(lens[b])
        if n == 0:
            assert np.all(O[b] == 0) and np.all(np.isneginf(L[b]))
            continue
        # contiguous cache written position by position (independent of the gather)
        K = np.stack([kc[table[b, p // bs], p % bs] for p in range(n)])[None]
        V = np.stack([vc[table[b, p // bs], p % bs] for p in range(n)])[None]
        Q = np.zeros((1, n, q.shape[1], q.shape[2]))
        Q[0, n - 1] = q[b]
        Op, Lp = orc.attention(Q, K, V, 0.3, causal=True)
        np.testing.assert_allclose(O[b], Op[0, n - 1], rtol=0, atol=1e-12)
        np.testing.assert_allclose(L[b], Lp[0, :, n - 1], rtol=0, atol=1e-12)


@pytest.mark.parametrize("splits", [1, 2, 3, 7, 9, 20])
def test_split_merge_equals_unsplit(splits):
    q, kc, vc, table, lens, bs = _paged_case(32)
    O1, L1 = orc.paged_decode(q, kc, vc, table, lens, bs, 0.3)
    O2, L2 = orc.split_paged_decode(q, kc, vc, table, lens, bs, 0.3, splits)
    np.testing.assert_allclose(O2, O1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L2, L1, rtol=0, atol=1e-12)


def test_merge_of_partials_closed_forms():
    # two key sets with sums 1 and 3 (lse 0 and ln 3): weights 1/4 and 3/4, total sum 4
    O, L = orc.merge_partials(np.array([[1.0, 0.0], [0.0, 1.0]]), np.array([0.0, math.log(3.0)]))
    np.testing.assert_allclose(O, [0.25, 0.75], rtol=0, atol=1e-15)
    assert abs(L - math.log(4.0)) < 1e-15
    # an empty set (-inf) takes no part, whatever its o holds
    O, L = orc.merge_partials(np.array([[np.nan, 7.0], [2.0, -1.0]]), np.array([-np.inf, 2.5]))
    np.testing.assert_array_equal(O, [2.0, -1.0])
    assert L == 2.5
    # no key anywhere: O = 0, LSE = -inf
    O, L = orc.merge_partials(np.ones((3, 4)), np.full(3, -np.inf))
    assert np.all(O == 0) and np.isneginf(L)


def _share_tables(table, lens, bs, cuts):
    """Shares of every sequence cut at the given block boundaries (fractions
    of its blocks), written position by position for the test."""
    B, max_blocks = table.shape
    shares = []
    for r in range(len(cuts) - 1):
        t = -np.ones((B, max_blocks), dtype=np.int32)
        n = np.zeros(B, dtype=np.int64)
        for b in range(B):
            nb = (int(lens[b]) + bs - 1) // bs
            lo, hi = int(cuts[r] * nb), int(cuts[r + 1] * nb)
            t[b, :hi - lo] = table[b, lo:hi]
            n[b] = max(0, min(int(lens[b]), hi * bs) - lo * bs)
        shares.append((t, n))
    return shares


@pytest.mark.parametrize("cuts", [(0, 1), (0, 0.5, 1), (0, 0.2, 0.3, 1), (0, 0, 0.7, 0.7, 1)])
def test_merge_of_context_shares_equals_unsplit_decode(cuts):
    q, kc, vc, table, lens, bs = _paged_case(34)
    O1, L1 = orc.paged_decode(q, kc, vc, table, lens, bs, 0.3)
    parts = [orc.paged_decode(q, kc, vc, t, n, bs, 0.3) for t, n in _share_tables(table, lens, bs, cuts)]
    assert sum(int(n.sum()) for _, n in _share_tables(table, lens, bs, cuts)) == int(lens.sum())
    O2, L2 = orc.merge_partials(np.stack([o for o, _ in parts]), np.stack([lse for _, lse in parts]))
    np.testing.assert_allclose(O2, O1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L2, L1, rtol=0, atol=1e-12)
    # the order of the parts does not matter
    O3, L3 = orc.merge_partials(np.stack([o for o, _ in parts][::-1]), np.stack([lse for _, lse in parts][::-1]))
    np.testing.assert_allclose(O3, O1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L3, L1, rtol=0, atol=1e-12)


def test_unused_table_entries_are_never_read():
    q, kc, vc, table, lens, bs = _paged_case(33)
    O1, L1 = orc.paged_decode(q, kc, vc, table, lens, bs, 0.3)
    t2 = table.copy()
    for b in range(len(lens)):
        t2[b, (int(lens[b]) + bs - 1) // bs:] = 10 ** 6  # would raise IndexError if read
    O2, L2 = orc.paged_decode(q, kc, vc, t2, lens, bs, 0.3)
    np.testing.assert_array_equal(O1, O2)
    np.testing.assert_array_equal(L1, L2)


def _varlen_case(seed, q_lens, k_lens, Hq=4, Hkv=2, d=8):
    rng = np.random.default_rng(seed)
    cu_q = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int64)
    cu_k = np.concatenate([[0], np.cumsum(k_lens)]).astype(np.int64)
    q = rng.standard_normal((cu_q[-1], Hq, d))
    k = rng.standard_normal((cu_k[-1], Hkv, d))
    v = rng.standard_normal((cu_k[-1], Hkv, d))
    return q, k, v, cu_q, cu_k


@pytest.mark.parametrize("causal", [True, False])
def test_varlen_brute_force_ragged(causal):
    q_lens, k_lens = [3, 0, 5, 1, 4], [3, 2, 7, 1, 2]
    q, k, v, cu_q, cu_k = _varlen_case(40, q_lens, k_lens)
    O, L = orc.attention_varlen(q, k, v, cu_q, cu_k, 0.3, causal)
    for b in range(len(q_lens)):
        q0, q1, k0, k1 = cu_q[b], cu_q[b + 1], cu_k[b], cu_k[b + 1]
        Ob, Lb = _brute_force(q[None, q0:q1], k[None, k0:k1], v[None, k0:k1], 0.3, causal)
        np.testing.assert_allclose(O[q0:q1], Ob[0], rtol=0, atol=1e-12)
        np.testing.assert_allclose(L[:, q0:q1], Lb[0], rtol=0, atol=1e-12)


def test_varlen_equal_lengths_equal_dense_batch():
    B, T = 3, 11
    q, k, v, cu_q, cu_k = _varlen_case(41, [T] * B, [T] * B)
    O, L = orc.attention_varlen(q, k, v, cu_q, cu_k, 0.3, True)
    Od, Ld = orc.attention(q.reshape(B, T, 4, 8), k.reshape(B, T, 2, 8), v.reshape(B, T, 2, 8), 0.3, True)
    np.testing.assert_array_equal(O, Od.reshape(B * T, 4, 8))
    np.testing.assert_array_equal(L, Ld.transpose(1, 0, 2).reshape(4, B * T))


def test_varlen_sequences_do_not_see_each_other():
    q, k, v, cu_q, cu_k = _varlen_case(42, [4, 6, 3], [5, 6, 2])
    O1, L1 = orc.attention_varlen(q, k, v, cu_q, cu_k, 0.3, True)
    k2, v2 = k.copy(), v.copy()
    k2[cu_k[1]:] = 100.0  # rewrite the keys/values of sequences 1 and 2
    v2[cu_k[1]:] = -7.0
    O2, L2 = orc.attention_varlen(q, k2, v2, cu_q, cu_k, 0.3, True)
    np.testing.assert_array_equal(O1[:cu_q[1]], O2[:cu_q[1]])
    np.testing.assert_array_equal(L1[:, :cu_q[1]], L2[:, :cu_q[1]])


def _chunked_case(seed, ctx, qlens, bs=4, max_blocks=10, Hq=4, Hkv=2, d=8):
    rng = np.random.default_rng(seed)
    nblk = [(c + bs - 1) // bs for c in ctx]
    pool = sum(nblk) + 2
    perm = rng.permutation(pool)
    table = -np.ones((len(ctx), max_blocks), dtype=np.int32)
    at = 0
    for b, n in enumerate(nblk):
        table[b, :n] = perm[at:at + n]
        at += n
    cu_q = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int64)
    q = rng.standard_normal((cu_q[-1], Hq, d))
    kc = rng.standard_normal((pool, bs, Hkv, d))
    vc = rng.standard_normal((pool, bs, Hkv, d))
    return q, kc, vc, table, np.array(ctx), cu_q, bs


def test_paged_prefill_one_token_is_decode():
    q, kc, vc, table, lens, cu_q, bs = _chunked_case(50, [7, 13, 1, 30], [1, 1, 1, 1])
    O, L = orc.paged_prefill(q, kc, vc, table, lens, cu_q, bs, 0.3, True)
    Od, Ld = orc.paged_decode(q, kc, vc, table, lens, bs, 0.3)
    np.testing.assert_allclose(O, Od, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L, Ld.T, rtol=0, atol=1e-12)


def test_paged_prefill_equals_contiguous_tail_rows():
    """The new tokens are the last rows of a causal prefill over the whole
    context written out position by position (independent of the gather)."""
    ctx, qlens = [9, 17, 30], [4, 17, 3]
    q, kc, vc, table, lens, cu_q, bs = _chunked_case(51, ctx, qlens)
    O, L = orc.paged_prefill(q, kc, vc, table, lens, cu_q, bs, 0.3, True)
    for b, (c, t) in enumerate(zip(ctx, qlens)):
        K = np.stack([kc[table[b, p // bs], p % bs] for p in range(c)])[None]
        V = np.stack([vc[table[b, p // bs], p % bs] for p in range(c)])[None]
        Q = np.zeros((1, c, q.shape[1], q.shape[2]))
        Q[0, c - t:] = q[cu_q[b]:cu_q[b + 1]]
        Of, Lf = orc.attention(Q, K, V, 0.3, True)
        np.testing.assert_allclose(O[cu_q[b]:cu_q[b + 1]], Of[0, c - t:], rtol=0, atol=1e-12)
        np.testing.assert_allclose(L[:, cu_q[b]:cu_q[b + 1]], Lf[0, :, c - t:], rtol=0, atol=1e-12)


def test_e4m3_decoder_hand_values_and_torch():
    # hand values from the format: 0x38 = 2^0, 0x7e = 448 (largest), 0x01 = 2^-9,
    # 0x08 = 2^-6 (smallest normal), 0xb0 = -0.5, 0x7f = NaN
    got = orc.decode_e4m3([0x38, 0x7E, 0x01, 0x08, 0xB0, 0x00, 0x80, 0x3C])
    np.testing.assert_array_equal(got, [1.0, 448.0, 2.0 ** -9, 2.0 ** -6, -0.5, 0.0, -0.0, 1.5])
    assert np.isnan(orc.decode_e4m3([0x7F, 0xFF])).all()
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(orc.decode_e4m3(codes), ref)


# ---- pool bound and seq_len clamp (readings: an id outside the pool masks its
# positions; a seq_len beyond the table row's capacity is clamped to it) ----

def test_pool_bound_that_holds_every_id_changes_nothing():
    q, kc, vc, table, lens, bs = _paged_case(60)
    O1, L1 = orc.paged_decode(q, kc, vc, table, lens, bs, 0.3)
    O2, L2 = orc.paged_decode(q, kc, vc, table, lens, bs, 0.3, num_blocks=kc.shape[0])
    np.testing.assert_array_equal(O1, O2)
    np.testing.assert_array_equal(L1, L2)


def test_masked_blocks_equal_a_cache_without_them():
    """Ids at or past num_blocks (and negative ones) drop their positions:
    the result equals the decode over a new cache that holds only the other
    positions, written out position by position into fresh blocks."""
    q, kc, vc, table, lens, bs = _paged_case(61)
    nb = kc.shape[0] // 2
    t2 = table.copy()
    t2[2, 1] = -5  # a negative id inside the sequence
    O, L = orc.paged_decode(q, kc, vc, t2, lens, bs, 0.3, num_blocks=nb)
    assert (t2[lens > 0] >= nb).any()  # some sequences lose blocks
    for b in range(len(lens)):
        keep = [p for p in range(int(lens[b])) if 0 <= t2[b, p // bs] < nb]
        n = len(keep)
        kb = np.zeros((max(1, -(-n // bs)), bs) + kc.shape[2:])
        vb = np.zeros_like(kb)
        for i, p in enumerate(keep):
            kb[i // bs, i % bs] = kc[t2[b, p // bs], p % bs]
            vb[i // bs, i % bs] = vc[t2[b, p // bs], p % bs]
        tb = np.arange(kb.shape[0])[None]
        Oc, Lc = orc.paged_decode(q[b:b + 1], kb, vb, tb, [n], bs, 0.3)
        np.testing.assert_allclose(O[b], Oc[0], rtol=0, atol=1e-12)
        np.testing.assert_allclose(L[b], Lc[0], rtol=0, atol=1e-12)
        if n == 0:
            assert np.all(O[b] == 0) and np.all(np.isneginf(L[b]))


def test_seq_len_beyond_the_table_row_is_clamped():
    q, kc, vc, table, lens, bs = _paged_case(62)
    cap = table.shape[1] * bs
    full = np.full_like(lens, cap)
    t2 = np.where(table >= 0, table, 0)  # every entry a valid id
    O1, L1 = orc.paged_decode(q, kc, vc, t2, full, bs, 0.3)
    O2, L2 = orc.paged_decode(q, kc, vc, t2, full + 1000, bs, 0.3)
    np.testing.assert_array_equal(O1, O2)
    np.testing.assert_array_equal(L1, L2)
    O3, L3 = orc.paged_decode(q, kc, vc, t2, -full, bs, 0.3)
    assert np.all(O3 == 0) and np.all(np.isneginf(L3))


def test_paged_prefill_with_masked_blocks_brute_force():
    """Chunked prefill with some ids outside the pool, against a loop over
    the positions in Python floats: row i of sequence b sits at position
    L - T + i and sees the kept positions up to it."""
    ctx, qlens = [9, 17, 30, 6], [4, 17, 3, 6]
    q, kc, vc, table, lens, cu_q, bs = _chunked_case(63, ctx, qlens)
    nb = kc.shape[0] - 4
    t2 = table.copy()
    t2[1, 2] = -1
    t2[2, 0] = nb + 1
    t2[3, :] = nb  # every block of sequence 3 outside the pool
    lens = np.array(ctx)
    lens[0] = 10 ** 6  # clamped to the row's capacity (10 blocks of 4)
    t2[0, :10] = np.where(t2[0, :10] >= 0, t2[0, :10], 0)
    for causal in (True, False):
        O, L = orc.paged_prefill(q, kc, vc, t2, lens, cu_q, bs, 0.3, causal, num_blocks=nb)
        Hq, Hkv = q.shape[1], kc.shape[2]
        for b in range(len(ctx)):
            S = min(max(int(lens[b]), 0), t2.shape[1] * bs)
            T = int(cu_q[b + 1] - cu_q[b])
            for i in range(T):
                r = int(cu_q[b]) + i
                for h in range(Hq):
                    hk = h // (Hq // Hkv)
                    ps = [p for p in range(S) if 0 <= t2[b, p // bs] < nb and (not causal or p <= S - T + i)]
                    if not ps:
                        assert np.all(O[r, h] == 0) and L[h, r] == -np.inf
                        continue
                    sc = [0.3 * sum(q[r, h, c] * kc[t2[b, p // bs], p % bs, hk, c] for c in range(q.shape[2]))
                          for p in ps]
                    m = max(sc)
                    w = [math.exp(x - m) for x in sc]
                    ref = [sum(wj * vc[t2[b, p // bs], p % bs, hk, c] for wj, p in zip(w, ps)) / sum(w)
                           for c in range(q.shape[2])]
                    np.testing.assert_allclose(O[r, h], ref, rtol=0, atol=1e-12)
                    assert abs(L[h, r] - (m + math.log(sum(w)))) < 1e-12
