"""Plain fp64 CPU oracle for softmax attention and paged-KV decode.

TEST INFRASTRUCTURE ONLY.  The tests, the smoke check and the CPU-baseline
leg of the benchmark import this module; the product path (the CUDA library
and its Python binding) never does, and this module imports nothing from it.

What is computed follows the page "Snelle attention-kernels en operatorfusie
versnellen AI-modellen" (the-ai.news), section "FlashAttention-type aandacht en
gepagineerde aandacht": classic attention forms a T x T score matrix per head,
turns each row into softmax weights and averages the values with them; the
blockwise FlashAttention schedule reaches the same function without storing
the matrix, so the oracle is that plain definition, one query row at a time:

    s_j  = scale * <q_i, k_j>            for every key j visible to row i
    m    = max_j s_j
    l    = sum_j exp(s_j - m)
    O_i  = sum_j exp(s_j - m) * v_j / l
    LSE_i = m + ln l

The same section fixes the paged cache: storage in fixed-size blocks, a block
table that maps logical positions to physical blocks, every position
translated through that table, and the number of logical elements unchanged.
The example there uses 16-token blocks.  The KV-cache passage of
"讨论CUDA图形优化与推理加速" (lzwjava.github.io), section "理解KV缓存", fixes
decode: the new token attends to the cached keys and values of the context.

Readings where the pages are silent (each listed in the design notes):
  * scale is an explicit argument (1/sqrt(d) in every workload);
  * causal masking is bottom-right aligned: row i sees key j iff
    j <= i + (S - T) (identical to j <= i when T == S);
  * grouped-query heads: query head h reads key/value head h // (Hq // Hkv);
  * a row with no visible key has O = 0 and LSE = -inf;
  * LSE is the natural log of the sum of exp of the *scaled* scores;
  * paged pool layout [num_blocks, block_size, Hkv, d]; block-table entries
    at or past ceil(seq_len / block_size) are never read;
  * a seq_len beyond the table row's capacity (row length x block_size) is
    clamped to it, a negative one to 0; when the pool size num_blocks is
    known, a table entry outside [0, num_blocks) names no block of the pool
    and its block_size positions are left out of the softmax (masked);
  * a decode query sits at position seq_len - 1 and sees all seq_len keys.

Inputs are float64 numpy arrays (bf16 tensors are widened exactly by the
caller); integer inputs are int32/int64 arrays.  Rows are evaluated in groups
only so that one numpy matrix product covers a group of rows: each row's
result depends on that row alone, exactly as in the definition above.
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "visible_key_count",
    "softmax_rows",
    "attention",
    "attention_varlen",
    "paged_positions",
    "gather_paged_kv",
    "paged_decode",
    "paged_prefill",
    "decode_e4m3",
    "split_paged_decode",
    "merge_partials",
]

_ROW_GROUP = 256  # rows per numpy matrix product (memory bound only)


def visible_key_count(i: int, T: int, S: int, causal: bool) -> int:
    """Number of keys row ``i`` may attend to (keys 0..count-1).

    Causal masking for a decoder prefill, bottom-right aligned so that the
    last query row always sees every key (the decode case is that last row).
    """
    if not causal:
        return S
    return max(0, min(S, i + (S - T) + 1))


def softmax_rows(scores: np.ndarray, counts: np.ndarray):
    """Row-wise softmax of ``scores`` [R, S] where row r keeps its first
    ``counts[r]`` entries and masks the rest.

    Returns (P [R, S] with masked entries exactly 0, m [R], l [R]) where
    P[r, j] = exp(s_rj - m_r) / l_r.  A row with no visible entry has P = 0,
    m = -inf and l = 0.  ("werkt het de statistieken van de softmax bij":
    m and l are the softmax statistics of the page's FlashAttention section.)
    """
    R, S = scores.shape
    cols = np.arange(S)[None, :]
    visible = cols < counts[:, None]
    masked = np.where(visible, scores, -np.inf)
    m = masked.max(axis=1) if S > 0 else np.full(R, -np.inf)
    safe_m = np.where(np.isfinite(m), m, 0.0)
    e = np.where(visible, np.exp(masked - safe_m[:, None]), 0.0)
    l = e.sum(axis=1)
    with np.errstate(invalid="ignore", divide="ignore"):
        P = np.where(l[:, None] > 0, e / np.where(l > 0, l, 1.0)[:, None], 0.0)
    return P, m, l


def attention(q, k, v, scale: float, causal: bool, rows=None, counts=None):
    """Softmax attention with grouped-query heads, fp64.

    q: [B, T, Hq, d]; k, v: [B, S, Hkv, d]  (float64)
    Returns O [B, T, Hq, d] and LSE [B, Hq, T].

    ``rows``: optional sorted iterable of query rows to evaluate (the others
    are left at O = 0, LSE = -inf).  Used to sample outputs of workloads too
    large to evaluate whole.
    ``counts``: optional [T] numbers of keys each row sees (keys
    0..counts[i]-1), in place of the causal / non-causal rule.  Used where
    some key positions of a paged cache are masked, so that the keys a row
    sees are a prefix of the keys that remain.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, T, Hq, d = q.shape
    S, Hkv = k.shape[1], k.shape[2]
    if Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    group = Hq // Hkv
    O = np.zeros((B, T, Hq, d))
    LSE = np.full((B, Hq, T), -np.inf)
    row_idx = np.arange(T) if rows is None else np.asarray(sorted(rows), dtype=np.int64)
    if row_idx.size == 0 or S == 0:
        return O, LSE
    if counts is None:
        counts_all = np.array([visible_key_count(int(i), T, S, causal) for i in row_idx])
    else:
        counts_all = np.asarray(counts, dtype=np.int64)[row_idx]
    for b in range(B):
        for h in range(Hq):
            hk = h // group  # grouped-query head map
            Kh = k[b, :, hk, :]  # [S, d]
            Vh = v[b, :, hk, :]
            for g0 in range(0, row_idx.size, _ROW_GROUP):
                ids = row_idx[g0:g0 + _ROW_GROUP]
                cnt = counts_all[g0:g0 + _ROW_GROUP]
                s = scale * (q[b, ids, h, :] @ Kh.T)  # [R, S] scores
                P, m, l = softmax_rows(s, cnt)
                O[b, ids, h, :] = P @ Vh
                with np.errstate(divide="ignore"):
                    LSE[b, h, ids] = np.where(l > 0, m + np.log(np.where(l > 0, l, 1.0)), -np.inf)
    return O, LSE


def attention_varlen(q, k, v, cu_q, cu_k, scale: float, causal: bool):
    """Packed sequences without padding ("dynamic sequence lengths without
    padding", FlashAttention-2 item of "内核更新内容一览", section 关键技术点).

    q: [total_q, Hq, d]; k, v: [total_k, Hkv, d]; cu_q, cu_k: [B + 1] prefix
    sums.  Sequence b is attended on its own (rows cu_q[b]..cu_q[b+1] against
    keys cu_k[b]..cu_k[b+1]) with `attention`.  Returns O [total_q, Hq, d]
    and LSE [Hq, total_q].
    """
    q = np.asarray(q, dtype=np.float64)
    total_q, Hq, d = q.shape
    O = np.zeros((total_q, Hq, d))
    LSE = np.full((Hq, total_q), -np.inf)
    for b in range(len(cu_q) - 1):
        q0, q1 = int(cu_q[b]), int(cu_q[b + 1])
        k0, k1 = int(cu_k[b]), int(cu_k[b + 1])
        if q1 == q0:
            continue
        ob, lb = attention(q[None, q0:q1], np.asarray(k)[None, k0:k1], np.asarray(v)[None, k0:k1], scale, causal)
        O[q0:q1] = ob[0]
        LSE[:, q0:q1] = lb[0]
    return O, LSE


def paged_positions(block_table_row, seq_len: int, block_size: int, num_blocks=None):
    """The logical positions of one sequence that take part in attention.

    Position p lives in physical block block_table_row[p // block_size] at
    slot p % block_size ("De aandachtskernel moet dan elke positie via deze
    tabel vertalen").  Positions run from 0 to seq_len - 1, with seq_len
    clamped to [0, len(row) * block_size] (the row cannot name more blocks).
    With ``num_blocks`` (the pool size) given, positions whose block id lies
    outside [0, num_blocks) are left out.  Only the table entries of
    positions below the clamped seq_len are read.

    Returns (pos, phys, slot, L): the kept positions (ascending), their
    physical block and slot, and the clamped length L.
    """
    row = np.asarray(block_table_row)
    L = min(max(int(seq_len), 0), row.shape[0] * block_size)
    pos = np.arange(L)
    phys = row[pos // block_size].astype(np.int64)
    slot = pos % block_size
    if num_blocks is not None:
        keep = (phys >= 0) & (phys < int(num_blocks))
        pos, phys, slot = pos[keep], phys[keep], slot[keep]
    return pos, phys, slot, L


def gather_paged_kv(k_cache, v_cache, block_table_row, seq_len: int, block_size: int, num_blocks=None):
    """Logical K/V of one sequence, read through its block-table row at the
    positions ``paged_positions`` keeps.  Returns (K [n, Hkv, d],
    V [n, Hkv, d]) as copies of the pool entries: the values are moved,
    never changed.
    """
    _, phys, slot, _ = paged_positions(block_table_row, seq_len, block_size, num_blocks)
    return k_cache[phys, slot], v_cache[phys, slot]


def paged_decode(q, k_cache, v_cache, block_table, seq_lens, block_size: int, scale: float, num_blocks=None):
    """Single-token decode against a paged KV cache, fp64.

    q: [B, Hq, d]; k_cache, v_cache: [pool, block_size, Hkv, d];
    block_table: [B, max_blocks] int; seq_lens: [B] int.
    Each query sits at position seq_len - 1 and sees all seq_len cached keys
    (the positions ``paged_positions`` keeps; ``num_blocks``: the pool size,
    when entries outside it are to be masked).  A query that sees no key
    gets O = 0, LSE = -inf.  Returns O [B, Hq, d], LSE [B, Hq].
    """
    q = np.asarray(q, dtype=np.float64)
    B, Hq, d = q.shape
    O = np.zeros((B, Hq, d))
    LSE = np.full((B, Hq), -np.inf)
    for b in range(B):
        Kb, Vb = gather_paged_kv(k_cache, v_cache, block_table[b], seq_lens[b], block_size, num_blocks)
        if Kb.shape[0] == 0:
            continue
        ob, lb = attention(q[b][None, None], Kb[None], Vb[None], scale, causal=False)
        O[b] = ob[0, 0]
        LSE[b] = lb[0, :, 0]
    return O, LSE


def paged_prefill(q, k_cache, v_cache, block_table, seq_lens, cu_q, block_size: int, scale: float, causal: bool,
                  num_blocks=None):
    """Chunked prefill against a paged cache, fp64.

    q: [total_q, Hq, d] (the new tokens of every sequence, back to back,
    rows cu_q[b]..cu_q[b+1]); the cache holds seq_lens[b] tokens of
    sequence b, the new ones included as its last T_b tokens.  The logical
    K/V are gathered through the block table, then `attention` is applied
    with T = T_b and S = seq_lens[b] (bottom-right causal alignment: the new
    token i sits at position S - T + i and sees the positions up to its own).
    Positions that ``paged_positions`` leaves out (``num_blocks`` given, an
    entry outside the pool) are seen by no row; S is the clamped length.
    Returns O [total_q, Hq, d] and LSE [Hq, total_q].
    """
    q = np.asarray(q, dtype=np.float64)
    total_q, Hq, d = q.shape
    O = np.zeros((total_q, Hq, d))
    LSE = np.full((Hq, total_q), -np.inf)
    for b in range(len(cu_q) - 1):
        q0, q1 = int(cu_q[b]), int(cu_q[b + 1])
        if q1 == q0:
            continue
        pos, phys, slot, L = paged_positions(block_table[b], seq_lens[b], block_size, num_blocks)
        Kb, Vb = k_cache[phys, slot], v_cache[phys, slot]
        T = q1 - q0
        # row i sees the kept positions p <= L - T + i (all of them if not causal)
        limit = [L - T + i if causal else L - 1 for i in range(T)]
        counts = np.searchsorted(pos, limit, side="right")
        ob, lb = attention(q[None, q0:q1], Kb[None], Vb[None], scale, causal, counts=counts)
        O[q0:q1] = ob[0]
        LSE[:, q0:q1] = lb[0]
    return O, LSE


def decode_e4m3(codes):
    """Exact values of FP8 e4m3 codes (OCP "e4m3fn": sign bit, 4 exponent
    bits with bias 7, 3 mantissa bits; exponent 0 is subnormal; the two codes
    with all exponent and mantissa bits set are NaN; there is no infinity).
    Used to state the FP8 KV cache in fp64: K = k_scale * decode_e4m3(k_cache).
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    val = np.where(e == 0, np.ldexp(m / 8.0, -6), np.ldexp(1.0 + m / 8.0, e - 7))
    val = np.where((e == 15) & (m == 7), np.nan, val)
    return sign * val


def split_paged_decode(q, k_cache, v_cache, block_table, seq_lens, block_size: int,
                       scale: float, num_splits: int):
    """Split-KV decode followed by the log-sum-exp merge, fp64.

    The logical blocks of every sequence are cut into ``num_splits`` ranges of
    c = ceil(max_blocks / num_splits) blocks; split i covers blocks
    [i*c, (i+1)*c).  Each non-empty split yields a normalised partial output
    o_i and its lse_i over its own keys; the merge is

        M = max_i lse_i,  w_i = exp(lse_i - M),
        O = sum_i w_i o_i / sum_i w_i,   LSE = M + ln sum_i w_i

    which equals ``paged_decode`` in exact arithmetic because
    sum_i w_i * exp(M) = sum over all keys of exp(s_j).  (The merge step is
    not on the pages; it is how long contexts are spread over several CTAs.)
    """
    q = np.asarray(q, dtype=np.float64)
    B, Hq, d = q.shape
    max_blocks = np.asarray(block_table).shape[1]
    chunk = -(-max_blocks // num_splits)
    O = np.zeros((B, Hq, d))
    LSE = np.full((B, Hq), -np.inf)
    for b in range(B):
        L = int(seq_lens[b])
        if L == 0:
            continue
        Kb, Vb = gather_paged_kv(k_cache, v_cache, block_table[b], L, block_size)
        parts_o, parts_lse = [], []
        for i in range(num_splits):
            lo = i * chunk * block_size
            hi = min(L, (i + 1) * chunk * block_size)
            if lo >= hi:
                continue
            ob, lb = attention(q[b][None, None], Kb[None, lo:hi], Vb[None, lo:hi], scale, causal=False)
            parts_o.append(ob[0, 0])
            parts_lse.append(lb[0, :, 0])
        po = np.stack(parts_o)      # [n, Hq, d]
        pl = np.stack(parts_lse)    # [n, Hq]
        M = pl.max(axis=0)
        w = np.exp(pl - M[None, :])
        O[b] = (w[:, :, None] * po).sum(axis=0) / w.sum(axis=0)[:, None]
        LSE[b] = M + np.log(w.sum(axis=0))
    return O, LSE


def merge_partials(o_parts, lse_parts):
    """Merge of R attention results over disjoint key sets of the same
    queries, fp64.

    o_parts [R, ..., d]: each result normalised by its own sum; lse_parts
    [R, ...]: ln of that sum of exp of the scaled scores (-inf for a key set
    that is empty for that query, whose o is then ignored).  Softmax over the
    union of the sets, from the definition in the module docstring: with
    M = max_r lse_r and w_r = exp(lse_r - M), the full sum of exp(s_j) is
    e^M sum_r w_r and the full weighted value sum is e^M sum_r w_r o_r, so

        O = sum_r w_r o_r / sum_r w_r,   LSE = M + ln sum_r w_r.

    A query with every lse_r = -inf gets O = 0, LSE = -inf.  Returns
    (O [..., d], LSE [...]).
    """
    po = np.asarray(o_parts, dtype=np.float64)
    pl = np.asarray(lse_parts, dtype=np.float64)
    M = pl.max(axis=0)
    seen = np.isfinite(M)
    Ms = np.where(seen, M, 0.0)
    w = np.where(np.isneginf(pl), 0.0, np.exp(pl - Ms[None]))
    wsum = w.sum(axis=0)
    num = (w[..., None] * np.where(np.isneginf(pl)[..., None], 0.0, po)).sum(axis=0)
    O = np.where(seen[..., None], num / np.where(seen, wsum, 1.0)[..., None], 0.0)
    LSE = np.where(seen, Ms + np.log(np.where(seen, wsum, 1.0)), -np.inf)
    return O, LSE
