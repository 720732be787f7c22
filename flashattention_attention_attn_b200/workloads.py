"""Algorithmic work of each call, for roofline accounting (no attention
arithmetic here: only counts of pairs, FLOPs and bytes).

Prefill FLOPs: every visible (query, key) pair costs 2*d for the score and
2*d for the value accumulation, so FLOPs = 4 * d * pairs * Hq * B; masked
pairs are not counted.

Decode bytes: every cached K and V element of every sequence is read once
(2 tensors x L x Hkv x d x 2 bytes), plus q and o (bf16), the block-table
entries that are used and seq_lens.
"""

from __future__ import annotations

import math


def visible_pairs(T: int, S: int, causal: bool) -> int:
    """Sum over rows i of the keys row i sees (bottom-right causal)."""
    if not causal:
        return T * S
    off = S - T
    total = 0
    # rows with i + off + 1 <= 0 see nothing; rows with i + off + 1 >= S see S
    lo = max(0, -off)                 # first row that sees >= 1 key
    hi = min(T, S - off - 1)          # rows [lo, hi) see i + off + 1 < S keys
    if hi > lo:
        a, b = lo + off + 1, hi - 1 + off + 1
        total += (a + b) * (hi - lo) // 2
    full_from = max(lo, hi, 0)
    total += max(0, T - full_from) * S
    return total


def prefill_flops(B: int, Hq: int, T: int, S: int, d: int, causal: bool) -> int:
    return 4 * d * visible_pairs(T, S, causal) * Hq * B


def prefill_min_bytes(B: int, Hq: int, Hkv: int, T: int, S: int, d: int) -> int:
    """Compulsory HBM traffic: read Q, K, V once, write O (bf16) and LSE (fp32)."""
    return 2 * d * (B * T * Hq * 2 + B * S * Hkv * 2) + 4 * B * Hq * T


def decode_bytes(seq_lens, Hq: int, Hkv: int, d: int, block_size: int, kv_elem_bytes: int = 2) -> int:
    """kv_elem_bytes: 2 for a bf16 cache, 1 for an FP8 cache."""
    lens = [int(x) for x in seq_lens]
    B = len(lens)
    kv = sum(lens) * Hkv * d * kv_elem_bytes * 2
    qo = 2 * B * Hq * d * 2
    table = sum(math.ceil(L / block_size) for L in lens) * 4 + B * 4
    return kv + qo + table
