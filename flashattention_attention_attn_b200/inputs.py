"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module draws random numbers and lays them out; it holds none of the
attention arithmetic.  Every tensor comes from a CPU ``torch.Generator``
seeded per workload, drawn as float32 N(0, 1) and rounded to bf16
(round-to-nearest-even), so the CUDA path and the fp64 oracle see the very
same values.

Workloads (all Llama3-8B-shaped except the tiny one):
  tiny_causal        B=1, H=2, T=S=128, d=64, causal; drawn in [B, H, T, d]
                     and handed to the library as [B, T, H, d]
  llama3_8b_prefill  B=2, Hq=32, Hkv=8, T=S=512, d=128, causal, [B, T, H, d]
  paged_decode_b64   B=64 one-token queries, Hq=32, Hkv=8, d=128,
                     block_size=16, context lengths uniform in [256, 4096],
                     every sequence's blocks a random permutation of the pool
  long_decode_131k   B=1, context 131072 (8192 blocks, permuted ids)
  long_prefill_16k   B=1, Hq=32, Hkv=8, T=S=16384, d=128, causal
"""

from __future__ import annotations

from dataclasses import dataclass, field

import torch

BF16 = torch.bfloat16


@dataclass(frozen=True)
class PrefillSpec:
    B: int
    Hq: int
    Hkv: int
    T: int
    S: int
    d: int
    causal: bool = True
    seed: int = 0
    drawn_layout: str = "BTHD"  # layout the values are drawn in

    @property
    def scale(self) -> float:
        return 1.0 / (self.d ** 0.5)


@dataclass(frozen=True)
class DecodeSpec:
    B: int
    Hq: int
    Hkv: int
    d: int
    block_size: int
    max_blocks: int
    ctx_lo: int
    ctx_hi: int
    seed: int = 0
    extra_pool_blocks: int = 0  # unused physical blocks added to the pool
    fixed_lens: tuple = field(default=())

    @property
    def scale(self) -> float:
        return 1.0 / (self.d ** 0.5)


WORKLOADS = {
    "tiny_causal": PrefillSpec(B=1, Hq=2, Hkv=2, T=128, S=128, d=64, causal=True, seed=1000,
                               drawn_layout="BHTD"),
    "llama3_8b_prefill": PrefillSpec(B=2, Hq=32, Hkv=8, T=512, S=512, d=128, causal=True, seed=1001),
    "paged_decode_b64": DecodeSpec(B=64, Hq=32, Hkv=8, d=128, block_size=16, max_blocks=256,
                                   ctx_lo=256, ctx_hi=4096, seed=1002),
    "long_decode_131k": DecodeSpec(B=1, Hq=32, Hkv=8, d=128, block_size=16, max_blocks=8192,
                                   ctx_lo=131072, ctx_hi=131072, seed=1003),
    "long_prefill_16k": PrefillSpec(B=1, Hq=32, Hkv=8, T=16384, S=16384, d=128, causal=True, seed=1004),
}


@dataclass(frozen=True)
class VarlenSpec:
    B: int
    Hq: int
    Hkv: int
    d: int
    len_lo: int
    len_hi: int
    causal: bool = True
    seed: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / (self.d ** 0.5)


# 16 packed Llama3-8B-shaped sequences, lengths uniform in [64, 2048]
VARLEN_WORKLOADS = {
    "varlen_prefill_16seq": VarlenSpec(B=16, Hq=32, Hkv=8, d=128, len_lo=64, len_hi=2048, causal=True, seed=1005),
}


def _randn_bf16(gen: torch.Generator, shape) -> torch.Tensor:
    return torch.randn(*shape, generator=gen, dtype=torch.float32).to(BF16)


def make_prefill(spec: PrefillSpec, seed: int | None = None):
    """Q [B,T,Hq,d], K [B,S,Hkv,d], V [B,S,Hkv,d] bf16 CPU tensors, contiguous.

    Values are drawn in the order Q, K, V.  For ``drawn_layout == "BHTD"`` the
    draw is in [B, H, T, d] order and the result is permuted to [B, T, H, d]
    (the layout the library takes) before it is returned.
    """
    gen = torch.Generator(device="cpu").manual_seed(spec.seed if seed is None else seed)
    s = spec
    if s.drawn_layout == "BHTD":
        q = _randn_bf16(gen, (s.B, s.Hq, s.T, s.d)).permute(0, 2, 1, 3).contiguous()
        k = _randn_bf16(gen, (s.B, s.Hkv, s.S, s.d)).permute(0, 2, 1, 3).contiguous()
        v = _randn_bf16(gen, (s.B, s.Hkv, s.S, s.d)).permute(0, 2, 1, 3).contiguous()
    else:
        q = _randn_bf16(gen, (s.B, s.T, s.Hq, s.d))
        k = _randn_bf16(gen, (s.B, s.S, s.Hkv, s.d))
        v = _randn_bf16(gen, (s.B, s.S, s.Hkv, s.d))
    return q, k, v


@dataclass
class PagedInputs:
    q: torch.Tensor            # [B, Hq, d] bf16
    k_cache: torch.Tensor      # [num_blocks, block_size, Hkv, d] bf16
    v_cache: torch.Tensor      # [num_blocks, block_size, Hkv, d] bf16
    block_table: torch.Tensor  # [B, max_blocks] int32, -1 where unused
    seq_lens: torch.Tensor     # [B] int32
    block_size: int

    @property
    def num_blocks(self) -> int:
        return int(self.k_cache.shape[0])


def make_paged(spec: DecodeSpec, seed: int | None = None, seq_lens=None) -> PagedInputs:
    """Paged decode inputs.

    Draw order: sequence lengths (uniform integers in [ctx_lo, ctx_hi], or
    ``seq_lens`` / ``spec.fixed_lens`` when given), a random permutation of
    the physical block ids, then q, the K pool and the V pool.  The pool holds
    sum(ceil(len / block_size)) blocks (+ ``extra_pool_blocks`` never
    referenced); the permuted ids are handed out in order, sequence 0 first.
    Unused block-table entries hold -1.
    """
    s = spec
    gen = torch.Generator(device="cpu").manual_seed(s.seed if seed is None else seed)
    if seq_lens is not None:
        lens = torch.as_tensor(list(seq_lens), dtype=torch.int64)
    elif s.fixed_lens:
        lens = torch.as_tensor(list(s.fixed_lens), dtype=torch.int64)
    else:
        lens = torch.randint(s.ctx_lo, s.ctx_hi + 1, (s.B,), generator=gen, dtype=torch.int64)
    assert lens.numel() == s.B
    nblk = [(int(L) + s.block_size - 1) // s.block_size for L in lens]
    if max(nblk, default=0) > s.max_blocks:
        raise ValueError("a sequence needs more blocks than max_blocks")
    pool = sum(nblk) + s.extra_pool_blocks
    perm = torch.randperm(max(pool, 1), generator=gen)[:pool].to(torch.int32)
    table = torch.full((s.B, s.max_blocks), -1, dtype=torch.int32)
    at = 0
    for b, n in enumerate(nblk):
        table[b, :n] = perm[at:at + n]
        at += n
    q = _randn_bf16(gen, (s.B, s.Hq, s.d))
    k_cache = _randn_bf16(gen, (max(pool, 1), s.block_size, s.Hkv, s.d))
    v_cache = _randn_bf16(gen, (max(pool, 1), s.block_size, s.Hkv, s.d))
    return PagedInputs(q=q, k_cache=k_cache, v_cache=v_cache, block_table=table,
                       seq_lens=lens.to(torch.int32), block_size=s.block_size)


def permute_pool(inp: PagedInputs, seed: int) -> PagedInputs:
    """The same logical cache stored under another physical-id permutation.

    Physical block p moves to slot perm[p]; the table is rewritten so that
    every logical position still names the same values.
    """
    gen = torch.Generator(device="cpu").manual_seed(seed)
    nb = inp.num_blocks
    perm = torch.randperm(nb, generator=gen)
    k2 = torch.empty_like(inp.k_cache)
    v2 = torch.empty_like(inp.v_cache)
    k2[perm] = inp.k_cache
    v2[perm] = inp.v_cache
    table = inp.block_table.clone()
    used = table >= 0
    table[used] = perm[table[used].long()].to(torch.int32)
    return PagedInputs(q=inp.q, k_cache=k2, v_cache=v2, block_table=table,
                       seq_lens=inp.seq_lens, block_size=inp.block_size)


@dataclass
class VarlenInputs:
    q: torch.Tensor      # [total_q, Hq, d] bf16
    k: torch.Tensor      # [total_k, Hkv, d] bf16
    v: torch.Tensor      # [total_k, Hkv, d] bf16
    cu_q: torch.Tensor   # [B + 1] int32
    cu_k: torch.Tensor   # [B + 1] int32

    @property
    def max_q(self) -> int:
        return int((self.cu_q[1:] - self.cu_q[:-1]).max()) if self.cu_q.numel() > 1 else 0


def make_varlen(spec: VarlenSpec, q_lens=None, k_lens=None, seed: int | None = None) -> VarlenInputs:
    """Packed sequences.  Draw order: query lengths (uniform in
    [len_lo, len_hi] unless given), then q, k, v.  Key lengths equal the
    query lengths (self-attention prefill) unless `k_lens` is given."""
    s = spec
    gen = torch.Generator(device="cpu").manual_seed(s.seed if seed is None else seed)
    if q_lens is None:
        q_lens = torch.randint(s.len_lo, s.len_hi + 1, (s.B,), generator=gen, dtype=torch.int64).tolist()
    q_lens = [int(x) for x in q_lens]
    k_lens = list(q_lens) if k_lens is None else [int(x) for x in k_lens]
    assert len(q_lens) == len(k_lens) == s.B
    cu_q = torch.zeros(s.B + 1, dtype=torch.int32)
    cu_k = torch.zeros(s.B + 1, dtype=torch.int32)
    cu_q[1:] = torch.cumsum(torch.tensor(q_lens, dtype=torch.int64), 0).to(torch.int32)
    cu_k[1:] = torch.cumsum(torch.tensor(k_lens, dtype=torch.int64), 0).to(torch.int32)
    q = _randn_bf16(gen, (int(cu_q[-1]), s.Hq, s.d))
    k = _randn_bf16(gen, (int(cu_k[-1]), s.Hkv, s.d))
    v = _randn_bf16(gen, (int(cu_k[-1]), s.Hkv, s.d))
    return VarlenInputs(q=q, k=k, v=v, cu_q=cu_q, cu_k=cu_k)


@dataclass(frozen=True)
class ChunkedSpec:
    """Chunked prefill against a paged cache: each sequence has ctx tokens in
    the cache, the last q_len of which are the new queries."""
    B: int
    Hq: int
    Hkv: int
    d: int
    block_size: int
    max_blocks: int
    ctx_lo: int
    ctx_hi: int
    q_lo: int
    q_hi: int
    causal: bool = True
    seed: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / (self.d ** 0.5)


# 8 Llama3-8B-shaped sequences with 1k..8k cached tokens, a new chunk of 512
CHUNKED_WORKLOADS = {
    "chunked_prefill_paged": ChunkedSpec(B=8, Hq=32, Hkv=8, d=128, block_size=16, max_blocks=512, ctx_lo=1024,
                                         ctx_hi=8192, q_lo=512, q_hi=512, causal=True, seed=1006),
}


@dataclass
class ChunkedInputs:
    q: torch.Tensor        # [total_q, Hq, d] bf16
    cu_q: torch.Tensor     # [B + 1] int32
    cache: PagedInputs     # pool, block table, seq_lens (its q is unused)

    @property
    def max_q(self) -> int:
        return int((self.cu_q[1:] - self.cu_q[:-1]).max()) if self.cu_q.numel() > 1 else 0


def make_chunked(spec: ChunkedSpec, ctx_lens=None, q_lens=None, seed: int | None = None) -> ChunkedInputs:
    """Draw order: context lengths (uniform in [ctx_lo, ctx_hi] unless given),
    query counts (uniform in [q_lo, q_hi], at most the context, unless
    given), then the paged cache as make_paged draws it (physical-id
    permutation, a decode q that is not used, the K pool, the V pool), then
    the queries."""
    s = spec
    gen = torch.Generator(device="cpu").manual_seed(s.seed if seed is None else seed)
    if ctx_lens is None:
        ctx_lens = torch.randint(s.ctx_lo, s.ctx_hi + 1, (s.B,), generator=gen, dtype=torch.int64).tolist()
    if q_lens is None:
        q_lens = torch.randint(s.q_lo, s.q_hi + 1, (s.B,), generator=gen, dtype=torch.int64).tolist()
    ctx_lens = [int(x) for x in ctx_lens]
    q_lens = [min(int(t), c) for t, c in zip(q_lens, ctx_lens)]
    dspec = DecodeSpec(B=s.B, Hq=s.Hq, Hkv=s.Hkv, d=s.d, block_size=s.block_size, max_blocks=s.max_blocks,
                       ctx_lo=0, ctx_hi=0, seed=int(torch.randint(0, 2 ** 31 - 1, (1,), generator=gen)))
    cache = make_paged(dspec, seq_lens=ctx_lens)
    cu_q = torch.zeros(s.B + 1, dtype=torch.int32)
    cu_q[1:] = torch.cumsum(torch.tensor(q_lens, dtype=torch.int64), 0).to(torch.int32)
    q = _randn_bf16(gen, (int(cu_q[-1]), s.Hq, s.d))
    return ChunkedInputs(q=q, cu_q=cu_q, cache=cache)


@dataclass
class PagedInputsFp8:
    """A paged cache stored as FP8 e4m3 codes with one scale per tensor."""
    q: torch.Tensor            # [B, Hq, d] bf16
    k_cache: torch.Tensor      # [num_blocks, block_size, Hkv, d] uint8 (e4m3 codes)
    v_cache: torch.Tensor      # same
    block_table: torch.Tensor
    seq_lens: torch.Tensor
    block_size: int
    k_scale: float
    v_scale: float


def make_paged_fp8(spec: DecodeSpec, seed: int | None = None, seq_lens=None, k_scale: float = 0.75,
                   v_scale: float = 1.25) -> PagedInputsFp8:
    """As make_paged (same draws), with the K and V pools rounded to e4m3
    (round to nearest even, values N(0, 1) fit without saturation) and kept
    as raw codes; the logical cache is k_scale * K and v_scale * V."""
    p = make_paged(spec, seed=seed, seq_lens=seq_lens)
    to8 = lambda t: t.to(torch.float32).to(torch.float8_e4m3fn).view(torch.uint8)  # noqa: E731
    return PagedInputsFp8(q=p.q, k_cache=to8(p.k_cache), v_cache=to8(p.v_cache), block_table=p.block_table,
                          seq_lens=p.seq_lens, block_size=p.block_size, k_scale=k_scale, v_scale=v_scale)
