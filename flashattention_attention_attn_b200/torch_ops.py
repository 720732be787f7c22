"""torch custom ops over the C ABI, so that the kernels compose with
torch.compile (no graph break: the ops have fake/meta implementations that
give output shapes without running anything) and with CUDA-graph capture.

    import flashattention_attention_attn_b200.torch_ops  # registers the ops
    o, lse = torch.ops.fa_b200.attn_fwd(q, k, v, causal, scale)
    o, lse = torch.ops.fa_b200.attn_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, causal, scale)
    o, lse = torch.ops.fa_b200.paged_attn_prefill(q, k_cache, v_cache, block_table, seq_lens, cu_seqlens_q,
                                                  max_seqlen_q, causal, scale)
    o = torch.ops.fa_b200.paged_attn_decode(q, k_cache, v_cache, block_table, seq_lens, num_splits)
    o = torch.ops.fa_b200.paged_attn_decode_fp8(q, k_cache, v_cache, block_table, seq_lens, num_splits,
                                                k_scale, v_scale)
    o_part, lse_part = torch.ops.fa_b200.paged_attn_decode_partial(q, k_cache, v_cache, block_table, seq_lens,
                                                                   num_splits)
    o = torch.ops.fa_b200.attn_lse_merge(o_parts, lse_parts)

The op bodies only allocate the outputs and call the library on the current
stream; there is no other path.  Shapes follow include/attn.h:
q [B,T,Hq,d], k/v [B,S,Hkv,d] -> o [B,T,Hq,d], lse [B,Hq,T];
packed q [total_q,Hq,d], k/v [total_k,Hkv,d], cu_seqlens int32 [B+1]
-> o [total_q,Hq,d], lse [Hq,total_q];
decode q [B,Hq,d], caches [num_blocks,16,Hkv,d] (bf16, or e4m3 bytes),
block_table [B,max_blocks], seq_lens [B] -> o [B,Hq,d];
partial decode (the keys held here, the pool size read from the cache
shape) -> o_part [B,Hq,d] fp32, lse_part [B,Hq] fp32; merge of R partials
o_parts [R,B,Hq,d], lse_parts [R,B,Hq] -> o [B,Hq,d] bf16.
"""

from __future__ import annotations

import torch

from . import _binding


@torch.library.custom_op("fa_b200::attn_fwd", mutates_args=())
def attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool,
             scale: float) -> tuple[torch.Tensor, torch.Tensor]:
    B, T, Hq, d = q.shape
    S, Hkv = k.shape[1], k.shape[2]
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, T), device=q.device, dtype=torch.float32)
    _binding.attn_fwd(q, k, v, o, lse, B, Hq, Hkv, T, S, d, causal, scale,
                      torch.cuda.current_stream(q.device))
    return o, lse


@attn_fwd.register_fake
def _(q, k, v, causal, scale):
    B, T, Hq, _ = q.shape
    return torch.empty_like(q), q.new_empty((B, Hq, T), dtype=torch.float32)


@torch.library.custom_op("fa_b200::paged_attn_decode", mutates_args=())
def paged_attn_decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, block_table: torch.Tensor,
                      seq_lens: torch.Tensor, num_splits: int) -> torch.Tensor:
    B, Hq, d = q.shape
    Hkv, block_size = k_cache.shape[2], k_cache.shape[1]
    o = torch.empty_like(q)
    _binding.paged_attn_decode(q, k_cache, v_cache, block_table, seq_lens, B, Hq, Hkv, d, block_size,
                               block_table.shape[1], num_splits, o, torch.cuda.current_stream(q.device))
    return o


@paged_attn_decode.register_fake
def _(q, k_cache, v_cache, block_table, seq_lens, num_splits):
    return torch.empty_like(q)


@torch.library.custom_op("fa_b200::attn_fwd_varlen", mutates_args=())
def attn_fwd_varlen(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens_q: torch.Tensor,
                    cu_seqlens_k: torch.Tensor, max_seqlen_q: int, causal: bool,
                    scale: float) -> tuple[torch.Tensor, torch.Tensor]:
    total_q, Hq, d = q.shape
    total_k, Hkv = k.shape[0], k.shape[1]
    B = cu_seqlens_q.shape[0] - 1
    o = torch.empty_like(q)
    lse = torch.empty((Hq, total_q), device=q.device, dtype=torch.float32)
    _binding.attn_fwd_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, B, max_seqlen_q, total_q, total_k, Hq,
                             Hkv, d, causal, scale, torch.cuda.current_stream(q.device))
    return o, lse


@attn_fwd_varlen.register_fake
def _(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, causal, scale):
    total_q, Hq, _ = q.shape
    return torch.empty_like(q), q.new_empty((Hq, total_q), dtype=torch.float32)


@torch.library.custom_op("fa_b200::paged_attn_prefill", mutates_args=())
def paged_attn_prefill(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, block_table: torch.Tensor,
                       seq_lens: torch.Tensor, cu_seqlens_q: torch.Tensor, max_seqlen_q: int, causal: bool,
                       scale: float) -> tuple[torch.Tensor, torch.Tensor]:
    total_q, Hq, d = q.shape
    Hkv, block_size = k_cache.shape[2], k_cache.shape[1]
    B = cu_seqlens_q.shape[0] - 1
    o = torch.empty_like(q)
    lse = torch.empty((Hq, total_q), device=q.device, dtype=torch.float32)
    _binding.paged_attn_prefill(q, k_cache, v_cache, block_table, seq_lens, cu_seqlens_q, B, Hq, Hkv, d, block_size,
                                block_table.shape[1], max_seqlen_q, total_q, causal, scale, o, lse,
                                torch.cuda.current_stream(q.device))
    return o, lse


@paged_attn_prefill.register_fake
def _(q, k_cache, v_cache, block_table, seq_lens, cu_seqlens_q, max_seqlen_q, causal, scale):
    total_q, Hq, _ = q.shape
    return torch.empty_like(q), q.new_empty((Hq, total_q), dtype=torch.float32)


@torch.library.custom_op("fa_b200::paged_attn_decode_fp8", mutates_args=())
def paged_attn_decode_fp8(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, block_table: torch.Tensor,
                          seq_lens: torch.Tensor, num_splits: int, k_scale: float, v_scale: float) -> torch.Tensor:
    B, Hq, d = q.shape
    Hkv, block_size = k_cache.shape[2], k_cache.shape[1]
    o = torch.empty_like(q)
    _binding.paged_attn_decode_fp8(q, k_cache, v_cache, block_table, seq_lens, B, Hq, Hkv, d, block_size,
                                   block_table.shape[1], num_splits, k_scale, v_scale, o,
                                   torch.cuda.current_stream(q.device))
    return o


@paged_attn_decode_fp8.register_fake
def _(q, k_cache, v_cache, block_table, seq_lens, num_splits, k_scale, v_scale):
    return torch.empty_like(q)


@torch.library.custom_op("fa_b200::paged_attn_decode_partial", mutates_args=())
def paged_attn_decode_partial(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                              block_table: torch.Tensor, seq_lens: torch.Tensor,
                              num_splits: int) -> tuple[torch.Tensor, torch.Tensor]:
    B, Hq, d = q.shape
    num_blocks, block_size, Hkv = k_cache.shape[0], k_cache.shape[1], k_cache.shape[2]
    o_part = torch.empty((B, Hq, d), device=q.device, dtype=torch.float32)
    lse_part = torch.empty((B, Hq), device=q.device, dtype=torch.float32)
    if B > 0:  # the entry point takes no empty outputs
        _binding.paged_attn_decode_partial(q, k_cache, v_cache, block_table, seq_lens, B, Hq, Hkv, d, block_size,
                                           block_table.shape[1], num_blocks, num_splits, o_part, lse_part,
                                           torch.cuda.current_stream(q.device))
    return o_part, lse_part


@paged_attn_decode_partial.register_fake
def _(q, k_cache, v_cache, block_table, seq_lens, num_splits):
    B, Hq, _ = q.shape
    return q.new_empty(q.shape, dtype=torch.float32), q.new_empty((B, Hq), dtype=torch.float32)


@torch.library.custom_op("fa_b200::attn_lse_merge", mutates_args=())
def attn_lse_merge(o_parts: torch.Tensor, lse_parts: torch.Tensor) -> torch.Tensor:
    R, B, Hq, d = o_parts.shape
    o = torch.empty((B, Hq, d), device=o_parts.device, dtype=torch.bfloat16)
    if B > 0:
        _binding.attn_lse_merge(o_parts, lse_parts, R, B, Hq, d, o, torch.cuda.current_stream(o_parts.device))
    return o


@attn_lse_merge.register_fake
def _(o_parts, lse_parts):
    return o_parts.new_empty(o_parts.shape[1:], dtype=torch.bfloat16)
