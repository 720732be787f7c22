"""Shared helpers for the GPU parity tests: run the CUDA path through the
C ABI binding, run the fp64 oracle on the same seeded inputs, compare."""

from __future__ import annotations

import numpy as np
import torch

from oracle import fp64_attention as orc

# Tolerances for bf16 inputs with fp32 accumulation (P rounded to bf16 before
# P V, O rounded to bf16 at the end).
MAX_ABS_O = 2e-2
MEAN_ABS_O = 2e-3
MAX_ABS_LSE = 1e-3


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").to(torch.float64).numpy()


def check_close(o_gpu, o_ref, lse_gpu=None, lse_ref=None, what=""):
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    assert np.all(np.isfinite(o_gpu)), f"{what}: non-finite output"
    d = np.abs(o_gpu - o_ref)
    assert d.max() <= MAX_ABS_O, f"{what}: max|dO| = {d.max():.3e}"
    assert d.mean() <= MEAN_ABS_O, f"{what}: mean|dO| = {d.mean():.3e}"
    if lse_gpu is not None:
        lg = np.asarray(lse_gpu, dtype=np.float64)
        lr = np.asarray(lse_ref, dtype=np.float64)
        assert np.array_equal(np.isneginf(lg), np.isneginf(lr)), f"{what}: -inf pattern of LSE differs"
        fin = np.isfinite(lr)
        assert np.all(np.isfinite(lg[fin])), f"{what}: non-finite LSE"
        dl = np.abs(lg[fin] - lr[fin]) if fin.any() else np.zeros(1)
        assert dl.max() <= MAX_ABS_LSE, f"{what}: max|dLSE| = {dl.max():.3e}"
    return float(d.max()), float(d.mean())


def run_prefill(q, k, v, causal, scale, with_lse=True):
    """q [B,T,Hq,d], k/v [B,S,Hkv,d] bf16 CPU tensors -> (O bf16 CPU, LSE fp32 CPU)."""
    import flashattention_attention_attn_b200 as fa
    B, T, Hq, d = q.shape
    S, Hkv = k.shape[1], k.shape[2]
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    o = torch.full_like(dq, float("nan"))
    lse = torch.full((B, Hq, T), float("nan"), device="cuda", dtype=torch.float32) if with_lse else None
    fa.attn_fwd(dq, dk, dv, o, lse, B, Hq, Hkv, T, S, d, causal, scale)
    torch.cuda.synchronize()
    assert fa.attn_read_device_status(clear=True) == 0
    return o.cpu(), (lse.cpu() if lse is not None else None)


def run_decode(inp, num_splits=0, Hq=None, Hkv=None):
    import flashattention_attention_attn_b200 as fa
    B, Hq_, d = inp.q.shape
    Hkv_ = inp.k_cache.shape[2]
    o = torch.full((B, Hq_, d), float("nan"), device="cuda", dtype=torch.bfloat16)
    fa.paged_attn_decode(inp.q.cuda(), inp.k_cache.cuda(), inp.v_cache.cuda(), inp.block_table.cuda(),
                         inp.seq_lens.cuda(), B, Hq_, Hkv_, d, inp.block_size, inp.block_table.shape[1],
                         num_splits, o)
    torch.cuda.synchronize()
    assert fa.attn_read_device_status(clear=True) == 0
    return o.cpu()


def oracle_prefill(q, k, v, causal, scale, rows=None):
    return orc.attention(f64(q), f64(k), f64(v), scale, causal, rows=rows)


def oracle_decode(inp):
    d = inp.q.shape[-1]
    return orc.paged_decode(f64(inp.q), f64(inp.k_cache), f64(inp.v_cache), inp.block_table.numpy(),
                            inp.seq_lens.numpy(), inp.block_size, 1.0 / np.sqrt(d))


def run_varlen(inp, causal, scale, max_q=None):
    import flashattention_attention_attn_b200 as fa
    total_q, Hq, d = inp.q.shape
    total_k, Hkv = inp.k.shape[0], inp.k.shape[1]
    B = inp.cu_q.numel() - 1
    dq, dk, dv = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    o = torch.full_like(dq, float("nan"))
    lse = torch.full((Hq, total_q), float("nan"), device="cuda", dtype=torch.float32)
    fa.attn_fwd_varlen(dq, dk, dv, o, lse, inp.cu_q.cuda(), inp.cu_k.cuda(), B,
                       inp.max_q if max_q is None else max_q, total_q, total_k, Hq, Hkv, d, causal, scale)
    torch.cuda.synchronize()
    assert fa.attn_read_device_status(clear=True) == 0
    return o.cpu(), lse.cpu()


def oracle_varlen(inp, causal, scale):
    return orc.attention_varlen(f64(inp.q), f64(inp.k), f64(inp.v), inp.cu_q.numpy(), inp.cu_k.numpy(), scale, causal)


def run_chunked(inp, causal, scale):
    import flashattention_attention_attn_b200 as fa
    total_q, Hq, d = inp.q.shape
    c = inp.cache
    Hkv = c.k_cache.shape[2]
    B = inp.cu_q.numel() - 1
    dq = inp.q.cuda()
    o = torch.full_like(dq, float("nan"))
    lse = torch.full((Hq, total_q), float("nan"), device="cuda", dtype=torch.float32)
    fa.paged_attn_prefill(dq, c.k_cache.cuda(), c.v_cache.cuda(), c.block_table.cuda(), c.seq_lens.cuda(),
                          inp.cu_q.cuda(), B, Hq, Hkv, d, c.block_size, c.block_table.shape[1], inp.max_q, total_q,
                          causal, scale, o, lse)
    torch.cuda.synchronize()
    assert fa.attn_read_device_status(clear=True) == 0
    return o.cpu(), lse.cpu()


def oracle_chunked(inp, causal, scale):
    c = inp.cache
    return orc.paged_prefill(f64(inp.q), f64(c.k_cache), f64(c.v_cache), c.block_table.numpy(), c.seq_lens.numpy(),
                             inp.cu_q.numpy(), c.block_size, scale, causal)


def run_decode_fp8(inp, num_splits=0):
    import flashattention_attention_attn_b200 as fa
    B, Hq, d = inp.q.shape
    Hkv = inp.k_cache.shape[2]
    o = torch.full((B, Hq, d), float("nan"), device="cuda", dtype=torch.bfloat16)
    fa.paged_attn_decode_fp8(inp.q.cuda(), inp.k_cache.cuda(), inp.v_cache.cuda(), inp.block_table.cuda(),
                             inp.seq_lens.cuda(), B, Hq, Hkv, d, inp.block_size, inp.block_table.shape[1],
                             num_splits, inp.k_scale, inp.v_scale, o)
    torch.cuda.synchronize()
    assert fa.attn_read_device_status(clear=True) == 0
    return o.cpu()


def oracle_decode_fp8(inp):
    d = inp.q.shape[-1]
    K = inp.k_scale * orc.decode_e4m3(inp.k_cache.numpy())
    V = inp.v_scale * orc.decode_e4m3(inp.v_cache.numpy())
    return orc.paged_decode(f64(inp.q), K, V, inp.block_table.numpy(), inp.seq_lens.numpy(), inp.block_size,
                            1.0 / np.sqrt(d))
