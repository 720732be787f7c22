"""ctypes binding of the C ABI in include/attn.h.

Argument marshalling only: tensors become device pointers, the current
torch stream becomes the cudaStream_t, and a non-zero status becomes an
exception.  Every step of the computation runs in the CUDA library; if it
cannot be loaded, every call raises.
"""

from __future__ import annotations

import ctypes
import os

import torch

library_path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "_lib", "libattn_b200.so")

ATTN_OK = 0
ATTN_DEVSTATUS_TIMEOUT = 0x1
ATTN_DEVSTATUS_BAD_BLOCK = 0x2
ATTN_DEVSTATUS_BAD_SEQLEN = 0x4
_lib = None


class AttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {attn_status_string(status)} (status {status})")


def library() -> ctypes.CDLL:
    """Load the library once (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(library_path):
            raise RuntimeError(
                f"CUDA library not built: {library_path} is missing "
                "(run `python -m flashattention_attention_attn_b200.build`)")
        lib = ctypes.CDLL(library_path)
        c_int, c_float, vp = ctypes.c_int, ctypes.c_float, ctypes.c_void_p
        lib.attn_fwd.argtypes = [vp, vp, vp, vp, vp, c_int, c_int, c_int, c_int, c_int, c_int, c_int, c_float, vp]
        lib.attn_fwd.restype = c_int
        lib.attn_fwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, c_int, c_int, c_int, c_int, c_int, c_int, c_int,
                                        c_int, c_float, vp]
        lib.attn_fwd_varlen.restype = c_int
        lib.paged_attn_prefill.argtypes = [vp, vp, vp, vp, vp, vp, c_int, c_int, c_int, c_int, c_int, c_int, c_int,
                                           c_int, c_int, c_float, vp, vp, vp]
        lib.paged_attn_prefill.restype = c_int
        lib.paged_attn_decode.argtypes = [vp, vp, vp, vp, vp, c_int, c_int, c_int, c_int, c_int, c_int, c_int,
                                          vp, vp]
        lib.paged_attn_decode.restype = c_int
        lib.paged_attn_decode_fp8.argtypes = [vp, vp, vp, vp, vp, c_int, c_int, c_int, c_int, c_int, c_int, c_int,
                                              c_float, c_float, vp, vp]
        lib.paged_attn_decode_fp8.restype = c_int
        lib.paged_attn_decode_noalloc.argtypes = lib.paged_attn_decode.argtypes
        lib.paged_attn_decode_noalloc.restype = c_int
        lib.paged_attn_decode_checked.argtypes = [vp, vp, vp, vp, vp, c_int, c_int, c_int, c_int, c_int, c_int,
                                                  c_int, c_int, vp, vp]
        lib.paged_attn_decode_checked.restype = c_int
        lib.paged_attn_decode_fp8_checked.argtypes = [vp, vp, vp, vp, vp, c_int, c_int, c_int, c_int, c_int, c_int,
                                                      c_int, c_int, c_float, c_float, vp, vp]
        lib.paged_attn_decode_fp8_checked.restype = c_int
        lib.paged_attn_prefill_checked.argtypes = [vp, vp, vp, vp, vp, vp, c_int, c_int, c_int, c_int, c_int, c_int,
                                                   c_int, c_int, c_int, c_int, c_float, vp, vp, vp]
        lib.paged_attn_prefill_checked.restype = c_int
        lib.paged_attn_decode_partial.argtypes = [vp, vp, vp, vp, vp, c_int, c_int, c_int, c_int, c_int, c_int,
                                                  c_int, c_int, vp, vp, vp]
        lib.paged_attn_decode_partial.restype = c_int
        lib.attn_lse_merge.argtypes = [vp, vp, c_int, c_int, c_int, c_int, vp, vp]
        lib.attn_lse_merge.restype = c_int
        lib.attn_check_support.argtypes = [c_int]
        lib.attn_check_support.restype = c_int
        lib.attn_status_string.argtypes = [c_int]
        lib.attn_status_string.restype = ctypes.c_char_p
        lib.attn_read_device_status.argtypes = [ctypes.POINTER(c_int), c_int]
        lib.attn_read_device_status.restype = c_int
        lib.attn_selftest_bounded_wait.argtypes = [vp]
        lib.attn_selftest_bounded_wait.restype = c_int
        _lib = lib
    return _lib


def _ptr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, torch.Tensor):
        return x.data_ptr() if x.numel() > 0 else None
    return int(x)


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def attn_status_string(status: int) -> str:
    return library().attn_status_string(int(status)).decode()


def attn_fwd(q, k, v, o, lse, B, Hq, Hkv, T, S, d, causal, scale, stream=None) -> None:
    """O = softmax(scale * Q K^T [+ causal mask]) V, plus LSE.

    q [B,T,Hq,d], k/v [B,S,Hkv,d], o [B,T,Hq,d] bf16; lse [B,Hq,T] fp32 or None.
    """
    rc = library().attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), int(B), int(Hq), int(Hkv), int(T),
                            int(S), int(d), int(bool(causal)), float(scale), _stream(stream))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_fwd")


def attn_fwd_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, B, max_seqlen_q, total_q, total_k, Hq, Hkv, d,
                    causal, scale, stream=None) -> None:
    """attn_fwd over packed sequences: q [total_q,Hq,d], k/v [total_k,Hkv,d],
    o [total_q,Hq,d], lse [Hq,total_q] or None, cu_seqlens_* int32 [B+1]."""
    rc = library().attn_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(cu_seqlens_q),
                                   _ptr(cu_seqlens_k), int(B), int(max_seqlen_q), int(total_q), int(total_k),
                                   int(Hq), int(Hkv), int(d), int(bool(causal)), float(scale), _stream(stream))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_fwd_varlen")


def paged_attn_prefill(q, k_cache, v_cache, block_table, seq_lens, cu_seqlens_q, B, Hq, Hkv, d, block_size,
                       max_blocks, max_seqlen_q, total_q, causal, scale, o, lse, stream=None) -> None:
    """Chunked prefill against the paged cache (see attn.h)."""
    rc = library().paged_attn_prefill(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), _ptr(seq_lens),
                                      _ptr(cu_seqlens_q), int(B), int(Hq), int(Hkv), int(d), int(block_size),
                                      int(max_blocks), int(max_seqlen_q), int(total_q), int(bool(causal)),
                                      float(scale), _ptr(o), _ptr(lse), _stream(stream))
    if rc != ATTN_OK:
        raise AttnError(rc, "paged_attn_prefill")


def paged_attn_decode(q, k_cache, v_cache, block_table, seq_lens, B, Hq, Hkv, d, block_size, max_blocks,
                      num_splits, o, stream=None) -> None:
    """One query token per sequence against a paged KV cache (see attn.h)."""
    rc = library().paged_attn_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), _ptr(seq_lens),
                                     int(B), int(Hq), int(Hkv), int(d), int(block_size), int(max_blocks),
                                     int(num_splits), _ptr(o), _stream(stream))
    if rc != ATTN_OK:
        raise AttnError(rc, "paged_attn_decode")


def paged_attn_decode_fp8(q, k_cache, v_cache, block_table, seq_lens, B, Hq, Hkv, d, block_size, max_blocks,
                          num_splits, k_scale, v_scale, o, stream=None) -> None:
    """paged_attn_decode over an FP8 e4m3 cache with per-tensor scales (see attn.h)."""
    rc = library().paged_attn_decode_fp8(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), _ptr(seq_lens),
                                         int(B), int(Hq), int(Hkv), int(d), int(block_size), int(max_blocks),
                                         int(num_splits), float(k_scale), float(v_scale), _ptr(o), _stream(stream))
    if rc != ATTN_OK:
        raise AttnError(rc, "paged_attn_decode_fp8")


def paged_attn_decode_checked(q, k_cache, v_cache, block_table, seq_lens, B, Hq, Hkv, d, block_size, max_blocks,
                              num_blocks, num_splits, o, stream=None) -> None:
    """paged_attn_decode for a pool of num_blocks blocks: table entries
    outside it are masked and flagged (see attn.h)."""
    rc = library().paged_attn_decode_checked(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                                             _ptr(seq_lens), int(B), int(Hq), int(Hkv), int(d), int(block_size),
                                             int(max_blocks), int(num_blocks), int(num_splits), _ptr(o),
                                             _stream(stream))
    if rc != ATTN_OK:
        raise AttnError(rc, "paged_attn_decode_checked")


def paged_attn_decode_partial(q, k_cache, v_cache, block_table, seq_lens, B, Hq, Hkv, d, block_size, max_blocks,
                              num_blocks, num_splits, o_part, lse_part, stream=None) -> None:
    """Decode over the keys held here, as fp32 o_part [B, Hq, d] and
    lse_part [B, Hq] for a later attn_lse_merge (see attn.h)."""
    rc = library().paged_attn_decode_partial(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                                             _ptr(seq_lens), int(B), int(Hq), int(Hkv), int(d), int(block_size),
                                             int(max_blocks), int(num_blocks), int(num_splits), _ptr(o_part),
                                             _ptr(lse_part), _stream(stream))
    if rc != ATTN_OK:
        raise AttnError(rc, "paged_attn_decode_partial")


def attn_lse_merge(o_parts, lse_parts, R, B, Hq, d, o, stream=None) -> None:
    """Merge R partial results [R, B, Hq, d] / [R, B, Hq] into bf16 o [B, Hq, d] (see attn.h)."""
    rc = library().attn_lse_merge(_ptr(o_parts), _ptr(lse_parts), int(R), int(B), int(Hq), int(d), _ptr(o),
                                  _stream(stream))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_lse_merge")


def paged_attn_decode_fp8_checked(q, k_cache, v_cache, block_table, seq_lens, B, Hq, Hkv, d, block_size, max_blocks,
                                  num_blocks, num_splits, k_scale, v_scale, o, stream=None) -> None:
    """paged_attn_decode_fp8 for a pool of num_blocks blocks (see attn.h)."""
    rc = library().paged_attn_decode_fp8_checked(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                                                 _ptr(seq_lens), int(B), int(Hq), int(Hkv), int(d), int(block_size),
                                                 int(max_blocks), int(num_blocks), int(num_splits), float(k_scale),
                                                 float(v_scale), _ptr(o), _stream(stream))
    if rc != ATTN_OK:
        raise AttnError(rc, "paged_attn_decode_fp8_checked")


def paged_attn_prefill_checked(q, k_cache, v_cache, block_table, seq_lens, cu_seqlens_q, B, Hq, Hkv, d, block_size,
                               max_blocks, num_blocks, max_seqlen_q, total_q, causal, scale, o, lse,
                               stream=None) -> None:
    """paged_attn_prefill for a pool of num_blocks blocks (see attn.h)."""
    rc = library().paged_attn_prefill_checked(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                                              _ptr(seq_lens), _ptr(cu_seqlens_q), int(B), int(Hq), int(Hkv), int(d),
                                              int(block_size), int(max_blocks), int(num_blocks), int(max_seqlen_q),
                                              int(total_q), int(bool(causal)), float(scale), _ptr(o), _ptr(lse),
                                              _stream(stream))
    if rc != ATTN_OK:
        raise AttnError(rc, "paged_attn_prefill_checked")


def paged_attn_decode_noalloc(q, k_cache, v_cache, block_table, seq_lens, B, Hq, Hkv, d, block_size,
                              max_blocks, num_splits, o, stream=None) -> None:
    """paged_attn_decode with its split partials in the library's fixed
    scratch array: for callers that must not allocate during the call (see
    attn.h for the size limit and the sharing rules)."""
    rc = library().paged_attn_decode_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                                             _ptr(seq_lens), int(B), int(Hq), int(Hkv), int(d), int(block_size),
                                             int(max_blocks), int(num_splits), _ptr(o), _stream(stream))
    if rc != ATTN_OK:
        raise AttnError(rc, "paged_attn_decode_noalloc")


def attn_check_support(device: int = 0) -> int:
    return int(library().attn_check_support(int(device)))


def attn_read_device_status(clear: bool = True) -> int:
    out = ctypes.c_int(0)
    rc = library().attn_read_device_status(ctypes.byref(out), int(bool(clear)))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_read_device_status")
    return int(out.value)


def attn_selftest_bounded_wait(stream=None) -> None:
    """Launch the bounded-wait self test (see attn.h); read the outcome with
    attn_read_device_status()."""
    rc = library().attn_selftest_bounded_wait(_stream(stream))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_selftest_bounded_wait")
