"""Fused softmax attention for NVIDIA B200 (sm_100a).

Two entry points, both implemented by hand-written CUDA kernels in the
shared library built from ``csrc/`` (C ABI declared in ``include/attn.h``):

  attn_fwd           dense (causal) prefill with grouped-query heads
  paged_attn_decode  one-token decode against a paged KV cache, split-KV
                     with a log-sum-exp merge

The Python functions here only marshal arguments into that library; there is
no CPU fallback.  Importing the package does not load the library; the first
call does, and raises if it is missing.
"""

from . import inputs  # noqa: F401  (seeded synthetic inputs; no arithmetic)

_BINDING_NAMES = {
    "attn_fwd", "attn_fwd_varlen", "paged_attn_decode", "paged_attn_decode_fp8", "paged_attn_decode_noalloc",
    "paged_attn_prefill", "paged_attn_decode_checked", "paged_attn_decode_fp8_checked", "paged_attn_prefill_checked",
    "attn_check_support", "attn_status_string", "attn_read_device_status", "attn_selftest_bounded_wait", "library",
    "library_path", "AttnError", "ATTN_DEVSTATUS_TIMEOUT", "ATTN_DEVSTATUS_BAD_BLOCK", "ATTN_DEVSTATUS_BAD_SEQLEN",
}


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import _binding
        return getattr(_binding, name)
    raise AttributeError(name)
