"""Fused softmax attention for NVIDIA B200 (sm_100a).

Entry points, all implemented by hand-written CUDA kernels in the shared
library built from ``csrc/`` (C ABI declared in ``include/attn.h``):

  attn_fwd                   dense (causal) prefill with grouped-query heads
  attn_fwd_varlen            packed sequences of different lengths
  paged_attn_prefill         a chunk of new queries against a paged KV cache
  paged_attn_decode          one-token decode against a paged KV cache,
                             split-KV with a log-sum-exp merge (also _fp8 for
                             an e4m3 cache, _checked for a pool of known size,
                             _noalloc without any allocation)
  paged_attn_decode_partial  the decode over the keys held here, as fp32 o
                             and lse, and
  attn_lse_merge             the merge of such partials (context-parallel
                             decode, see dist_util.context_parallel_decode)

The Python functions here only marshal arguments into that library; there is
no CPU fallback.  Importing the package does not load the library; the first
call does, and raises if it is missing.
"""

from . import inputs  # noqa: F401  (seeded synthetic inputs; no arithmetic)

_BINDING_NAMES = {
    "attn_fwd", "attn_fwd_varlen", "paged_attn_decode", "paged_attn_decode_fp8", "paged_attn_decode_noalloc",
    "paged_attn_prefill", "paged_attn_decode_checked", "paged_attn_decode_fp8_checked", "paged_attn_prefill_checked",
    "paged_attn_decode_partial", "attn_lse_merge",
    "attn_check_support", "attn_status_string", "attn_read_device_status", "attn_selftest_bounded_wait", "library",
    "library_path", "AttnError", "ATTN_DEVSTATUS_TIMEOUT", "ATTN_DEVSTATUS_BAD_BLOCK", "ATTN_DEVSTATUS_BAD_SEQLEN",
}


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import _binding
        return getattr(_binding, name)
    raise AttributeError(name)
