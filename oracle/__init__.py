"""fp64 CPU oracle (test infrastructure; never used by the product path)."""
from .fp64_attention import (  # noqa: F401
    attention,
    attention_varlen,
    decode_e4m3,
    gather_paged_kv,
    paged_decode,
    paged_prefill,
    softmax_rows,
    split_paged_decode,
    visible_key_count,
)
