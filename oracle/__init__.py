"""fp64 CPU oracle (test infrastructure; never imported by the library)."""

from .attention import (  # noqa: F401
    NEG_INF,
    allowed_keys,
    attention_ref,
    bf16_bits_to_f64,
    e4m3_bits_to_f64,
    gather_kv,
    lse_combine_ref,
    mha_ref,
    online_softmax_attention_ref,
    page_count,
    paged_attention_ref,
    resolve,
    softmax_rows,
    split_partial_ref,
    to_f64,
)
