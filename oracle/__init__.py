"""fp64 CPU oracle for the KV-cache decode step (test infrastructure only).

Only the test suite, ``__graft_entry__.smoke()`` and the bench's CPU-baseline
and reference legs may import this package; the CUDA library never does.
"""
from .kv_decode import (  # noqa: F401
    append_rope,
    attend,
    attend_partial,
    bf16_round,
    decode_attention,
    decode_attention_rows,
    decode_attention_shard,
    full_causal_attention,
    gather_tokens,
    max_abs_diff,
    merge_partials,
    rope,
    rope_inv_freq,
    rotate_new_tokens,
    round_store,
)
