"""Decode attention over a shared prefix, read once per group of sequences.

Sequences that start with the same tokens can share those tokens' pages (the
ferrox-models index's `prefix_cache`: the KV state of a shared leading
subsequence is reused instead of recomputed).  The plain paged decode then
reads the shared pages once per sequence; they come from L2 after the first
reader, but every SM still pulls every sequence's copy through its loads.

`cascade_decode` splits the keys at the end of the shared prefix and merges by
log-sum-exp, the split-K scheme of "Flash Decoding" (ferrum-sampler 0.7.0
README, Key Optimizations) applied along the prefix boundary:

1. prefix: G sequences at a time form one virtual sequence whose G * T query
   tokens (G * g * T rows per kv head, up to a full 128-row tensor-core tile)
   attend the shared pages together, so a prefix page is read once per group;
2. suffix: each sequence attends its own tokens (positions prefix_len ..
   L_b + T - 1, causal among the new tokens) on its private pages;
3. merge of the two (o, lse) per row.

Steps 1 and 2 are `decode_attention_shard` calls and step 3 is
`kvd_merge_partials`: everything runs in the library's kernels.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import decode_attention_shard, merge_partials


def group_size(batch: int, rows_per_seq: int, row_cap: int) -> int:
    """Largest divisor G of batch with G * rows_per_seq <= row_cap (at least 1)."""
    best = 1
    for G in range(1, batch + 1):
        if batch % G == 0 and G * rows_per_seq <= row_cap:
            best = G
    return best


def cascade_decode(q, k_cache, v_cache, seq_lens, block_table, prefix_len: int, *,
                   scale: Optional[float] = None, out=None, out_dtype=None):
    """Paged decode attention of ``q [B, T, Hq, D]`` (rotated) for a batch whose
    sequences all start with the same ``prefix_len`` tokens, held in the same
    pages: block_table[:, :prefix_len / page_size] is equal for every row, and
    prefix_len is a multiple of the page size.  Same result as
    decode_attention_paged."""
    B, T, Hq, D = q.shape
    Hkv, P = k_cache.shape[1], k_cache.shape[2]
    if prefix_len % P or prefix_len <= 0:
        raise ValueError("prefix_len must be a positive multiple of the page size")
    n_sh = prefix_len // P
    if block_table.shape[1] <= n_sh:
        raise ValueError("the block table has no private pages after the prefix")
    g = Hq // Hkv
    tc = q.dtype == torch.bfloat16 and D == 128
    G = group_size(B, g * T, 128 if tc else 64)
    Bv = B // G
    dev = q.device
    q = q.contiguous()
    # 1. the shared prefix, G sequences per virtual sequence; every prefix token
    #    is visible to every row (global length prefix_len, all of it held here)
    full = torch.full((Bv,), prefix_len, dtype=torch.int32, device=dev)
    bt_pre = block_table[:1, :n_sh].expand(Bv, n_sh).contiguous()
    o1, l1 = decode_attention_shard(q.view(Bv, G * T, Hq, D), k_cache, v_cache, full,
                                    torch.zeros_like(full), full, bt_pre, scale=scale,
                                    max_kv_len=prefix_len)
    # 2. each sequence's own tokens, on its private pages
    bt_suf = block_table[:, n_sh:].contiguous()
    start = torch.full((B,), prefix_len, dtype=torch.int32, device=dev)
    lens = (seq_lens + T - prefix_len).to(torch.int32)
    o2, l2 = decode_attention_shard(q, k_cache, v_cache, seq_lens, start, lens, bt_suf,
                                    scale=scale, max_kv_len=bt_suf.shape[1] * P)
    # 3. merge
    parts_o = torch.stack([o1.view(B, T, Hq, D), o2])
    parts_l = torch.stack([l1.view(B, T, Hq), l2])
    return merge_partials(parts_o, parts_l, out=out, out_dtype=out_dtype or q.dtype)
