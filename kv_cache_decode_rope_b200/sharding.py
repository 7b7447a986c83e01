"""Sequence-sharded (context-parallel) decode across devices.

Every rank holds one contiguous range of positions of every sequence's cache:
rank r holds global positions [r C, (r + 1) C) as its local tokens 0 .. C-1
(C = the per-rank capacity).  A decode step on rank r:

1. `append_rope_shard`: rotate q and k at the global positions; store k, v of
   the new tokens where rank r holds them (a rank that holds none of a
   sequence's new tokens only rotates q);
2. `decode_attention_shard`: attention of the new tokens over rank r's tokens,
   as (o, log2-sum-exp) per query row;
3. all-gather of (o, lse) over the ranks (NCCL over NVLink in a multi-GPU job;
   B T Hq (D + 1) fp32 per rank, 66 KB for four sequences of 32 heads);
4. `merge_partials`: the log-sum-exp merge ("Flash Decoding: split-K", the
   ferrum-sampler 0.7.0 README, Key Optimizations) gives every rank the output.

The exchanged tensors land in each rank's own memory before the merge reads
them; nothing reads another device's memory directly.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch
import torch.distributed as dist

from . import append_rope_shard, decode_attention_shard, merge_partials


def shard_bounds(seq_lens: torch.Tensor, q_len: int, rank: int, capacity: int
                 ) -> Tuple[torch.Tensor, torch.Tensor]:
    """(shard_start, shard_lens) int32 of `rank` for the attention of a step:
    rank r holds positions [r C, (r + 1) C) and, after the step's append, the
    first clamp(seq_lens + q_len - r C, 0, C) of them."""
    start = torch.full_like(seq_lens, rank * capacity, dtype=torch.int32)
    lens = (seq_lens.to(torch.int64) + q_len - rank * capacity).clamp(0, capacity).to(torch.int32)
    return start, lens


def gather_partials(o: torch.Tensor, lse: torch.Tensor, group=None
                    ) -> Tuple[torch.Tensor, torch.Tensor]:
    """All-gather every rank's (o, lse) into [world, ...] stacks (rank order)."""
    world = dist.get_world_size(group)
    # the concatenated form [world * B, ...] is the one every backend accepts
    o_all = torch.empty((world * o.shape[0],) + tuple(o.shape[1:]), dtype=o.dtype, device=o.device)
    l_all = torch.empty((world * lse.shape[0],) + tuple(lse.shape[1:]), dtype=lse.dtype,
                        device=lse.device)
    dist.all_gather_into_tensor(o_all, o.contiguous(), group=group)
    dist.all_gather_into_tensor(l_all, lse.contiguous(), group=group)
    return o_all.view((world,) + tuple(o.shape)), l_all.view((world,) + tuple(lse.shape))


def sharded_decode_step(q, k_new, v_new, k_cache, v_cache, seq_lens, *, rank: int, world: int,
                        capacity: int, block_table=None, scale: Optional[float] = None,
                        rope_base: float = 10000.0, out_dtype=None, group=None, workspace=None):
    """One decode step of a sequence-sharded cache on this rank (steps 1-4
    above).  ``k_cache``/``v_cache`` are this rank's local caches of
    ``capacity`` positions per sequence; ``seq_lens`` is the global length
    before the step (not advanced).  Returns the merged output on every rank."""
    T = q.shape[1]
    start, lens = shard_bounds(seq_lens, T, rank, capacity)
    append_rope_shard(q, k_new, v_new, k_cache, v_cache, seq_lens, start, block_table,
                      rope_base=rope_base)
    o, lse = decode_attention_shard(q, k_cache, v_cache, seq_lens, start, lens, block_table,
                                    scale=scale, max_kv_len=capacity, workspace=workspace)
    if world == 1:
        return merge_partials(o[None], lse[None], out_dtype=out_dtype or q.dtype)
    o_all, l_all = gather_partials(o, lse, group)
    return merge_partials(o_all, l_all, out_dtype=out_dtype or q.dtype)
