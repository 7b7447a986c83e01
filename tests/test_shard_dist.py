"""Host side of the sequence-sharded decode on two gloo ranks (CPU): the shard
bounds and the all-gather of the per-rank partials, with the oracle providing
each rank's shard attention and the merge."""
import math
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from kv_cache_decode_rope_b200.sharding import gather_partials, shard_bounds


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, result):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r = np.random.default_rng(5)
        B, T, Hq, Hkv, D, C = 3, 2, 4, 2, 16, 40
        L = np.array([10, 45, 70])
        q = r.standard_normal((B, T, Hq, D))
        k = r.standard_normal((B, Hkv, C * world, D))
        v = r.standard_normal((B, Hkv, C * world, D))
        sc = 1 / math.sqrt(D)
        start, lens = shard_bounds(torch.tensor(L, dtype=torch.int32), T, rank, C)
        assert int(start[0]) == rank * C
        assert np.array_equal(lens.numpy(), np.clip(L + T - rank * C, 0, C))
        o, lse = oracle.decode_attention_shard(q, k[:, :, rank * C:(rank + 1) * C],
                                               v[:, :, rank * C:(rank + 1) * C], L,
                                               start.numpy(), lens.numpy(), sc)
        o_all, l_all = gather_partials(torch.from_numpy(o), torch.from_numpy(lse))
        got = oracle.merge_partials(o_all.numpy(), l_all.numpy())
        ref = oracle.decode_attention(q, k, v, L, sc)
        result[rank] = float(np.max(np.abs(got - ref)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_gather_and_merge():
    world = 2
    ctx = mp.get_context("spawn")
    result = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, result)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert len(result) == world
    assert max(result.values()) <= 1e-12
