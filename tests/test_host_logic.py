"""Host-side logic that needs no GPU: the sharded bounds, the cascade group
size, the seeded page tables and byte counts of the workloads, and the lookup
of committed ncu traffic."""
import json

import pytest
import torch

from kv_cache_decode_rope_b200 import prefix
from kv_cache_decode_rope_b200.sharding import shard_bounds
from kv_cache_decode_rope_b200.workloads import WORKLOADS, draw_lengths, page_table, step_bytes


@pytest.mark.parametrize("world,capacity", [(1, 64), (2, 40), (4, 16)])
def test_shard_bounds_cover_every_position_once(world, capacity):
    q_len = 3
    seq_lens = torch.tensor([0, 1, 15, 16, 17, 33, world * capacity - q_len], dtype=torch.int32)
    held = torch.zeros(len(seq_lens), dtype=torch.int64)
    for r in range(world):
        start, lens = shard_bounds(seq_lens, q_len, r, capacity)
        assert start.dtype == torch.int32 and lens.dtype == torch.int32
        assert torch.all(start == r * capacity)
        assert torch.all((lens >= 0) & (lens <= capacity))
        # rank r holds a prefix of its range: positions start .. start + lens - 1
        for b in range(len(seq_lens)):
            n = int(seq_lens[b]) + q_len
            assert int(lens[b]) == max(0, min(capacity, n - r * capacity))
        held += lens.to(torch.int64)
    assert torch.equal(held, seq_lens.to(torch.int64) + q_len)


@pytest.mark.parametrize("batch,rows,cap,expect", [(64, 8, 128, 16), (64, 8, 64, 8), (6, 24, 128, 3),
                                                   (7, 8, 128, 7), (5, 200, 128, 1)])
def test_cascade_group_size(batch, rows, cap, expect):
    G = prefix.group_size(batch, rows, cap)
    assert G == expect
    assert batch % G == 0 and (G == 1 or G * rows <= cap)


def test_page_table_shares_the_prefix_pages_only():
    w = WORKLOADS["shared_prefix"].with_(batch=6, len_range=(1, 300), shared_prefix=64)
    gen = torch.Generator().manual_seed(3)
    lens = draw_lengths(w, gen)
    bt, num_pages = page_table(w, lens, gen)
    P, T = w.page_size, w.q_len
    n_sh = w.shared_prefix // P
    assert torch.all(lens >= w.shared_prefix)
    assert torch.all(bt[:, :n_sh] == bt[0, :n_sh])
    own = set()
    for b, L in enumerate(lens.tolist()):
        n = (L + T + P - 1) // P
        pages = bt[b, :n].tolist()
        assert all(0 <= p < num_pages for p in pages)
        assert torch.all(bt[b, n:] == -1)
        private = pages[n_sh:]
        assert not own & set(private), "private pages must not be shared"
        own |= set(private)
    assert not own & set(bt[0, :n_sh].tolist())
    assert len(own) + n_sh == num_pages


def test_page_table_without_prefix_is_a_permutation():
    w = WORKLOADS["paged_cb"].with_(batch=9, len_range=(1, 200))
    gen = torch.Generator().manual_seed(4)
    lens = draw_lengths(w, gen)
    bt, num_pages = page_table(w, lens, gen)
    used = [p for p in bt.flatten().tolist() if p >= 0]
    assert sorted(used) == list(range(num_pages))


def test_step_bytes_count_each_stored_row_once():
    w = WORKLOADS["batched_gqa"].with_(batch=3, cache_len=100)
    lens = [100, 100, 100]
    d = step_bytes(w, lens, out_esize=2)
    D, es, Hkv, Hq, T = w.head_dim, w.esize, w.num_kv_heads, w.num_heads, w.q_len
    kv = sum(L + T for L in lens) * Hkv * 2 * D * es
    assert d["kv"] == d["kv_logical"] == kv
    assert d["decode"] == kv + 3 * T * Hq * D * es + 3 * T * Hq * D * 2 + 3 * 4
    # a shared prefix is read from HBM once, however many sequences attend it
    ws = WORKLOADS["shared_prefix"].with_(batch=4, len_range=(1, 50), shared_prefix=64)
    lens = [64 + 10, 64 + 20, 64 + 30, 64 + 40]
    ds = step_bytes(ws, lens, out_esize=2)
    row = ws.num_kv_heads * 2 * ws.head_dim * ws.esize
    assert ds["kv_logical"] - ds["kv"] == 3 * 64 * row


def test_committed_traffic_only_for_matching_sources(tmp_path, monkeypatch):
    import bench
    entry = {"kernel": "k", "source_hash": "abc", "traffic_bytes_per_launch": 123}
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "ncu_traffic.json").write_text(json.dumps({"batched_gqa": entry}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "abc")
    assert bench.committed_traffic("batched_gqa") == 123
    assert bench.committed_traffic("mtp_verify") is None
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "changed")
    assert bench.committed_traffic("batched_gqa") is None
