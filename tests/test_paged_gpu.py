"""Paged decode: the same logical cache under any page permutation gives the
same bits, and equals the contiguous layout; device-side checks flag bad
inputs instead of faulting."""
import pytest
import torch

import kv_cache_decode_rope_b200 as kvd
from kv_cache_decode_rope_b200 import _lib
from kv_cache_decode_rope_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


def _contiguous_copy(inp):
    w = inp["workload"]
    seq = inp["seq_lens"]
    cap = int(seq.max()) + w.q_len
    cap = (cap + 15) // 16 * 16
    kc = torch.zeros((w.batch, w.num_kv_heads, cap, w.head_dim), dtype=w.torch_dtype)
    vc = torch.zeros_like(kc)
    P = w.page_size
    for b in range(w.batch):
        n = int(seq[b]) + w.q_len
        t = torch.arange(n)
        pages = inp["block_table"][b, t // P].long()
        kc[b, :, :n] = inp["k_cache"][pages, :, t % P].transpose(0, 1)
        vc[b, :, :n] = inp["v_cache"][pages, :, t % P].transpose(0, 1)
    return kc, vc


def _permuted(inp, seed):
    """Same logical cache, pages moved to a new random permutation of the pool."""
    gen = torch.Generator().manual_seed(seed)
    n = inp["k_cache"].shape[0]
    perm = torch.randperm(n, generator=gen)       # new physical id of old page j = perm[j]
    kc = torch.empty_like(inp["k_cache"])
    vc = torch.empty_like(inp["v_cache"])
    kc[perm] = inp["k_cache"]
    vc[perm] = inp["v_cache"]
    bt = inp["block_table"].clone()
    valid = bt >= 0
    bt[valid] = perm[bt[valid].long()].to(torch.int32)
    return kc, vc, bt


@pytest.mark.parametrize("wname,kw", [
    ("paged_cb", dict(batch=7, len_range=(1, 2500))),
    ("mtp_verify", dict(batch=3, cache_len=900)),
    ("paged_cb", dict(batch=4, len_range=(16, 600), page_size=32)),
])
def test_page_permutation_invariance_and_contiguous_equality(wname, kw):
    w = WORKLOADS[wname].with_(**kw)
    inp = make_inputs(w, seed=21, fill="zero")
    # the new tokens' pages must exist: append first on the paged layout
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    kvd.append_rope(d["q"], d["k_new"], d["v_new"], d["k_cache"], d["v_cache"], d["seq_lens"],
                    d["block_table"], rope_base=w.rope_base)
    torch.cuda.synchronize()
    host = dict(inp, q=d["q"].cpu(), k_cache=d["k_cache"].cpu(), v_cache=d["v_cache"].cpu())
    mkl = int(inp["seq_lens"].max()) + w.q_len
    args = dict(scale=w.scale, max_kv_len=mkl, out_dtype=torch.float32)
    base = kvd.decode_attention_paged(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"],
                                      d["block_table"], **args)
    for s in (1, 2):
        kc, vc, bt = _permuted(host, s)
        o = kvd.decode_attention_paged(d["q"], kc.cuda(), vc.cuda(), d["seq_lens"], bt.cuda(), **args)
        assert torch.equal(o, base)
    kc, vc = _contiguous_copy(host)
    oc = kvd.decode_attention(d["q"], kc.cuda(), vc.cuda(), d["seq_lens"], **args)
    assert torch.equal(oc, base)


def test_out_of_range_page_is_flagged_not_faulted():
    w = WORKLOADS["paged_cb"].with_(batch=3, len_range=(40, 200))
    inp = make_inputs(w, seed=2, fill="zero")
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    bt = d["block_table"].clone()
    bt[1, 1] = inp["num_pages"] + 5          # points past the pool: must be skipped
    kvd.decode_attention_paged(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], bt, scale=w.scale,
                               max_kv_len=int(inp["seq_lens"].max()) + 1, status=status)
    torch.cuda.synchronize()
    assert status.item() & _lib.KVD_FLAG_PAGE_OUT_OF_RANGE
    # the other sequences are unaffected
    status.zero_()
    good = kvd.decode_attention_paged(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"],
                                      d["block_table"], scale=w.scale,
                                      max_kv_len=int(inp["seq_lens"].max()) + 1, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0


def test_capacity_overflow_is_flagged_not_faulted():
    w = WORKLOADS["batched_gqa"].with_(batch=2, cache_len=40)
    inp = make_inputs(w, seed=3, fill="zero")
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    cap = d["k_cache"].shape[2]
    seq = torch.tensor([cap, 5], dtype=torch.int32, device="cuda")   # sequence 0 has no room left
    kvd.append_rope(d["q"], d["k_new"], d["v_new"], d["k_cache"], d["v_cache"], seq, status=status)
    torch.cuda.synchronize()
    assert status.item() & _lib.KVD_FLAG_CAPACITY
    status.zero_()
    kvd.decode_attention(d["q"], d["k_cache"], d["v_cache"], seq, scale=w.scale, max_kv_len=cap,
                         status=status)
    torch.cuda.synchronize()
    assert status.item() & _lib.KVD_FLAG_CAPACITY
