"""decode_attention_static: the decode entry point for callers that cannot
allocate device memory (a host framework that owns all device memory, a
latency-critical path where an allocation would synchronise the device, a
foreign-function caller without a device allocator).  It keeps its split
scratch in an array inside the library instead of a caller workspace.

Checked through the C ABI against the workspace entry points, bit for bit, on
two calls in a row with different inputs (the shared array keeps the first
call's contents, which must not leak into the second), against the fp64 oracle,
and for not allocating: the second call leaves the device's free memory as it
was.  This file is collected last
so that a stop at the first failure has already run every other test."""
import ctypes

import pytest
import torch

import kv_cache_decode_rope_b200 as kvd
import oracle
from kv_cache_decode_rope_b200 import _lib
from kv_cache_decode_rope_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

TOL = 2e-3   # the bf16-input tolerance the parity tests use (fp32 output vs the fp64 oracle)

CASES = {
    "contiguous": WORKLOADS["batched_gqa"].with_(batch=4, cache_len=3000),
    "paged": WORKLOADS["paged_cb"].with_(batch=6, len_range=(1, 5000)),
    "rows64_paged": WORKLOADS["mtp_verify"].with_(batch=2, cache_len=2000),
}


def _device(inp):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}


def _params(w, d, mkl):
    bt = d["block_table"]
    if bt is None:
        paging = dict(max_seq_len=d["k_cache"].shape[2])
    else:
        paging = dict(page_size=d["k_cache"].shape[2], num_pages=d["k_cache"].shape[0],
                      max_pages_per_seq=bt.shape[1])
    return kvd.make_params(batch=w.batch, num_heads=w.num_heads, num_kv_heads=w.num_kv_heads,
                           head_dim=w.head_dim, q_len=w.q_len, dtype=w.torch_dtype, scale=w.scale,
                           out_dtype=torch.float32, max_kv_len=mkl, **paging)


def oracle_step_no_append(host):
    """The oracle's decode of the cache as drawn (no append: the static call
    attends the cache it is given)."""
    w = host["workload"]
    f64 = lambda t: t.float().numpy().astype("float64")  # noqa: E731
    bt = None if host["block_table"] is None else host["block_table"].numpy()
    q = f64(host["q"])
    kc, vc = f64(host["k_cache"]), f64(host["v_cache"])
    return q, kc, vc, oracle.decode_attention(q, kc, vc, host["seq_lens"].numpy(), w.scale, bt)


def _call_static(p, d, out):
    lib = _lib.get_lib()
    bt = d["block_table"]
    return lib.decode_attention_static(ctypes.byref(p), d["q"].data_ptr(), d["k_cache"].data_ptr(),
                                       d["v_cache"].data_ptr(), d["seq_lens"].data_ptr(),
                                       None if bt is None else bt.data_ptr(), out.data_ptr(),
                                       torch.cuda.current_stream().cuda_stream)


def _workspace_call(w, d, mkl):
    if d["block_table"] is None:
        return kvd.decode_attention(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], scale=w.scale,
                                    max_kv_len=mkl, out_dtype=torch.float32)
    return kvd.decode_attention_paged(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"],
                                      d["block_table"], scale=w.scale, max_kv_len=mkl,
                                      out_dtype=torch.float32)


@pytest.mark.parametrize("name", sorted(CASES))
def test_static_scratch_matches_workspace_entry_point(name):
    """Two static calls in a row, on different inputs, each bit for bit equal
    to the workspace entry point: the same kernels with the same grid and the
    same arithmetic per partial slot, so any difference would be stale or
    misplaced scratch.  The second call is also checked against the fp64
    oracle, and it must leave the device's free memory and torch's
    allocations unchanged (it allocates nothing)."""
    w = CASES[name]
    runs = []
    for seed in (31, 32):   # two different inputs for the two calls in a row
        host = make_inputs(w, seed=seed, fill="zero")
        d = _device(host)
        mkl = int(d["seq_lens"].max()) + w.q_len
        ref = _workspace_call(w, d, mkl)
        runs.append((host, d, ref, _params(w, d, mkl), torch.full_like(ref, float("nan"))))
    torch.cuda.synchronize()
    # first static call: resolves the array's address (once per device)
    _, d0, _, p0, out0 = runs[0]
    assert _call_static(p0, d0, out0) == _lib.KVD_OK
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    _, d1, _, p1, out1 = runs[1]
    assert _call_static(p1, d1, out1) == _lib.KVD_OK
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, f"a static call changed free device memory by {free0 - free1} bytes"
    assert torch.cuda.memory_allocated() == alloc0
    for _, _, ref, _, out in runs:
        assert torch.isfinite(out).all()
        assert torch.equal(out, ref)
    host, _, _, _, out = runs[1]
    _, _, _, ref64 = oracle_step_no_append(host)
    err = oracle.max_abs_diff(out.cpu().double().numpy(), ref64)
    assert err <= TOL, f"{name}: max abs diff vs the oracle {err:.3e}"


def test_static_scratch_rejects_oversized_problems():
    """A problem whose partials exceed the array is refused before any launch.
    The tensors are real and sized for the declared shape, so the call would be
    safe even if it were (wrongly) launched."""
    w = WORKLOADS["mtp_verify"].with_(batch=4096, num_heads=64, num_kv_heads=8, q_len=1)
    q = torch.zeros((w.batch, 1, w.num_heads, w.head_dim), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((w.batch, w.num_kv_heads, 16, w.head_dim), dtype=torch.bfloat16, device="cuda")
    seq = torch.zeros(w.batch, dtype=torch.int32, device="cuda")
    out = torch.zeros((w.batch, 1, w.num_heads, w.head_dim), dtype=torch.float32, device="cuda")
    d = {"q": q, "k_cache": kc, "v_cache": kc, "seq_lens": seq, "block_table": None}
    p = _params(w, d, 1)
    assert _call_static(p, d, out) == _lib.KVD_ERR_WORKSPACE
    assert torch.count_nonzero(out).item() == 0
