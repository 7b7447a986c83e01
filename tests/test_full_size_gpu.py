"""The five workloads at full size, in the launch configuration the bench
times: sampled rows against the oracle row by row, and a property every
output row must satisfy (a softmax average lies inside the per-dimension
range of the values it averages)."""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_decode_rope_b200.workloads import WORKLOADS, make_inputs
from tests.gpu_util import gpu_step, log_error, np64, oracle_rows, tol_for

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

NAMES = ["tiny_mha", "batched_gqa", "paged_cb", "mtp_verify", "long_ctx"]


def _samples(w, inp, n, seed):
    rng = np.random.default_rng(seed)
    n = min(n, w.batch * w.q_len * w.num_heads)
    picks = {(0, 0, 0), (w.batch - 1, w.q_len - 1, w.num_heads - 1)}
    if w.cache_len is None:   # ragged: include the longest and the shortest sequence
        picks.add((int(inp["seq_lens"].argmax()), 0, 0))
        picks.add((int(inp["seq_lens"].argmin()), 0, w.num_heads - 1))
    while len(picks) < n:
        picks.add((int(rng.integers(w.batch)), int(rng.integers(w.q_len)), int(rng.integers(w.num_heads))))
    return sorted(picks)


def _value_range(inp, d):
    """Per (b, q-head, dim) min and max over the visible V rows, on the GPU
    (test-side check; includes the appended token)."""
    w = inp["workload"]
    vc = d["v_cache"]
    lo = torch.empty((w.batch, w.num_kv_heads, w.head_dim), device="cuda")
    hi = torch.empty_like(lo)
    P = w.page_size
    for b in range(w.batch):
        n = int(inp["seq_lens"][b]) + w.q_len
        if d["block_table"] is None:
            rows = vc[b, :, :n].float()
        else:
            t = torch.arange(n, device="cuda")
            rows = vc[d["block_table"][b, t // P].long(), :, t % P].transpose(0, 1).float()
        lo[b] = rows.amin(1)
        hi[b] = rows.amax(1)
    g = w.group
    return lo.repeat_interleave(g, 1)[:, None], hi.repeat_interleave(g, 1)[:, None]


@pytest.mark.parametrize("name", NAMES)
def test_full_size_sampled_parity(name):
    w = WORKLOADS[name]
    if w.cache_mode == "prefill":
        w = w.with_(cache_mode="random")
    inp = make_inputs(w, seed=1000 + w.config_id, fill="zero")
    d, out = gpu_step(inp, out_dtype=torch.float32)
    got = out.cpu()
    assert torch.isfinite(got).all()
    lo, hi = _value_range(inp, d)
    slack = 1e-5
    assert bool((out >= lo - slack).all()) and bool((out <= hi + slack).all())
    samples = _samples(w, inp, 24, seed=w.config_id)
    ref = oracle_rows(inp, samples)
    worst = 0.0
    for (b, i, h), r in ref.items():
        worst = max(worst, oracle.max_abs_diff(np64(got[b, i, h]), r))
    log_error(f"full_size[{name}]", worst)
    assert worst <= tol_for(w), f"{name}: max abs diff {worst:.3e}"
