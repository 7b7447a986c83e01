"""The decode-step driver (per-layer caches, prefill = decode, CUDA-graph
replay) against the oracle's full causal recompute at every step: the check of
ferric-core 0.1.0, examples/generate.rs `run`, made for every step and layer."""
import math

import numpy as np
import pytest
import torch

import kv_cache_decode_rope_b200 as kvd
import oracle
from tests.gpu_util import log_error, np64

pytestmark = pytest.mark.gpu


def _tokens(gen, n_layers, B, N, H, D, dtype):
    return (torch.rand((n_layers, B, N, H, D), generator=gen) * 2 - 1).to(dtype)


@pytest.mark.parametrize("dtype,paged,graphs,layout", [
    (torch.float32, False, True, (False, 0)),
    (torch.bfloat16, True, True, (False, 0)),
    (torch.bfloat16, False, False, (True, 64)),
    (torch.bfloat16, True, True, (True, 0)),
])
def test_decode_loop_matches_full_recompute(dtype, paged, graphs, layout):
    n_layers, B, Hq, Hkv, D = 3, 2, 16, 2, 128      # 8 rows per unit: tensor-core path in bf16
    interleaved, rotary_dim = layout
    steps = [5, 1, 1, 3, 1, 1, 1, 2, 1, 1]             # prompt chunk, decode, a 3-token draft, ...
    N = sum(steps)
    gen = torch.Generator().manual_seed(17)
    q = _tokens(gen, n_layers, B, N, Hq, D, dtype)
    k = _tokens(gen, n_layers, B, N, Hkv, D, dtype)
    v = _tokens(gen, n_layers, B, N, Hkv, D, dtype)
    loop = kvd.DecodeLoop(n_layers=n_layers, batch=B, num_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                          capacity=48, dtype=dtype, out_dtype=torch.float32, paged=paged,
                          interleaved=interleaved, rotary_dim=rotary_dim, graphs=graphs)
    sc = 1 / math.sqrt(D)
    sdt = "f32" if dtype == torch.float32 else "bf16"
    ref = [oracle.full_causal_attention(np64(q[l]), np64(k[l]), np64(v[l]), sc, 10000.0, sdt,
                                        interleaved, rotary_dim) for l in range(n_layers)]
    tol = 1e-5 if dtype == torch.float32 else 2e-3
    pos = 0
    worst = 0.0
    for T in steps:
        sl = slice(pos, pos + T)
        out = loop.step(q[:, :, sl].cuda(), k[:, :, sl].cuda(), v[:, :, sl].cuda())
        got = np64(out)
        for l in range(n_layers):
            worst = max(worst, oracle.max_abs_diff(got[l], ref[l][:, sl]))
        pos += T
    torch.cuda.synchronize()
    assert int(loop.seq_lens[0]) == N
    log_error(f"driver[{sdt},paged={paged},graphs={graphs},layout={layout}]", worst)
    assert worst <= tol, worst


def test_prefill_chunks_long_prompt():
    """A prompt longer than one step may carry (g = 1: 64 rows) goes through
    chunked decode steps and matches the full recompute on every token."""
    n_layers, B, H, D, N = 2, 1, 4, 64, 150
    gen = torch.Generator().manual_seed(23)
    q = _tokens(gen, n_layers, B, N, H, D, torch.float32)
    k = _tokens(gen, n_layers, B, N, H, D, torch.float32)
    v = _tokens(gen, n_layers, B, N, H, D, torch.float32)
    loop = kvd.DecodeLoop(n_layers=n_layers, batch=B, num_heads=H, num_kv_heads=H, head_dim=D,
                          capacity=N + 1, dtype=torch.float32)
    out = np64(loop.prefill(q.cuda(), k.cuda(), v.cuda()))
    sc = 1 / math.sqrt(D)
    for l in range(n_layers):
        ref = oracle.full_causal_attention(np64(q[l]), np64(k[l]), np64(v[l]), sc, 10000.0, "f32")
        assert oracle.max_abs_diff(out[l], ref) <= 1e-5


def test_decode_step_validates_before_launch():
    """A bad decode argument fails the whole step: the append must not run."""
    B, H, D = 1, 4, 64
    q = torch.rand((B, 1, H, D), device="cuda")
    k = torch.rand((B, 1, H, D), device="cuda")
    kc = torch.zeros((B, H, 8, D), device="cuda")
    vc = torch.zeros_like(kc)
    seq = torch.zeros(B, dtype=torch.int32, device="cuda")
    q0 = q.clone()
    with pytest.raises(kvd.KvdError):
        kvd.decode_step(q, k, k.clone(), kc, vc, seq, scale=float("nan"), max_kv_len=1)
    torch.cuda.synchronize()
    assert torch.equal(q, q0) and not kc.any()
