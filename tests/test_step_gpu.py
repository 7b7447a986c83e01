"""kvd_decode_step against kv_append_rope followed by decode_attention[_paged].

The one-call step must equal the two separate calls bit for bit: output,
rotated q, both caches, every slot.  The caches start NaN-filled, so a slot
read before its append shows up in the output.  The cases span both decode
kernels (CUDA cores, and tensor cores for units of 8 or more bf16 rows at
D = 128), both cache layouts, every head size, the RoPE layouts, an empty
prefix, positions up to 2^17, and consecutive steps across a stage
boundary."""
import numpy as np
import pytest
import torch

import kv_cache_decode_rope_b200 as kvd
import oracle
from kv_cache_decode_rope_b200.workloads import WORKLOADS, make_inputs
from tests.gpu_util import log_error, max_kv_len, np64, oracle_step, to_device, tol_for

pytestmark = pytest.mark.gpu

G, P, M, L = (WORKLOADS[n] for n in ("batched_gqa", "paged_cb", "mtp_verify", "long_ctx"))
T1 = WORKLOADS["tiny_mha"].with_(cache_mode="random")

CASES = {
    # name: (workload, rope layout (interleaved, rotary_dim))
    "gqa_stage_end": (G.with_(batch=3, cache_len=63), (False, 0)),        # new token at 63
    "gqa_split": (G.with_(batch=2, cache_len=1000), (False, 0)),          # units over several CTAs
    "gqa_interleaved_partial": (G.with_(batch=2, cache_len=300), (True, 64)),
    "gqa_half_partial": (G.with_(batch=2, cache_len=130), (False, 32)),
    "g2_q2_paged": (P.with_(batch=5, num_heads=16, len_range=(1, 300), q_len=2), (False, 0)),
    "g1_q4_paged_p32": (P.with_(batch=3, num_heads=8, len_range=(1, 40), q_len=4, page_size=32),
                        (False, 0)),
    "g1_q3_f32": (T1.with_(cache_len=20, q_len=3, num_heads=4, num_kv_heads=4), (False, 0)),
    "empty_prefix_f32": (T1.with_(cache_len=0, q_len=2, num_heads=4, num_kv_heads=2), (False, 0)),
    "d16_f32_paged": (P.with_(batch=3, dtype="f32", head_dim=16, num_heads=4, num_kv_heads=4,
                              len_range=(1, 70), q_len=4), (True, 0)),
    "d32_bf16": (G.with_(batch=2, head_dim=32, num_heads=8, num_kv_heads=2, cache_len=77), (False, 0)),
    "d64_bf16_paged": (P.with_(batch=4, head_dim=64, num_heads=16, len_range=(5, 500)), (False, 16)),
    "d256_bf16": (G.with_(batch=2, head_dim=256, num_heads=8, num_kv_heads=2, cache_len=200),
                  (False, 0)),
    "long_pos": (L.with_(batch=1, num_heads=4, num_kv_heads=1, cache_len=131072, peaked_frac=0.0),
                 (False, 0)),
    # 6 and 8 rows on CUDA cores, 16 rows on tensor cores
    "g6_bf16_two_launch": (G.with_(batch=2, num_heads=12, num_kv_heads=2, cache_len=90), (False, 0)),
    "g8_f32_two_launch": (T1.with_(cache_len=50, num_heads=8, num_kv_heads=1), (False, 0)),
    "mtp_tc_two_launch": (M.with_(batch=2, cache_len=200), (False, 0)),
}


def bits(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    return (t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)).numpy()


def run_two_calls(inp, d, layout, out_dtype):
    w = inp["workload"]
    kvd.append_rope(d["q"], d["k_new"], d["v_new"], d["k_cache"], d["v_cache"], d["seq_lens"],
                    d["block_table"], rope_base=w.rope_base, interleaved=layout[0],
                    rotary_dim=layout[1])
    kw = dict(scale=w.scale, max_kv_len=max_kv_len(inp), out_dtype=out_dtype)
    if d["block_table"] is None:
        return kvd.decode_attention(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], **kw)
    return kvd.decode_attention_paged(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"],
                                      d["block_table"], **kw)


def run_step(inp, d, layout, out_dtype, status=None):
    w = inp["workload"]
    return kvd.decode_step(d["q"], d["k_new"], d["v_new"], d["k_cache"], d["v_cache"], d["seq_lens"],
                           d["block_table"], scale=w.scale, max_kv_len=max_kv_len(inp),
                           out_dtype=out_dtype, rope_base=w.rope_base, interleaved=layout[0],
                           rotary_dim=layout[1], status=status)


@pytest.mark.parametrize("name", sorted(CASES))
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_step_equals_append_then_decode(name, out_dtype):
    w, layout = CASES[name]
    inp = make_inputs(w, seed=11, fill="nan")
    ref_d = to_device(inp)
    ref_out = run_two_calls(inp, ref_d, layout, out_dtype)
    d = to_device(inp)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = run_step(inp, d, layout, out_dtype, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert np.array_equal(bits(out), bits(ref_out)), name
    assert np.array_equal(bits(d["q"]), bits(ref_d["q"])), name
    assert np.array_equal(bits(d["k_cache"]), bits(ref_d["k_cache"])), name
    assert np.array_equal(bits(d["v_cache"]), bits(ref_d["v_cache"])), name
    assert torch.isfinite(out).all()


@pytest.mark.parametrize("name", ["gqa_split", "g2_q2_paged", "g1_q3_f32", "g1_q4_paged_p32"])
def test_step_matches_oracle(name):
    """The one-call step against the fp64 oracle (cases of the half-split,
    full-width rotation that oracle_step applies)."""
    w, layout = CASES[name]
    assert layout == (False, 0)
    inp = make_inputs(w, seed=12, fill="nan")
    d = to_device(inp)
    out = np64(run_step(inp, d, layout, torch.float32))
    torch.cuda.synchronize()
    _, _, _, ref = oracle_step(inp)
    err = oracle.max_abs_diff(out, ref)
    log_error(f"decode_step[{name}]", err)
    assert err <= tol_for(w), err


def test_step_repeated_advances_like_two_calls():
    """Four consecutive steps (seq_lens advanced between them, as a decode
    loop does, over the stage boundary at 64) through both routes stay
    bit-identical."""
    w = G.with_(batch=2, num_heads=8, num_kv_heads=2, cache_len=61)
    inp = make_inputs(w, seed=13, fill="nan")
    for k in ("k_cache", "v_cache"):   # room for the four steps
        c = inp[k]
        inp[k] = torch.cat([c, torch.full_like(c[:, :, :16], float("nan"))], dim=2)
    a, b = to_device(inp), to_device(inp)
    gen = torch.Generator().manual_seed(5)
    for step in range(4):
        new = {k: torch.randn(inp[k].shape, generator=gen).to(inp[k].dtype).cuda()
               for k in ("q", "k_new", "v_new")}
        for dd in (a, b):
            for k, v in new.items():
                dd[k] = v.clone()
        cur = dict(inp)
        cur["seq_lens"] = a["seq_lens"].cpu()
        ref = run_two_calls(cur, a, (False, 0), torch.float32)
        out = run_step(cur, b, (False, 0), torch.float32)
        torch.cuda.synchronize()
        assert np.array_equal(bits(out), bits(ref)), step
        assert np.array_equal(bits(b["k_cache"]), bits(a["k_cache"])), step
        a["seq_lens"] += 1
        b["seq_lens"] += 1
