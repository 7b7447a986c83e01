"""decode_attention[_paged] on the GPU against the fp64 oracle, element by
element, over shapes that span several stages, CTAs and a ragged tail."""
import math

import numpy as np
import pytest
import torch

import kv_cache_decode_rope_b200 as kvd
import oracle
from kv_cache_decode_rope_b200.workloads import WORKLOADS, make_inputs
from tests.gpu_util import (gpu_append, gpu_decode, gpu_step, log_error, np64, oracle_step,
                            to_device, tol_for)

# fp32 error allowed on top of one bf16 ulp when comparing a bf16 output: the
# CUDA-core path accumulates in fp32 (errors ~1e-7 to 6e-6); the tensor-core
# path (g * q_len >= 8, bf16, D = 128) feeds each probability to the MMA as a
# bf16 high part plus the remainder rounded to bf16 (relative error at most
# 2^-15 per weight) and accumulates in fp32 TMEM: measured at most 1.45e-5
# against the fp64 oracle on these shapes, so 5e-5 leaves a 3x margin.
F32_ABS_CORE = 1e-5
F32_ABS_TC = 5e-5


def f32_allowance(w):
    tc = w.dtype == "bf16" and w.head_dim == 128 and w.rows >= 8
    return F32_ABS_TC if tc else F32_ABS_CORE

pytestmark = pytest.mark.gpu

SHAPES = {
    # name: workload (reduced sizes of the five workloads, plus other geometries)
    "tiny_mha_rand": WORKLOADS["tiny_mha"].with_(cache_mode="random"),
    "gqa": WORKLOADS["batched_gqa"].with_(batch=3, cache_len=1000),
    "paged_cb": WORKLOADS["paged_cb"].with_(batch=6, len_range=(1, 3000)),
    "mtp": WORKLOADS["mtp_verify"].with_(batch=2, cache_len=700),
    "long_peaked": WORKLOADS["long_ctx"].with_(batch=1, num_heads=8, num_kv_heads=2, cache_len=20000),
    "g1_bf16": WORKLOADS["batched_gqa"].with_(batch=2, num_heads=4, num_kv_heads=4, cache_len=333),
    "g2_q2": WORKLOADS["batched_gqa"].with_(batch=2, num_heads=8, num_kv_heads=4, cache_len=129, q_len=2),
    "g16_q1_paged": WORKLOADS["mtp_verify"].with_(batch=3, q_len=1, cache_len=515),
    "g8_q2_rows16": WORKLOADS["batched_gqa"].with_(batch=2, num_heads=16, num_kv_heads=2, cache_len=260,
                                                    q_len=2),
    "g3_rows3": WORKLOADS["batched_gqa"].with_(batch=2, num_heads=6, num_kv_heads=2, cache_len=90),
    "d64_bf16": WORKLOADS["batched_gqa"].with_(batch=2, head_dim=64, cache_len=500),
    "d256_bf16": WORKLOADS["batched_gqa"].with_(batch=2, head_dim=256, cache_len=300),
    "d32_bf16_paged": WORKLOADS["paged_cb"].with_(batch=3, head_dim=32, len_range=(2, 700)),
    "d16_bf16": WORKLOADS["batched_gqa"].with_(batch=2, head_dim=16, num_heads=4, num_kv_heads=2,
                                                cache_len=77, q_len=3),
    "f32_d128": WORKLOADS["batched_gqa"].with_(batch=2, dtype="f32", cache_len=400),
    "f32_d16_ferric": WORKLOADS["tiny_mha"].with_(cache_mode="random", num_heads=4, num_kv_heads=4,
                                                   head_dim=16, cache_len=8),
    "f32_d32_paged_q4": WORKLOADS["paged_cb"].with_(batch=2, dtype="f32", head_dim=32, num_heads=8,
                                                    num_kv_heads=2, len_range=(1, 150), q_len=4),
    "short_lens": WORKLOADS["paged_cb"].with_(batch=9, len_range=(1, 20)),
    "tc_rows128": WORKLOADS["batched_gqa"].with_(batch=2, num_heads=64, num_kv_heads=2, q_len=4,
                                                  cache_len=300),
    "tc_rows18_paged": WORKLOADS["paged_cb"].with_(batch=3, num_heads=12, num_kv_heads=2, q_len=3,
                                                   len_range=(1, 900)),
    "shared_prefix": WORKLOADS["shared_prefix"].with_(batch=6, len_range=(1, 300), shared_prefix=512),
}


@pytest.mark.parametrize("name", sorted(SHAPES))
@pytest.mark.parametrize("seed", [0, 1])
def test_step_matches_oracle(name, seed):
    w = SHAPES[name]
    inp = make_inputs(w, seed=seed, fill="nan")
    _, out = gpu_step(inp, out_dtype=torch.float32)
    _, _, _, ref = oracle_step(inp)
    got = np64(out)
    assert np.isfinite(got).all()
    err = oracle.max_abs_diff(got, ref)
    log_error(f"f32_out[{name}][seed{seed}]", err)
    assert err <= tol_for(w), f"{name}: max abs diff {err:.3e}"


@pytest.mark.parametrize("name", ["gqa", "paged_cb", "mtp", "f32_d128"])
def test_bf16_output_within_one_ulp(name):
    w = SHAPES[name]
    inp = make_inputs(w, seed=2, fill="nan")
    _, out = gpu_step(inp, out_dtype=torch.bfloat16)
    _, _, _, ref = oracle_step(inp)
    got = np64(out)
    ref_b = oracle.bf16_round(ref)
    # bf16(o32) vs bf16(o_exact): at most one bf16 ulp apart when |o32 - o| is
    # below half an ulp; near zero the ulp shrinks below the fp32 accumulation
    # error, so that error (F32_ABS) is allowed on top.
    e = np.floor(np.log2(np.maximum(np.abs(ref_b), 1e-30)))
    err = np.abs(got - ref_b) - np.exp2(e - 7)
    log_error(f"bf16_out[{name}]", float(np.max(np.abs(got - ref_b))))
    assert np.all(err <= f32_allowance(w)), float(err.max())


def test_tiny_mha_prefill_then_decode_equals_full_recompute():
    """The tiny workload as the pages run it: the 128-token prefix goes in
    through the append (prefill = decode), then one step at position 128; the
    result must equal the last row of a full causal recompute (fp32: 1e-5)."""
    w = WORKLOADS["tiny_mha"]
    inp = make_inputs(w, seed=1001, fill="nan")
    L = w.cache_len
    d = to_device(inp)
    zero = torch.zeros(w.batch, dtype=torch.int32, device="cuda")
    qp = inp["q_prefix"].cuda()
    kvd.append_rope(qp, inp["k_prefix"].cuda(), inp["v_prefix"].cuda(), d["k_cache"], d["v_cache"], zero,
                    rope_base=w.rope_base)
    kvd.append_rope(d["q"], d["k_new"], d["v_new"], d["k_cache"], d["v_cache"], d["seq_lens"],
                    rope_base=w.rope_base)
    out = kvd.decode_attention(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], scale=w.scale,
                               max_kv_len=L + 1, out_dtype=torch.float32)
    torch.cuda.synchronize()
    q_all = np.concatenate([np64(inp["q_prefix"]), np64(inp["q"])], 1)
    k_all = np.concatenate([np64(inp["k_prefix"]), np64(inp["k_new"])], 1)
    v_all = np.concatenate([np64(inp["v_prefix"]), np64(inp["v_new"])], 1)
    ref = oracle.full_causal_attention(q_all, k_all, v_all, w.scale, w.rope_base, "f32")[:, -1:]
    assert oracle.max_abs_diff(np64(out), ref) <= 1e-5


def test_ferric_example_steps():
    """The worked example's shape (4 heads, head dim 16, base 10000): the
    prompt's 4 tokens are fed one per step, then 5 more steps; every step's
    output equals the full causal recompute of its prefix."""
    import json, os
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "ferric_example.json")))
    H, D, base = g["num_heads"], g["head_dim"], g["rope_base"]
    N = g["prompt_len"] + g["gen_steps"]
    gen = torch.Generator().manual_seed(7)
    q = torch.rand((1, N, H, D), generator=gen) * 0.2 - 0.1
    k = torch.rand((1, N, H, D), generator=gen) * 0.2 - 0.1
    v = torch.rand((1, N, H, D), generator=gen) * 0.2 - 0.1
    kc = torch.full((1, H, 16, D), float("nan"), device="cuda")
    vc = torch.full_like(kc, float("nan"))
    scale = 1 / math.sqrt(D)
    ref = oracle.full_causal_attention(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                       scale, base, "f32")
    worst = 0.0
    for pos in range(N):
        qs = q[:, pos:pos + 1].cuda().contiguous()
        sl = torch.tensor([pos], dtype=torch.int32, device="cuda")
        kvd.append_rope(qs, k[:, pos:pos + 1].cuda().contiguous(), v[:, pos:pos + 1].cuda().contiguous(),
                        kc, vc, sl, rope_base=base)
        out = kvd.decode_attention(qs, kc, vc, sl, scale=scale, max_kv_len=pos + 1, out_dtype=torch.float32)
        torch.cuda.synchronize()
        worst = max(worst, oracle.max_abs_diff(np64(out)[0, 0], ref[0, pos]))
    assert worst < g["tolerance_max_abs"]
    assert worst <= 1e-6


# ---------------------------------------------------------------- special cases
def _decode_only(q, kc, vc, seq, scale, out_dtype=torch.float32, q_len=1):
    return kvd.decode_attention(q.cuda(), kc.cuda(), vc.cuda(), seq.cuda(), scale=scale,
                                max_kv_len=int(seq.max()) + q_len, out_dtype=out_dtype)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_length_one_cache_returns_v(dtype):
    w = WORKLOADS["batched_gqa"].with_(batch=4, cache_len=0, dtype="bf16" if dtype == torch.bfloat16 else "f32")
    inp = make_inputs(w, seed=11)
    for od in (torch.float32, dtype):
        _, out = gpu_step(inp, out_dtype=od)
        v = inp["v_new"].to(od)        # [B, 1, Hkv, D]
        exp = v.repeat_interleave(w.group, dim=2)
        assert torch.equal(out.cpu(), exp)


# (num_heads, num_kv_heads): 4 rows per unit (CUDA-core kernel), 8 and 16 rows
# (64-row tensor-core tile), 128 rows (128-row tensor-core tile)
GEOMS = [(8, 2), (16, 2), (32, 2), (128, 1)]


@pytest.mark.parametrize("Hq,Hkv", GEOMS)
def test_identical_keys_give_mean_of_v(Hq, Hkv):
    B, D, L = 2, 128, 777
    gen = torch.Generator().manual_seed(3)
    q = torch.randn((B, 1, Hq, D), generator=gen).bfloat16()
    key = torch.randn(D, generator=gen).bfloat16()
    kc = key.expand(B, Hkv, L + 1, D).contiguous()
    vc = torch.randn((B, Hkv, L + 1, D), generator=gen).bfloat16()
    seq = torch.full((B,), L, dtype=torch.int32)
    out = _decode_only(q, kc, vc, seq, 0.3)
    mean = vc.double().mean(dim=2)                          # [B, Hkv, D]
    exp = mean.repeat_interleave(Hq // Hkv, dim=1)[:, None]
    assert (out.cpu().double() - exp).abs().max().item() <= 2e-6


@pytest.mark.parametrize("Hq,Hkv", GEOMS)
def test_dominant_key_returns_its_v_row(Hq, Hkv):
    B, D, L = 2, 128, 3000
    g = Hq // Hkv
    gen = torch.Generator().manual_seed(4)
    q = torch.randn((B, 1, Hq, D), generator=gen).bfloat16()
    kc = (torch.randn((B, Hkv, L + 1, D), generator=gen) * 0.01).bfloat16()
    vc = torch.randn((B, Hkv, L + 1, D), generator=gen).bfloat16()
    star = [123, 2900]
    for b in range(B):
        for hk in range(Hkv):
            # all q heads of the group point the same way: one key dominates every one of them
            q[b, 0, hk * g:(hk + 1) * g] = q[b, 0, hk * g]
            kc[b, hk, star[b]] = (q[b, 0, hk * g].float() * 4.0).bfloat16()
    seq = torch.full((B,), L, dtype=torch.int32)
    scale = 1 / math.sqrt(D)
    # margin: scale * 4 |q|^2 ~ 45 natural units vs others ~0.01 scale -> weight ratio e^-45
    s_star = scale * 4.0 * (q[:, 0].float() ** 2).sum(-1)
    assert s_star.min().item() > 30
    for od in (torch.float32, torch.bfloat16):
        out = _decode_only(q, kc, vc, seq, scale * 3.0, out_dtype=od)   # margin > 100
        for b in range(B):
            exp = vc[b, :, star[b]].to(od).repeat_interleave(g, dim=0)
            got = out[b, 0].cpu()
            if g >= 8 and od == torch.float32:
                # tensor-core path: the dominant weight reaches the MMA as a bf16
                # high part plus a bf16 residual, within 2^-16 of itself
                assert ((got - exp).abs() <= 2.0 ** -14 * exp.abs()).all()
            else:
                assert torch.equal(got, exp)


def test_empty_batch_is_noop():
    q = torch.empty((0, 1, 8, 128), dtype=torch.bfloat16, device="cuda")
    kc = torch.empty((0, 2, 16, 128), dtype=torch.bfloat16, device="cuda")
    seq = torch.empty((0,), dtype=torch.int32, device="cuda")
    kvd.append_rope(q, torch.empty((0, 1, 2, 128), dtype=torch.bfloat16, device="cuda"),
                    torch.empty((0, 1, 2, 128), dtype=torch.bfloat16, device="cuda"), kc, kc.clone(), seq)
    out = kvd.decode_attention(q, kc, kc.clone(), seq, scale=0.1, max_kv_len=1)
    assert out.shape == (0, 1, 8, 128)


@pytest.mark.parametrize("Hq,Hkv", GEOMS)
def test_scale_zero_is_uniform_average(Hq, Hkv):
    """scale = 0 makes every visible key equally likely: out = mean of V."""
    w = WORKLOADS["batched_gqa"].with_(batch=2, cache_len=500, num_heads=Hq, num_kv_heads=Hkv)
    inp = make_inputs(w, seed=8, fill="zero")
    d = to_device(inp)
    out = kvd.decode_attention(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], scale=0.0,
                               max_kv_len=501, out_dtype=torch.float32)
    exp = inp["v_cache"][:, :, :501].double().mean(2).repeat_interleave(w.group, 1)[:, None]
    assert (out.cpu().double() - exp).abs().max().item() <= 2e-6


@pytest.mark.parametrize("Hq,Hkv,q_len", [(8, 2, 1), (16, 2, 2), (64, 1, 2)])
def test_negative_scale_matches_oracle(Hq, Hkv, q_len):
    """A negative scale is a valid softmax temperature: the step still matches
    the oracle (the kernels may not assume scale > 0 when they track the
    running maximum)."""
    w = WORKLOADS["batched_gqa"].with_(batch=2, cache_len=300, num_heads=Hq, num_kv_heads=Hkv,
                                       q_len=q_len)
    inp = make_inputs(w, seed=21, fill="nan")
    d = to_device(inp)
    gpu_append(inp, d)
    out = kvd.decode_attention(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], scale=-w.scale,
                               max_kv_len=int(inp["seq_lens"].max()) + q_len, out_dtype=torch.float32)
    q_rot, kc, vc = oracle.append_rope(np64(inp["q"]), np64(inp["k_new"]), np64(inp["v_new"]),
                                       np64(inp["k_cache"]), np64(inp["v_cache"]),
                                       inp["seq_lens"].numpy(), w.rope_base, w.dtype)
    ref = oracle.decode_attention(q_rot, kc, vc, inp["seq_lens"].numpy(), -w.scale)
    err = oracle.max_abs_diff(np64(out), ref)
    log_error(f"neg_scale[{Hq},{Hkv},{q_len}]", err)
    assert err < tol_for(w)


def test_repeated_calls_are_deterministic():
    w = SHAPES["paged_cb"]
    inp = make_inputs(w, seed=4, fill="zero")
    d = to_device(inp)
    a = gpu_decode(inp, d)
    b = gpu_decode(inp, d)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


# The CUDA-core kernel runs two CTAs of the split per block for up to 4 rows
# per unit, while both groups' shared memory and the per-sequence tables fit;
# a batch this large takes the one-group-per-block launch, a small one leaves
# the second group of the last block without a CTA (odd grid).
@pytest.mark.parametrize("batch,len_range,paged", [(1800, (1, 40), False), (3, (1, 40), False),
                                                    (24, (1, 3000), True), (900, (1, 40), True)])
def test_block_group_layouts_match_oracle(batch, len_range, paged):
    w = WORKLOADS["paged_cb"].with_(batch=batch, num_heads=8, num_kv_heads=2, len_range=len_range,
                                    paged=paged)
    inp = make_inputs(w, seed=5, fill="nan")
    _, out = gpu_step(inp, out_dtype=torch.float32)
    _, _, _, ref = oracle_step(inp)
    err = oracle.max_abs_diff(np64(out), ref)
    log_error(f"f32_out[groups_b{batch}_{'paged' if paged else 'contig'}]", err)
    assert err <= tol_for(w), f"max abs diff {err:.3e}"

