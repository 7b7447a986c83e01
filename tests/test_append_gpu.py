"""kv_append_rope on the GPU against the oracle: RoPE values, slot indexing and
untouched memory."""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_decode_rope_b200.workloads import WORKLOADS, make_inputs
from tests.gpu_util import gpu_append, np64, to_device

pytestmark = pytest.mark.gpu


def ulp(x: np.ndarray, dtype: str) -> np.ndarray:
    mant = 7 if dtype == "bf16" else 23
    e = np.floor(np.log2(np.maximum(np.abs(x), 1e-30)))
    return np.exp2(e - mant)


def bits(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    return (t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)).numpy()


CASES = {
    "gqa_bf16": WORKLOADS["batched_gqa"].with_(batch=3, cache_len=37),
    "paged_bf16": WORKLOADS["paged_cb"].with_(batch=5, len_range=(1, 300)),
    "mtp_bf16": WORKLOADS["mtp_verify"].with_(batch=2, cache_len=45),
    "tiny_f32": WORKLOADS["tiny_mha"].with_(cache_mode="random", cache_len=20, q_len=3),
    "ferric_f32_d16": WORKLOADS["tiny_mha"].with_(cache_mode="random", num_heads=4, num_kv_heads=4,
                                                   head_dim=16, cache_len=4),
    "long_pos_bf16": WORKLOADS["long_ctx"].with_(batch=1, num_heads=4, num_kv_heads=1,
                                                 cache_len=131072, peaked_frac=0.0),
    "d256_bf16": WORKLOADS["batched_gqa"].with_(batch=2, head_dim=256, cache_len=17, q_len=2),
    "d32_f32_paged": WORKLOADS["paged_cb"].with_(batch=3, dtype="f32", head_dim=32, num_heads=4,
                                                 num_kv_heads=2, len_range=(5, 90), q_len=2),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_append_matches_oracle(name):
    w = CASES[name]
    inp = make_inputs(w, seed=3, fill="nan")
    d = to_device(inp)
    gpu_append(inp, d)
    torch.cuda.synchronize()
    bt = None if inp["block_table"] is None else inp["block_table"].numpy()
    seq = inp["seq_lens"].numpy()
    q_rot, k_rot, v_st = oracle.rotate_new_tokens(np64(inp["q"]), np64(inp["k_new"]), np64(inp["v_new"]),
                                                  seq, w.rope_base, w.dtype)
    # rotated q: within one storage ulp, nearly always identical
    gq = np64(d["q"])
    assert np.all(np.abs(gq - q_rot) <= ulp(q_rot, w.dtype)), name
    mism_q = int(np.sum(gq != q_rot))
    assert mism_q <= max(2, gq.size // 10000), f"{name}: {mism_q} q elements off by one ulp"

    kc, vc = d["k_cache"].cpu(), d["v_cache"].cpu()
    k_bits_before, v_bits_before = bits(inp["k_cache"]), bits(inp["v_cache"])
    k_bits, v_bits = bits(kc), bits(vc)
    written = np.zeros(k_bits.shape[:-1], bool)  # (…, slot) of every written row
    P = kc.shape[2]
    for b in range(w.batch):
        for i in range(w.q_len):
            p = int(seq[b]) + i
            if bt is None:
                idx = (b, slice(None), p)
            else:
                idx = (int(bt[b, p // P]), slice(None), p % P)
            written[idx] = True
            gk = kc[idx].float().numpy().astype(np.float64)          # [Hkv, D]
            assert np.all(np.abs(gk - k_rot[b, i]) <= ulp(k_rot[b, i], w.dtype)), (name, b, i)
            # v is copied bit for bit
            assert np.array_equal(v_bits[idx], bits(inp["v_new"][b, i])), (name, b, i)
    # every other slot is untouched (bitwise, NaN sentinels included)
    assert np.array_equal(k_bits[~written], k_bits_before[~written])
    assert np.array_equal(v_bits[~written], v_bits_before[~written])


def test_paged_append_equals_contiguous_append():
    w = WORKLOADS["paged_cb"].with_(batch=4, len_range=(3, 200), q_len=3)
    inp = make_inputs(w, seed=5, fill="zero")
    d = to_device(inp)
    gpu_append(inp, d)
    # the same tokens into a contiguous cache
    cap = int(inp["seq_lens"].max()) + w.q_len
    kc = torch.zeros((w.batch, w.num_kv_heads, cap, w.head_dim), dtype=w.torch_dtype, device="cuda")
    vc = torch.zeros_like(kc)
    inp2 = dict(inp, block_table=None)
    d2 = dict(to_device(inp2), k_cache=kc, v_cache=vc)
    gpu_append(inp2, d2)
    torch.cuda.synchronize()
    bt = inp["block_table"]
    P = w.page_size
    for b in range(w.batch):
        for i in range(w.q_len):
            p = int(inp["seq_lens"][b]) + i
            page = int(bt[b, p // P])
            assert torch.equal(d["k_cache"][page, :, p % P].view(torch.int16), kc[b, :, p].view(torch.int16))
            assert torch.equal(d["v_cache"][page, :, p % P].view(torch.int16), vc[b, :, p].view(torch.int16))
    assert torch.equal(d["q"].view(torch.int16), d2["q"].view(torch.int16))


def test_position_zero_keeps_k():
    """RoPE at position 0 is the identity: k lands bit for bit."""
    w = WORKLOADS["batched_gqa"].with_(batch=2, cache_len=0)
    inp = make_inputs(w, seed=1)
    d = to_device(inp)
    gpu_append(inp, d)
    torch.cuda.synchronize()
    for b in range(w.batch):
        assert torch.equal(d["k_cache"][b, :, 0].cpu().view(torch.int16), inp["k_new"][b, 0].view(torch.int16))


# ---------------------------------------------------------------- RoPE layouts
LAYOUT_CASES = [
    # (name, workload, interleaved, rotary_dim)
    ("interleaved_bf16", WORKLOADS["batched_gqa"].with_(batch=3, cache_len=1000), True, 0),
    ("partial64_bf16_paged", WORKLOADS["paged_cb"].with_(batch=3, len_range=(1, 5000)), False, 64),
    ("interleaved_partial32_f32", WORKLOADS["tiny_mha"].with_(cache_mode="random", cache_len=77,
                                                              q_len=2), True, 32),
    ("partial16_d16_f32", WORKLOADS["tiny_mha"].with_(cache_mode="random", num_heads=4,
                                                      num_kv_heads=2, head_dim=16, cache_len=9),
     False, 16),
    ("interleaved_partial128_d256", WORKLOADS["batched_gqa"].with_(batch=2, head_dim=256,
                                                                   cache_len=17, q_len=2), True, 128),
    ("interleaved_long_pos", WORKLOADS["long_ctx"].with_(batch=1, num_heads=4, num_kv_heads=1,
                                                         cache_len=131072, peaked_frac=0.0), True, 0),
]


@pytest.mark.parametrize("name,w,inter,rd", LAYOUT_CASES, ids=[c[0] for c in LAYOUT_CASES])
def test_append_layouts_match_oracle(name, w, inter, rd):
    """Interleaved pairing and partial rotary width: rotated q and k within one
    storage ulp of the oracle, the unrotated tail of k copied bit for bit,
    v bit for bit, every other slot untouched."""
    import kv_cache_decode_rope_b200 as kvd
    inp = make_inputs(w, seed=5, fill="nan")
    d = to_device(inp)
    kvd.append_rope(d["q"], d["k_new"], d["v_new"], d["k_cache"], d["v_cache"], d["seq_lens"],
                    d["block_table"], rope_base=w.rope_base, interleaved=inter, rotary_dim=rd)
    torch.cuda.synchronize()
    bt = None if inp["block_table"] is None else inp["block_table"].numpy()
    seq = inp["seq_lens"].numpy()
    q_rot, k_rot, _ = oracle.rotate_new_tokens(np64(inp["q"]), np64(inp["k_new"]), np64(inp["v_new"]),
                                               seq, w.rope_base, w.dtype, inter, rd)
    gq = np64(d["q"])
    assert np.all(np.abs(gq - q_rot) <= ulp(q_rot, w.dtype)), name
    assert int(np.sum(gq != q_rot)) <= max(2, gq.size // 10000)
    r = rd or w.head_dim
    # the unrotated tail of q is left exactly as it was
    assert np.array_equal(bits(d["q"])[..., r:], bits(inp["q"])[..., r:])
    kc, vc = d["k_cache"].cpu(), d["v_cache"].cpu()
    k_bits_before, v_bits_before = bits(inp["k_cache"]), bits(inp["v_cache"])
    k_bits, v_bits = bits(kc), bits(vc)
    written = np.zeros(k_bits.shape[:-1], bool)
    P = kc.shape[2]
    for b in range(w.batch):
        for i in range(w.q_len):
            p = int(seq[b]) + i
            idx = (b, slice(None), p) if bt is None else (int(bt[b, p // P]), slice(None), p % P)
            written[idx] = True
            gk = kc[idx].float().numpy().astype(np.float64)
            assert np.all(np.abs(gk - k_rot[b, i]) <= ulp(k_rot[b, i], w.dtype)), (name, b, i)
            assert np.array_equal(k_bits[idx][..., r:], bits(inp["k_new"][b, i])[..., r:])
            assert np.array_equal(v_bits[idx], bits(inp["v_new"][b, i]))
    assert np.array_equal(k_bits[~written], k_bits_before[~written])
    assert np.array_equal(v_bits[~written], v_bits_before[~written])


@pytest.mark.parametrize("inter,rd", [(True, 0), (False, 32), (True, 64)])
def test_layout_step_matches_full_recompute(inter, rd):
    """Prefill by feeding tokens through append + decode with a RoPE layout,
    then compare every step with the oracle's full causal recompute (fp32)."""
    import math
    import kv_cache_decode_rope_b200 as kvd
    B, N, Hq, Hkv, D = 2, 24, 8, 2, 64
    gen = torch.Generator().manual_seed(31)
    q_raw = torch.rand((B, N, Hq, D), generator=gen) * 0.2 - 0.1
    k_raw = torch.rand((B, N, Hkv, D), generator=gen) * 0.2 - 0.1
    v_raw = torch.rand((B, N, Hkv, D), generator=gen) * 0.2 - 0.1
    kc = torch.zeros((B, Hkv, N, D), device="cuda")
    vc = torch.zeros_like(kc)
    sc = 1 / math.sqrt(D)
    ref = oracle.full_causal_attention(q_raw.double().numpy(), k_raw.double().numpy(),
                                       v_raw.double().numpy(), sc, 10000.0, "f32", inter, rd)
    worst = 0.0
    for L in range(N):
        q = q_raw[:, L:L + 1].contiguous().cuda()
        seq = torch.full((B,), L, dtype=torch.int32, device="cuda")
        kvd.append_rope(q, k_raw[:, L:L + 1].contiguous().cuda(), v_raw[:, L:L + 1].contiguous().cuda(),
                        kc, vc, seq, interleaved=inter, rotary_dim=rd)
        out = kvd.decode_attention(q, kc, vc, seq, scale=sc, max_kv_len=L + 1)
        worst = max(worst, float(np.max(np.abs(np64(out)[:, 0] - ref[:, L]))))
    assert worst <= 1e-5, worst
