"""Sequence-sharded decode on one GPU, the shards emulated one after another:
shard appends + shard attention + the library merge against the oracle's
unsharded append + decode."""
import math

import numpy as np
import pytest
import torch

import kv_cache_decode_rope_b200 as kvd
import oracle
from kv_cache_decode_rope_b200.sharding import shard_bounds
from tests.gpu_util import log_error, np64

pytestmark = pytest.mark.gpu

CASES = [
    # name, dtype, B, Hq, Hkv, D, T, lens, capacity per shard, shards, paged
    ("core_f32_2", torch.float32, 3, 8, 2, 64, 1, [40, 7, 100], 64, 2, False),
    ("core_bf16_3_empty", torch.bfloat16, 2, 8, 2, 128, 1, [20, 150], 64, 3, False),
    ("tc_bf16_2", torch.bfloat16, 2, 32, 4, 128, 2, [300, 90], 256, 2, False),
    ("tc_bf16_3_paged", torch.bfloat16, 3, 64, 4, 128, 4, [500, 33, 260], 256, 3, True),
    ("tc_bf16_1", torch.bfloat16, 2, 16, 2, 128, 1, [70, 130], 160, 1, False),
]


def _paged(cache, P, gen):
    """[B, Hkv, C, D] -> pool [B*C/P, Hkv, P, D] and block table (random order)."""
    B, Hkv, C, D = cache.shape
    n = C // P
    perm = torch.randperm(B * n, generator=gen).to(torch.int32)
    bt = perm.view(B, n)
    pool = torch.empty((B * n, Hkv, P, D), dtype=cache.dtype)
    for b in range(B):
        for j in range(n):
            pool[bt[b, j]] = cache[b, :, j * P:(j + 1) * P]
    return pool, bt


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_sharded_step_matches_unsharded_oracle(case):
    name, dtype, B, Hq, Hkv, D, T, lens, C, S, paged = case
    gen = torch.Generator().manual_seed(7)
    L = torch.tensor(lens, dtype=torch.int32)
    cap_total = C * S
    assert int(L.max()) + T <= cap_total
    full_k = torch.randn((B, Hkv, cap_total, D), generator=gen).to(dtype)
    full_v = torch.randn((B, Hkv, cap_total, D), generator=gen).to(dtype)
    q = torch.randn((B, T, Hq, D), generator=gen).to(dtype)
    kn = torch.randn((B, T, Hkv, D), generator=gen).to(dtype)
    vn = torch.randn((B, T, Hkv, D), generator=gen).to(dtype)
    sc = 1 / math.sqrt(D)
    sdt = "f32" if dtype == torch.float32 else "bf16"
    q_rot, kc, vc = oracle.append_rope(np64(q), np64(kn), np64(vn), np64(full_k), np64(full_v),
                                       L.numpy(), 10000.0, sdt)
    ref = oracle.decode_attention(q_rot, kc, vc, L.numpy(), sc)

    seq = L.cuda()
    parts_o, parts_l = [], []
    for r in range(S):
        k_loc = full_k[:, :, r * C:(r + 1) * C].contiguous()
        v_loc = full_v[:, :, r * C:(r + 1) * C].contiguous()
        bt = None
        if paged:
            k_loc, bt = _paged(k_loc, 16, torch.Generator().manual_seed(r))
            v_loc, _ = _paged(v_loc, 16, torch.Generator().manual_seed(r))
            bt = bt.cuda()
        k_loc, v_loc = k_loc.cuda(), v_loc.cuda()
        qr = q.clone().cuda()
        start, slen = shard_bounds(seq, T, r, C)
        kvd.append_rope_shard(qr, kn.cuda(), vn.cuda(), k_loc, v_loc, seq, start, bt)
        o, lse = kvd.decode_attention_shard(qr, k_loc, v_loc, seq, start, slen, bt, scale=sc,
                                            max_kv_len=C)
        parts_o.append(o)
        parts_l.append(lse)
        if r == 0:   # rotated q equals the oracle's
            assert np.all(np.abs(np64(qr) - q_rot) <= np.abs(q_rot) * 2.0 ** -7 + 1e-30)
        # each shard alone against the oracle's shard attention on its own tokens
        kc_s = kc[:, :, r * C:(r + 1) * C]
        vc_s = vc[:, :, r * C:(r + 1) * C]
        o_ref, l_ref = oracle.decode_attention_shard(q_rot, kc_s, vc_s, L.numpy(), start.cpu().numpy(),
                                                     slen.cpu().numpy(), sc)
        live = np.isfinite(l_ref)
        assert np.array_equal(np.isfinite(np64(lse)), live), name
        assert np.max(np.abs(np64(lse)[live] - l_ref[live]), initial=0.0) <= 1e-3
        assert np.max(np.abs(np64(o) - o_ref)) <= (1e-5 if dtype == torch.float32 else 2e-3)
    out = kvd.merge_partials(torch.stack(parts_o), torch.stack(parts_l))
    torch.cuda.synchronize()
    err = oracle.max_abs_diff(np64(out), ref)
    log_error(f"shard[{name}]", err)
    assert err <= (1e-5 if dtype == torch.float32 else 2e-3), err


def test_rotate_only_matches_append():
    gen = torch.Generator().manual_seed(3)
    B, T, Hq, Hkv, D = 2, 3, 8, 2, 64
    q = torch.randn((B, T, Hq, D), generator=gen).to(torch.bfloat16).cuda()
    kn = torch.randn((B, T, Hkv, D), generator=gen).to(torch.bfloat16).cuda()
    seq = torch.tensor([5, 1000], dtype=torch.int32).cuda()
    q1, q2 = q.clone(), q.clone()
    kc = torch.zeros((B, Hkv, 1100, D), dtype=torch.bfloat16).cuda()
    kvd.append_rope(q1, kn, kn.clone(), kc, kc.clone(), seq)
    kvd.append_rope_shard(q2, None, None, None, None, seq, torch.zeros_like(seq))
    torch.cuda.synchronize()
    assert torch.equal(q1, q2)


def test_merge_of_one_shard_is_identity_and_empty_is_zero():
    gen = torch.Generator().manual_seed(4)
    o = torch.randn((1, 2, 1, 4, 64), generator=gen).cuda()
    lse = torch.randn((1, 2, 1, 4), generator=gen).cuda()
    assert torch.allclose(kvd.merge_partials(o, lse), o[0], atol=1e-6)
    lse_empty = torch.full_like(lse, -float("inf"))
    assert torch.equal(kvd.merge_partials(o, lse_empty), torch.zeros_like(o[0]))



@pytest.mark.parametrize("dtype,sdt,positions", [
    (torch.bfloat16, "bf16", [1_000_003, 16_777_219, 300_000_017, 1_073_741_000]),
    (torch.float32, "f32", [131_071, 262_147, 524_309, 1_048_573])])
def test_rotation_at_large_positions_matches_oracle(dtype, sdt, positions):
    """RoPE far beyond any cache here (bf16 up to ~2^30, fp32 up to 2^20:
    angles where the kernel's reduction by pi/2 does most of the work),
    through the rotate-only shard call.  Each rotated element lies within one
    storage ulp of the oracle's fp64 rotation rounded to the dtype, plus the
    spread that the fp64 angle itself carries at that position (about
    position x 2^-52 rad, both sides forming it from base^(-2j/r) in fp64),
    and nearly all are bit-exact."""
    gen = torch.Generator().manual_seed(8)
    B, T, Hq, D = len(positions), 2, 4, 128
    q = torch.randn((B, T, Hq, D), generator=gen).to(dtype)
    L = torch.tensor(positions, dtype=torch.int32)
    dq = q.cuda()
    kvd.append_rope_shard(dq, None, None, None, None, L.cuda(), torch.zeros_like(L).cuda())
    torch.cuda.synchronize()
    pos = (L[:, None].to(torch.float64) + torch.arange(T, dtype=torch.float64)[None, :]).numpy()
    x = np64(q)
    ref = oracle.round_store(oracle.rope(x, pos[:, :, None], 10000.0), sdt)
    got = np64(dq)
    ulp = 2.0 ** (-7 if dtype == torch.bfloat16 else -23)
    angle_spread = 8 * float(pos.max()) * 2.0 ** -52                     # rad
    pair_mag = np.abs(x) + np.abs(np.concatenate([x[..., D // 2:], x[..., :D // 2]], -1))
    bound = np.abs(ref) * ulp + angle_spread * pair_mag + 1e-30
    assert np.all(np.abs(got - ref) <= bound), float(np.max(np.abs(got - ref) / bound))
    # the angle spread can flip a rounding tie: rarely in bf16, up to a few
    # tenths of a percent of fp32 values at 2^20
    assert np.mean(got == ref) >= (0.995 if dtype == torch.bfloat16 else 0.98), float(np.mean(got == ref))
