"""Pins for the fp64 oracle: checks against facts fixed by the pages and by
mathematics, not against the oracle itself.

Each pin takes the oracle module ``m`` and raises AssertionError on failure, so
the same checks run on the real oracle (all must pass) and on copies with a
planted mistake (at least one must fail).
"""
from __future__ import annotations

import json
import math
import os
import struct
from fractions import Fraction

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rng(seed=0):
    return np.random.default_rng(seed)


# --------------------------------------------------------------- bf16 rounding
def pin_bf16_matches_torch_cast(m):
    """For fp32 inputs a single fp64 -> bf16 rounding equals torch's fp32 ->
    bf16 cast (round to nearest even): random magnitudes, exact ties, values
    next to ties, subnormals and the overflow edge."""
    r = rng(1)
    vals = [r.standard_normal(20000).astype(np.float32),
            (r.standard_normal(20000) * 10.0 ** r.integers(-40, 38, 20000)).astype(np.float32)]
    # exact ties and their neighbours: low 16 bits 0x8000, 0x7fff, 0x8001
    hi = r.integers(0, 0x7f7f, 5000, dtype=np.uint32) << 16
    for low in (0x8000, 0x7FFF, 0x8001, 0x0000):
        vals.append((hi | np.uint32(low)).view(np.float32))
    vals.append(np.array([1e-40, -3e-39, 3.3895e38, 3.3896e38, 3.4e38, -3.39e38,
                          np.finfo(np.float32).max, 2.0 ** -133, 2.0 ** -134], np.float32))
    x = np.concatenate(vals)
    x = x[np.isfinite(x)]
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = m.bf16_round(x.astype(np.float64))
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all(), f"bf16 mismatch at {x[~same][:5]}"


def _bf16_value(bits: int) -> Fraction:
    return Fraction(struct.unpack(">f", struct.pack(">I", bits << 16))[0])


def _bf16_nearest_bruteforce(x: float) -> float:
    """Exact nearest bfloat16 (ties to even) by search over the 16-bit codes."""
    if x == 0:
        return x
    sign = 0x8000 if x < 0 else 0
    ax = Fraction(abs(x))
    lo, hi = 0, 0x7F80          # positive finite codes 0..0x7f7f; 0x7f80 = inf
    while hi - lo > 1:          # largest code with value <= ax
        mid = (lo + hi) // 2
        if _bf16_value(mid) <= ax:
            lo = mid
        else:
            hi = mid
    below = lo
    above = lo + 1
    if above == 0x7F80:
        # above the largest finite value: the halfway point to 2^128 decides
        if ax >= _bf16_value(0x7F7F) + (Fraction(2) ** 128 - _bf16_value(0x7F7F)) / 2:
            return math.copysign(math.inf, x)
        return math.copysign(float(_bf16_value(below)), x)
    d_lo = ax - _bf16_value(below)
    d_hi = _bf16_value(above) - ax
    code = below if (d_lo < d_hi or (d_lo == d_hi and below % 2 == 0)) else above
    return math.copysign(float(_bf16_value(code)), x)


def pin_bf16_bruteforce_fp64(m):
    """fp64 inputs (not representable in fp32) against an exact search."""
    r = rng(2)
    xs = list(r.standard_normal(300) * 10.0 ** r.integers(-30, 30, 300))
    # fp64 values within 1 fp64 ulp of a bf16 tie
    for base_bits in r.integers(0x0080, 0x7F7F, 100):
        tie = (_bf16_value(int(base_bits)) + _bf16_value(int(base_bits) + 1)) / 2
        t = float(tie)
        xs += [t, np.nextafter(t, 0), np.nextafter(t, np.inf), -t]
    xs += [1e-41, -7.1e-40, 3.3961e38, 3.40e38]
    got = m.bf16_round(np.array(xs, np.float64))
    for x, g in zip(xs, got):
        e = _bf16_nearest_bruteforce(float(x))
        assert g == e, f"bf16_round({x!r}) = {g!r}, expected {e!r}"


# ------------------------------------------------------------------------ RoPE
def pin_rope_inv_freq_closed_form(m):
    assert np.array_equal(m.rope_inv_freq(4, 10000.0), [1.0, 0.01])
    np.testing.assert_allclose(m.rope_inv_freq(8, 10000.0), [1.0, 0.1, 0.01, 0.001],
                               rtol=1e-15)


def pin_rope_hand_case(m):
    """D=4, base 10000: pairs (0,2), (1,3) with angles p*1 and p*0.01."""
    x = np.array([1.0, 0.0, 0.0, 0.0])
    got = m.rope(x, 1, 10000.0)
    np.testing.assert_allclose(got, [math.cos(1), 0.0, math.sin(1), 0.0], atol=1e-15)
    y = np.array([0.0, 2.0, 0.0, 0.0])
    got = m.rope(y, 100, 10000.0)       # angle 100 * 0.01 = 1 on pair (1,3)
    np.testing.assert_allclose(got, [0.0, 2 * math.cos(1), 0.0, 2 * math.sin(1)], atol=1e-14)
    z = np.array([0.0, 0.0, 3.0, 0.0])  # second member of pair 0: (0,3) -> (-3 sin, 3 cos)
    got = m.rope(z, 2, 10000.0)
    np.testing.assert_allclose(got, [-3 * math.sin(2), 0.0, 3 * math.cos(2), 0.0], atol=1e-14)


def pin_rope_2d_rotation(m):
    """D = 2 is a plain rotation of the plane by p radians (theta_0 = 1)."""
    r = rng(3)
    for _ in range(20):
        v = r.standard_normal(2)
        p = int(r.integers(0, 100000))
        c, s = math.cos(p), math.sin(p)
        np.testing.assert_allclose(m.rope(v, p, 10000.0),
                                   [c * v[0] - s * v[1], s * v[0] + c * v[1]], atol=1e-12)


def pin_rope_identity_norm_shift(m):
    r = rng(4)
    x = r.standard_normal((6, 64))
    assert np.array_equal(m.rope(x, 0, 10000.0), x)                     # p = 0: identity
    pos = r.integers(0, 131073, 6)
    y = m.rope(x, pos, 10000.0)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1),
                               rtol=1e-13)                                # rotation: norm kept
    q, k = r.standard_normal(64), r.standard_normal(64)
    for (p, mm, s) in [(5, 3, 11), (131072, 7, 1000), (0, 4096, 123457)]:
        a = np.dot(m.rope(q, p + s, 10000.0), m.rope(k, mm + s, 10000.0))
        b = np.dot(m.rope(q, p, 10000.0), m.rope(k, mm, 10000.0))
        assert abs(a - b) <= 1e-9 * (1 + abs(b)), (p, mm, s, a, b)        # depends on p - m only


def pin_rope_complex_form(m):
    """Half-split RoPE equals multiplying z_j = x_j + i x_{j+D/2} by
    exp(i p theta_j)."""
    r = rng(5)
    x = r.standard_normal((3, 128))
    pos = np.array([0, 17, 131072])
    theta = 10000.0 ** (-np.arange(64) * 2.0 / 128)
    z = (x[:, :64] + 1j * x[:, 64:]) * np.exp(1j * pos[:, None] * theta[None, :])
    np.testing.assert_allclose(m.rope(x, pos, 10000.0),
                               np.concatenate([z.real, z.imag], -1), atol=1e-9)


def pin_rope_interleaved_hand_case(m):
    """Interleaved D=4, base 10000: pairs (0,1) and (2,3) with angles p*1 and p*0.01."""
    got = m.rope(np.array([1.0, 0.0, 0.0, 0.0]), 1, 10000.0, interleaved=True)
    np.testing.assert_allclose(got, [math.cos(1), math.sin(1), 0.0, 0.0], atol=1e-15)
    got = m.rope(np.array([0.0, 0.0, 0.0, 2.0]), 100, 10000.0, interleaved=True)
    np.testing.assert_allclose(got, [0.0, 0.0, -2 * math.sin(1), 2 * math.cos(1)], atol=1e-14)


def pin_rope_interleaved_is_permuted_half_split(m):
    """Interleaved pairing is half-split pairing of the vector whose first half
    holds the even elements and second half the odd ones."""
    r = rng(12)
    for D in (2, 8, 64, 128):
        x = r.standard_normal((5, D))
        pos = r.integers(0, 131073, 5)
        perm = np.concatenate([np.arange(0, D, 2), np.arange(1, D, 2)])
        half = m.rope(x[:, perm], pos, 10000.0)
        back = np.empty_like(half)
        back[:, perm] = half
        np.testing.assert_allclose(m.rope(x, pos, 10000.0, interleaved=True), back,
                                   rtol=0, atol=1e-12)


def pin_rope_partial_dims(m):
    """rotary_dim r < D: the last D - r elements pass through untouched and the
    first r are the full rotation of an r-vector (theta_j = base^(-2j/r)), for
    both pairings; r = D is the plain rotation."""
    r_ = rng(13)
    for (D, r, inter) in [(8, 4, False), (8, 4, True), (64, 32, False), (128, 64, True),
                          (128, 16, False)]:
        x = r_.standard_normal((4, D))
        pos = r_.integers(0, 131073, 4)
        got = m.rope(x, pos, 10000.0, interleaved=inter, rotary_dim=r)
        assert np.array_equal(got[:, r:], x[:, r:])
        np.testing.assert_allclose(got[:, :r], m.rope(x[:, :r], pos, 10000.0, interleaved=inter),
                                   rtol=0, atol=1e-12)
        assert np.array_equal(m.rope(x, pos, 10000.0, inter, D), m.rope(x, pos, 10000.0, inter))
    # closed form: D = 8, r = 4, base 100 -> theta = (1, 0.1), pair (0, 2) and (1, 3)
    got = m.rope(np.array([0.0, 1.0, 0.0, 0.0, 5.0, 6.0, 7.0, 8.0]), 10, 100.0, rotary_dim=4)
    np.testing.assert_allclose(got, [0.0, math.cos(1), 0.0, math.sin(1), 5.0, 6.0, 7.0, 8.0],
                               atol=1e-14)


def pin_rope_layouts_keep_relative_position(m):
    """Every layout keeps <rope(q, p + s), rope(k, m + s)> a function of p - m."""
    r = rng(14)
    q, k = r.standard_normal(64), r.standard_normal(64)
    for (inter, rd) in [(True, 0), (False, 32), (True, 16)]:
        for (p, mm, s) in [(5, 3, 11), (131072, 7, 1000)]:
            a = np.dot(m.rope(q, p + s, 10000.0, inter, rd), m.rope(k, mm + s, 10000.0, inter, rd))
            b = np.dot(m.rope(q, p, 10000.0, inter, rd), m.rope(k, mm, 10000.0, inter, rd))
            assert abs(a - b) <= 1e-9 * (1 + abs(b)), (inter, rd, p, mm, s)


def pin_layouts_decode_equals_full_recompute(m):
    """Cached decode with each RoPE layout equals the full recompute with it."""
    for (inter, rd, D) in [(True, 0, 16), (False, 8, 16), (True, 16, 32)]:
        B, N, Hq, Hkv = 2, 7, 4, 2
        q, k, v = _raw_sequence(40 + D, B, N, Hq, Hkv, D)
        sc = 1 / math.sqrt(D)
        kc = np.full((B, Hkv, N + 1, D), np.nan)
        vc = kc.copy()
        outs = []
        for L in range(N):
            seq = np.full(B, L)
            q_rot, kc, vc = m.append_rope(q[:, L:L + 1], k[:, L:L + 1], v[:, L:L + 1], kc, vc, seq,
                                          10000.0, "f32", None, inter, rd)
            outs.append(m.decode_attention(q_rot, kc, vc, seq, sc))
        got = np.concatenate(outs, 1)
        ref = m.full_causal_attention(q, k, v, sc, 10000.0, "f32", inter, rd)
        assert np.max(np.abs(got - ref)) <= 1e-12


# ------------------------------------------------------------------- attention
def _attend_bruteforce(q_rows, K, V, scale, visible):
    """Pure-Python softmax attention, one element at a time."""
    R, D = len(q_rows), len(q_rows[0])
    out = []
    for r in range(R):
        n = visible[r]
        s = [scale * sum(q_rows[r][d] * K[t][d] for d in range(D)) for t in range(n)]
        mx = max(s)
        w = [math.exp(v - mx) for v in s]
        tot = sum(w)
        out.append([sum(w[t] * V[t][d] for t in range(n)) / tot for d in range(len(V[0]))])
    return np.array(out)


def pin_attend_bruteforce(m):
    r = rng(6)
    for (R, N, D) in [(1, 1, 4), (3, 7, 8), (4, 40, 16), (2, 33, 5)]:
        q = r.standard_normal((R, D))
        K = r.standard_normal((N, D))
        V = r.standard_normal((N, D))
        vis = r.integers(1, N + 1, R)
        sc = 1 / math.sqrt(D)
        np.testing.assert_allclose(m.attend(q, K, V, sc, vis),
                                   _attend_bruteforce(q.tolist(), K.tolist(), V.tolist(), sc, vis),
                                   atol=1e-13)


def pin_attend_special_cases(m):
    r = rng(7)
    D = 16
    V = r.standard_normal((9, D))
    q = r.standard_normal((1, D))
    # length 1: the single weight is 1
    K = r.standard_normal((9, D))
    np.testing.assert_allclose(m.attend(q, K, V, 0.3, [1]), V[:1], atol=0)
    # identical keys: uniform weights -> mean of V
    Ks = np.repeat(K[:1], 9, 0)
    np.testing.assert_allclose(m.attend(q, Ks, V, 0.3, [9]), V.mean(0, keepdims=True), atol=1e-14)
    # one dominant key (score margin > 100): that V row
    Kd = K.copy()
    Kd[4] = q[0] * 200.0
    np.testing.assert_allclose(m.attend(q, Kd, V, 1.0, [9]), V[4:5], atol=1e-14)
    # two keys: w0 = 1 / (1 + exp(s1 - s0))
    s0 = 0.25 * float(q[0] @ K[0])
    s1 = 0.25 * float(q[0] @ K[1])
    w0 = 1.0 / (1.0 + math.exp(s1 - s0))
    np.testing.assert_allclose(m.attend(q, K[:2], V[:2], 0.25, [2])[0],
                               w0 * V[0] + (1 - w0) * V[1], atol=1e-14)
    # masked keys do not matter
    V2 = V.copy()
    V2[5:] = 1e6
    np.testing.assert_allclose(m.attend(q, K, V2, 0.3, [5]), m.attend(q, K[:5], V[:5], 0.3, [5]),
                               atol=1e-13)


# ------------------------------------------------------------ decode vs recompute
def _raw_sequence(seed, B, N, Hq, Hkv, D):
    r = rng(seed)
    return (r.uniform(-1, 1, (B, N, Hq, D)), r.uniform(-1, 1, (B, N, Hkv, D)),
            r.uniform(-1, 1, (B, N, Hkv, D)))


def _cached_steps(m, q_raw, k_raw, v_raw, steps, dtype, base, scale, paged=False, seed=0):
    """Feed the sequences through append + decode in chunks ``steps`` (token
    counts per step, all sequences alike); return the decode outputs stacked in
    position order, plus the final caches."""
    B, N, Hq, D = q_raw.shape
    Hkv = k_raw.shape[2]
    P = 4
    if paged:
        pages = (N + P - 1) // P
        perm = rng(seed + 99).permutation(B * pages)
        bt = perm.reshape(B, pages)
        kc = np.full((B * pages, Hkv, P, D), np.nan)
    else:
        bt = None
        kc = np.full((B, Hkv, N + 3, D), np.nan)
    vc = kc.copy()
    outs = []
    L = 0
    for T in steps:
        seq = np.full(B, L)
        q_rot, kc, vc = m.append_rope(q_raw[:, L:L + T], k_raw[:, L:L + T], v_raw[:, L:L + T],
                                      kc, vc, seq, base, dtype, bt)
        outs.append(m.decode_attention(q_rot, kc, vc, seq, scale, bt))
        L += T
    return np.concatenate(outs, 1), kc, vc, bt


def pin_decode_equals_full_recompute(m):
    """The central check of generate.rs `run`: cached decode equals a full
    non-cached causal recompute, here at every position of the sequence."""
    for (B, N, Hq, Hkv, D, steps, dtype) in [
        (2, 12, 4, 2, 8, [1] * 12, "f32"),
        (2, 13, 6, 2, 16, [5, 1, 4, 3], "bf16"),
        (1, 9, 4, 4, 16, [9], "f32"),
    ]:
        q, k, v = _raw_sequence(N, B, N, Hq, Hkv, D)
        sc = 1 / math.sqrt(D)
        got, _, _, _ = _cached_steps(m, q, k, v, steps, dtype, 10000.0, sc)
        ref = m.full_causal_attention(q, k, v, sc, 10000.0, dtype)
        assert np.max(np.abs(got - ref)) <= 1e-12, np.max(np.abs(got - ref))


def pin_ferric_example(m):
    """The worked example's shape (h=4, dh=16, base 10000): prompt tokens fed
    one per step, then the generated steps; each step vs full recompute."""
    g = json.load(open(os.path.join(GOLDEN, "ferric_example.json")))
    H, D, base = g["num_heads"], g["head_dim"], g["rope_base"]
    N = g["prompt_len"] + g["gen_steps"]
    q, k, v = _raw_sequence(42, 1, N, H, H, D)
    sc = 1 / math.sqrt(D)
    got, _, _, _ = _cached_steps(m, q, k, v, [1] * N, "f32", base, sc)
    ref = m.full_causal_attention(q, k, v, sc, base, "f32")
    assert np.max(np.abs(got - ref)) < 1e-12


def pin_paged_equals_contiguous(m):
    B, N, Hq, Hkv, D = 3, 11, 4, 2, 8
    q, k, v = _raw_sequence(8, B, N, Hq, Hkv, D)
    sc = 0.35
    a, _, _, _ = _cached_steps(m, q, k, v, [6, 2, 3], "bf16", 500.0, sc, paged=False)
    for seed in (1, 2):
        b, _, _, _ = _cached_steps(m, q, k, v, [6, 2, 3], "bf16", 500.0, sc, paged=True, seed=seed)
        assert np.array_equal(a, b)
    ref = m.full_causal_attention(q, k, v, sc, 500.0, "bf16")
    assert np.max(np.abs(a - ref)) <= 1e-12


def pin_append_layout(m):
    """k lands rotated at slot L_b + i, v unrotated, other slots untouched."""
    r = rng(9)
    B, T, Hq, Hkv, D = 2, 2, 2, 1, 4
    q = r.standard_normal((B, T, Hq, D))
    kn = r.standard_normal((B, T, Hkv, D))
    vn = r.standard_normal((B, T, Hkv, D))
    kc = np.full((B, Hkv, 8, D), 7.0)
    vc = np.full((B, Hkv, 8, D), 7.0)
    seq = np.array([0, 5])
    q_rot, kc2, vc2 = m.append_rope(q, kn, vn, kc, vc, seq, 10000.0, "f32")
    for b in range(B):
        for i in range(T):
            p = seq[b] + i
            # hand rotation of the D=4 vector at position p: pairs (0,2) angle p, (1,3) angle p/100
            x = kn[b, i, 0]
            c0, s0, c1, s1 = math.cos(p), math.sin(p), math.cos(p * 0.01), math.sin(p * 0.01)
            exp = [x[0] * c0 - x[2] * s0, x[1] * c1 - x[3] * s1,
                   x[0] * s0 + x[2] * c0, x[1] * s1 + x[3] * c1]
            np.testing.assert_allclose(kc2[b, 0, p], np.float32(exp), atol=1e-7)
            assert np.array_equal(vc2[b, 0, p], vn[b, i, 0].astype(np.float32))
    untouched = np.ones(8, bool)
    assert np.all(kc2[0, 0, 2:] == 7.0) and np.all(kc2[1, 0, :5] == 7.0) and np.all(kc2[1, 0, 7:] == 7.0)
    assert np.all(vc2[0, 0, 2:] == 7.0) and untouched.all()


def pin_gqa_mapping(m):
    """q head h reads kv head h // g: give each kv head a constant V."""
    B, T, Hq, Hkv, D, L = 1, 1, 8, 2, 4, 6
    r = rng(10)
    q = r.standard_normal((B, T, Hq, D))
    kc = r.standard_normal((B, Hkv, L + 1, D))
    vc = np.zeros((B, Hkv, L + 1, D))
    for h in range(Hkv):
        vc[:, h] = h + 1.0
    out = m.decode_attention(q, kc, vc, np.array([L]), 0.5)
    for h in range(Hq):
        np.testing.assert_allclose(out[0, 0, h], h // (Hq // Hkv) + 1.0, atol=1e-14)
    # Hkv = Hq with K/V repeated per group gives the same output
    kc_rep = np.repeat(kc, Hq // Hkv, axis=1)
    vc_rep = r.standard_normal((B, Hq, L + 1, D))
    vc_grp = vc_rep[:, ::Hq // Hkv]
    vc_rep = np.repeat(vc_grp, Hq // Hkv, axis=1)
    a = m.decode_attention(q, kc, vc_grp, np.array([L]), 0.5)
    b = m.decode_attention(q, kc_rep, vc_rep, np.array([L]), 0.5)
    np.testing.assert_allclose(a, b, atol=1e-14)


def pin_causal_among_drafts(m):
    """New token i must not see new tokens after it: editing token L_b + 1
    leaves draft 0 unchanged and moves draft 1."""
    r = rng(11)
    B, T, Hq, Hkv, D, L = 1, 3, 2, 1, 8, 5
    q = r.standard_normal((B, T, Hq, D))
    kc = r.standard_normal((B, Hkv, L + T, D))
    vc = r.standard_normal((B, Hkv, L + T, D))
    a = m.decode_attention(q, kc, vc, np.array([L]), 0.4)
    vc2 = vc.copy()
    vc2[0, 0, L + 1] += 10.0
    b = m.decode_attention(q, kc, vc2, np.array([L]), 0.4)
    assert np.array_equal(a[0, 0], b[0, 0])
    assert np.all(np.abs(a[0, 1] - b[0, 1]) > 1e-6)
    assert np.all(np.abs(a[0, 2] - b[0, 2]) > 1e-6)


# ------------------------------------------------------------ shared prefixes
def pin_copy_on_write_boundary_page(m):
    """Two sequences share a prefix of 6 tokens (P = 4: one full page and a
    boundary page half used).  Each gets a fresh boundary page by copy on
    write; after the append, each decodes exactly as with private pages, and
    the shared pages are unchanged."""
    r = rng(17)
    B, T, Hq, Hkv, D, P = 2, 2, 4, 2, 8, 4
    shared = r.standard_normal((2, Hkv, P, D)), r.standard_normal((2, Hkv, P, D))  # pages 0, 1
    kc = np.full((8, Hkv, P, D), np.nan)
    vc = kc.copy()
    kc[0:2], vc[0:2] = shared[0], shared[1]
    L = np.array([6, 6])
    bt = np.array([[0, 2, 3], [0, 4, 5]])          # boundary pages 2 and 4 are fresh
    cow = np.array([1, 1])                          # both shared page 1
    q, kn, vn = (r.standard_normal((B, T, Hq, D)), r.standard_normal((B, T, Hkv, D)),
                 r.standard_normal((B, T, Hkv, D)))
    q_rot, kc2, vc2 = m.append_rope(q, kn, vn, kc, vc, L, 10000.0, "f32", bt, cow_src=cow)
    assert np.array_equal(kc2[0:2], kc[0:2]) and np.array_equal(vc2[0:2], vc[0:2])
    # private reference: each sequence's own contiguous copy of the prefix
    kp = np.full((B, Hkv, 12, D), np.nan)
    vp = kp.copy()
    for b in range(B):
        for t in range(6):
            kp[b, :, t] = kc[t // P, :, t % P]
            vp[b, :, t] = vc[t // P, :, t % P]
    q_p, kp2, vp2 = m.append_rope(q, kn, vn, kp, vp, L, 10000.0, "f32")
    a = m.decode_attention(q_rot, kc2, vc2, L, 0.3, bt)
    b_ = m.decode_attention(q_p, kp2, vp2, L, 0.3)
    np.testing.assert_allclose(a, b_, atol=1e-14)
    for b in range(B):   # the fresh page holds the copied slots, then the new tokens
        np.testing.assert_array_equal(kc2[bt[b, 1], :, :2], kc[1, :, :2])
    # no copy when the boundary falls on a page start
    _, kc3, _ = m.append_rope(q, kn, vn, kc2, vc2, np.array([8, 8]), 10000.0, "f32", bt,
                              cow_src=np.array([2, 4]))
    assert np.array_equal(kc3[3, :, 2:], kc2[3, :, 2:], equal_nan=True)


def pin_shared_prefix_decode(m):
    """Sequences whose block tables share prefix pages decode as with private copies."""
    r = rng(18)
    B, T, Hq, Hkv, D, P = 3, 1, 4, 2, 8, 4
    pool = 2 + 3 * 2
    kc = r.standard_normal((pool, Hkv, P, D))
    vc = r.standard_normal((pool, Hkv, P, D))
    bt = np.array([[0, 1, 2, 3], [0, 1, 4, 5], [0, 1, 6, 7]])   # 8 shared tokens
    L = np.array([10, 12, 8])
    q = r.standard_normal((B, T, Hq, D))
    kp = np.stack([np.concatenate([kc[bt[b, j]] for j in range(4)], axis=1) for b in range(B)])
    vp = np.stack([np.concatenate([vc[bt[b, j]] for j in range(4)], axis=1) for b in range(B)])
    np.testing.assert_allclose(m.decode_attention(q, kc, vc, L, 0.5, bt),
                               m.decode_attention(q, kp, vp, L, 0.5), atol=1e-14)


# ------------------------------------------------------------ sequence sharding
def pin_attend_partial_closed_forms(m):
    """One visible key: o = its v, lse2 = s / ln 2.  Two keys: lse2 = log2(e^s1 + e^s2).
    None visible: o = 0, lse2 = -inf."""
    q = np.array([[0.5, -1.0, 2.0, 0.25]])
    K = np.array([[1.0, 2.0, 0.5, -1.0], [0.0, 1.0, 1.0, 3.0], [9.0, 9.0, 9.0, 9.0]])
    V = np.array([[1.0, 2.0, 3.0, 4.0], [-1.0, 0.5, 0.0, 2.0], [7.0, 7.0, 7.0, 7.0]])
    sc = 0.7
    s1, s2 = sc * float(q[0] @ K[0]), sc * float(q[0] @ K[1])
    o, lse = m.attend_partial(q, K, V, sc, [1])
    np.testing.assert_allclose(o[0], V[0], atol=1e-15)
    assert abs(lse[0] - s1 / math.log(2)) <= 1e-14
    o, lse = m.attend_partial(q, K, V, sc, [2])
    assert abs(lse[0] - math.log2(math.exp(s1) + math.exp(s2))) <= 1e-13
    w1 = math.exp(s1) / (math.exp(s1) + math.exp(s2))
    np.testing.assert_allclose(o[0], w1 * V[0] + (1 - w1) * V[1], atol=1e-14)
    o, lse = m.attend_partial(q, K, V, sc, [0])
    assert np.all(o == 0) and lse[0] == -np.inf


def _split_cache(kc, vc, lens_total, cuts):
    """Per-shard contiguous caches holding tokens [cuts[s], cuts[s+1]) of each sequence."""
    B, Hkv, _, D = kc.shape
    shards = []
    for s in range(len(cuts) - 1):
        start = np.array([min(cuts[s], n) for n in lens_total])
        end = np.array([min(cuts[s + 1], n) for n in lens_total])
        n_loc = end - start
        cap = max(1, int(n_loc.max()))
        k_loc = np.full((B, Hkv, cap, D), np.nan)
        v_loc = np.full((B, Hkv, cap, D), np.nan)
        for b in range(B):
            k_loc[b, :, :n_loc[b]] = kc[b, :, start[b]:end[b]]
            v_loc[b, :, :n_loc[b]] = vc[b, :, start[b]:end[b]]
        shards.append((k_loc, v_loc, start, n_loc))
    return shards


def pin_shard_merge_equals_full_decode(m):
    """Any cut of each sequence's keys into shards (empty shards and a shard of
    new tokens only included), computed shard by shard and merged, equals the
    unsharded decode; a single shard gives it directly with the brute-force
    log-sum-exp."""
    r = rng(15)
    B, T, Hq, Hkv, D = 3, 3, 4, 2, 8
    L = np.array([11, 4, 20])
    N = L + T
    q = r.standard_normal((B, T, Hq, D))
    kc = r.standard_normal((B, Hkv, N.max() + 2, D))
    vc = r.standard_normal((B, Hkv, N.max() + 2, D))
    ref = m.decode_attention(q, kc, vc, L, 0.4)
    for cuts in ([0, 30], [0, 5, 12, 30], [0, 0, 9, 9, 21, 22, 30], [0, 4, 5, 6, 7, 30]):
        parts = [m.decode_attention_shard(q, k_loc, v_loc, L, start, n_loc, 0.4)
                 for (k_loc, v_loc, start, n_loc) in _split_cache(kc, vc, N, cuts)]
        got = m.merge_partials([p[0] for p in parts], [p[1] for p in parts])
        assert np.max(np.abs(got - ref)) <= 1e-12, cuts
    # one shard: lse equals the brute-force log2-sum-exp of the visible scores
    o, lse = m.decode_attention_shard(q, kc, vc, L, np.zeros(B, int), N, 0.4)
    b, i, h = 2, 1, 3
    sc = [0.4 * float(q[b, i, h] @ kc[b, h // 2, t]) for t in range(L[b] + i + 1)]
    assert abs(lse[b, i, h] - math.log2(sum(math.exp(x) for x in sc))) <= 1e-12
    np.testing.assert_allclose(o, ref, atol=1e-12)


def pin_shard_paged_equals_contiguous(m):
    """A shard's paged cache (any page permutation) gives its contiguous result."""
    r = rng(16)
    B, T, Hq, Hkv, D, P = 2, 2, 4, 1, 8, 4
    start = np.array([8, 3])
    n_loc = np.array([9, 6])
    L = np.array([15, 7])
    q = r.standard_normal((B, T, Hq, D))
    kc = r.standard_normal((B, Hkv, 12, D))
    vc = r.standard_normal((B, Hkv, 12, D))
    a = m.decode_attention_shard(q, kc, vc, L, start, n_loc, 0.3)
    pages = 3
    perm = r.permutation(B * pages)
    bt = perm.reshape(B, pages)
    kp = np.full((B * pages, Hkv, P, D), np.nan)
    vp = kp.copy()
    for b in range(B):
        for t in range(12):
            kp[bt[b, t // P], :, t % P] = kc[b, :, t]
            vp[bt[b, t // P], :, t % P] = vc[b, :, t]
    b_ = m.decode_attention_shard(q, kp, vp, L, start, n_loc, 0.3, bt)
    np.testing.assert_allclose(a[0], b_[0], atol=1e-14)
    np.testing.assert_allclose(a[1], b_[1], atol=1e-14)


# ------------------------------------------------------------- the comparator
def pin_max_abs_diff_hand_cases(m):
    """The exactness measure of generate.rs ``run`` (max |cached - recompute|)
    on hand-computed cases: the largest difference wins whatever its sign or
    position, a difference is never averaged, NaN is never skipped (a NaN in a
    result must fail every ``<= tol`` check), equal arrays differ by exactly 0,
    empty arrays by 0, and arrays of different shapes are refused rather than
    broadcast."""
    assert m.max_abs_diff([1.0, -3.0], [0.0, 0.0]) == 3.0
    assert m.max_abs_diff([0.0], [-2.0]) == 2.0
    assert m.max_abs_diff([-5.0, 1.0], [0.0, 0.0]) == 5.0       # a negative difference dominates
    assert m.max_abs_diff([[0.0, 0.0], [0.0, 7.5]], np.zeros((2, 2))) == 7.5
    # one large difference among many small ones: max, not mean or sum
    a = np.zeros(1000)
    a[637] = 0.25
    assert m.max_abs_diff(a, np.zeros(1000)) == 0.25
    b = np.full(1000, 1e-3)
    assert m.max_abs_diff(b, np.zeros(1000)) == 1e-3
    x = np.linspace(-4.0, 4.0, 33)
    assert m.max_abs_diff(x, x) == 0.0
    assert m.max_abs_diff(np.zeros(0), np.zeros(0)) == 0.0
    assert math.isnan(m.max_abs_diff([0.0, float("nan")], [0.0, 0.0]))
    assert math.isnan(m.max_abs_diff([1.0], [float("nan")]))
    assert not (m.max_abs_diff([float("nan"), 0.0], [0.0, 0.0]) <= 2e-3)
    try:
        m.max_abs_diff(np.zeros((4, 1)), np.zeros(4))
    except ValueError:
        pass
    else:
        raise AssertionError("max_abs_diff broadcast arrays of different shapes")


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
