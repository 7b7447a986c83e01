"""Plain fp64 CPU oracle for the KV-cache decode step with RoPE.

TEST INFRASTRUCTURE.  Only the test suite, ``__graft_entry__.smoke()`` and the
bench's CPU-baseline / reference leg may import or call this module.  The
product path (the CUDA library and its Python binding) never touches it and
shares no code with it.

What is computed follows ferric-core 0.1.0 ``examples/generate.rs``:

* module doc comment ("Autoregressive generation with a KV cache"): each decode
  step projects only the new token, rotates it with RoPE at its absolute
  position, appends its K/V to the per-layer cache and attends the query
  against the whole cache; the result must equal a full non-cached recompute;
* ``step_gpu``: ``rope_off_t(x, 1, h, dh, base, pos)`` on the new q and k, v
  left unrotated, ``kc.extend`` / ``vc.extend`` (append), then
  ``mha_decode_t(q1, kc, vc, h, h, dh, s)`` over all ``s`` cached tokens;
* ``layer_cpu`` / ``forward_cpu`` (the non-cached reference): ``cpu::rope`` at
  positions 0..t-1 and ``cpu::mha_causal`` over all t tokens, last row kept;
* ``run``: the exactness check (max abs difference of cached decode vs full
  recompute below 2e-3).

Grouped-query heads follow ferrox-models' ``decoder`` (GQA attention with
RoPE) and the separate q-head / kv-head counts in ``mha_decode_t``'s signature.

Readings where the pages are silent (each also listed in the design notes):

* RoPE pairing is half-split: element j pairs with j + D/2 (Llama-style, as the
  example calls its model), rotation (a, b) -> (a cos t - b sin t,
  a sin t + b cos t), angle t = pos * base^(-2j/D), j < D/2, over the full
  head dimension.
* ``seq_lens[b]`` = tokens cached before the step; the q_len new tokens sit at
  positions L_b .. L_b+q_len-1; new token i sees positions <= L_b + i.
* q head h reads kv head h // (Hq/Hkv).
* Stored values are rounded to the storage dtype (bf16: round to nearest,
  ties to even); the rotated q is rounded to the q dtype before attention.

All arithmetic is fp64 on the values as stored.  Layouts match the library's:
q ``[B, T, Hq, D]``; k_new/v_new ``[B, T, Hkv, D]``; contiguous cache
``[B, Hkv, capacity, D]``; paged cache ``[num_pages, Hkv, P, D]`` with
``block_table [B, max_pages]``.
"""
from __future__ import annotations

import math

import numpy as np

F64 = np.float64


# ----------------------------------------------------------------------------
# bfloat16 rounding, from the format's definition: 1 sign bit, 8 exponent bits
# (bias 127), 7 stored mantissa bits -- an IEEE-754 binary32 keeping only its
# top 16 bits.  A binade [2^(e-1), 2^e) therefore holds 128 values spaced
# 2^(e-8); below the smallest normal 2^-126 the spacing stays 2^-133.
# ----------------------------------------------------------------------------
def bf16_round(x) -> np.ndarray:
    """Round fp64 values to the nearest bfloat16 value (ties to even), as fp64.

    Overflow past the largest finite bfloat16 gives +-inf; NaN, inf and signed
    zeros pass through.
    """
    x = np.asarray(x, dtype=F64)
    out = x.copy()
    sel = np.isfinite(x) & (x != 0.0)
    v = x[sel]
    _, e = np.frexp(v)                       # v = m * 2^e, 0.5 <= |m| < 1
    spacing = np.maximum(e - 8, -133)        # exponent of the bf16 grid spacing
    r = np.ldexp(np.rint(np.ldexp(v, -spacing)), spacing)   # rint: half to even
    r = np.where(np.abs(r) >= 2.0 ** 128, np.copysign(np.inf, v), r)
    out[sel] = r
    return out


def round_store(x, dtype: str) -> np.ndarray:
    """Value as held in a buffer of ``dtype`` ("bf16" or "f32")."""
    x = np.asarray(x, dtype=F64)
    if dtype == "bf16":
        return bf16_round(x)
    if dtype == "f32":
        return x.astype(np.float32).astype(F64)   # IEEE binary32, round to nearest even
    raise ValueError(dtype)


# ----------------------------------------------------------------------------
# RoPE (ferric-core generate.rs, `rope_off_t` in `step_gpu`, `cpu::rope` in
# `layer_cpu`): rotate each (j, j + D/2) pair by pos * theta_j.  The layout
# variants (the ferrox-models index exports a `RopeLayout` type but defines no
# member) are read as the two common ones: interleaved pairs (2j, 2j + 1), and a
# rotary dimension r < D where only the first r elements rotate, with
# theta_j = base^(-2j/r), and the other D - r pass through unchanged.
# ----------------------------------------------------------------------------
def rope_inv_freq(head_dim: int, base: float) -> np.ndarray:
    """theta_j = base^(-2j/D) for j = 0 .. D/2-1 (D = the rotated width)."""
    j = np.arange(head_dim // 2, dtype=F64)
    return np.power(F64(base), -2.0 * j / head_dim)


def rope(x, positions, base: float, interleaved: bool = False, rotary_dim: int = 0) -> np.ndarray:
    """Rotate the last axis of ``x`` (length D) at the given absolute positions.

    ``positions`` broadcasts against ``x.shape[:-1]``.  ``interleaved`` pairs
    elements (2j, 2j + 1) instead of (j, j + r/2); ``rotary_dim`` = r (0 means
    D) rotates the first r elements only.
    """
    x = np.asarray(x, dtype=F64)
    D = x.shape[-1]
    r = D if not rotary_dim else int(rotary_dim)
    half = r // 2
    pos = np.asarray(positions, dtype=F64)
    ang = pos[..., None] * rope_inv_freq(r, base)      # [..., r/2]
    c, s = np.cos(ang), np.sin(ang)
    if interleaved:
        a, b = x[..., 0:r:2], x[..., 1:r:2]
    else:
        a, b = x[..., :half], x[..., half:r]
    ra, rb = a * c - b * s, a * s + b * c
    out = x.copy()
    if interleaved:
        out[..., 0:r:2], out[..., 1:r:2] = ra, rb
    else:
        out[..., :half], out[..., half:r] = ra, rb
    return out


# ----------------------------------------------------------------------------
# Append (generate.rs `step_gpu`: rope the new q and k, `kc.extend(knew)`,
# `vc.extend(vnew)`), into the library's contiguous or paged cache layout.
# ----------------------------------------------------------------------------
def _slot(b, p, cache_shape, block_table, page_size):
    """(index tuple prefix) of position p of sequence b: contiguous -> (b, p);
    paged -> (page, p % P)."""
    if block_table is None:
        return b, p
    return int(block_table[b, p // page_size]), p % page_size


def rotate_new_tokens(q, k_new, v_new, seq_lens, base: float, dtype: str,
                      interleaved: bool = False, rotary_dim: int = 0):
    """q and k of the new tokens rotated at positions seq_lens[b] + i, and v,
    each rounded to the storage dtype: ``(q_rot, k_rot, v_stored)``."""
    q = np.asarray(q, F64)
    T = q.shape[1]
    pos = np.asarray(seq_lens, dtype=np.int64)[:, None] + np.arange(T)[None, :]  # [B, T]
    q_rot = round_store(rope(q, pos[:, :, None], base, interleaved, rotary_dim), dtype)
    k_rot = round_store(rope(np.asarray(k_new, F64), pos[:, :, None], base, interleaved, rotary_dim),
                        dtype)
    v_st = round_store(np.asarray(v_new, F64), dtype)
    return q_rot, k_rot, v_st


def append_rope(q, k_new, v_new, k_cache, v_cache, seq_lens, base: float,
                dtype: str, block_table=None, interleaved: bool = False, rotary_dim: int = 0,
                cow_src=None):
    """Rotate q and k_new at positions seq_lens[b] + i, store k and v.

    Returns ``(q_rot, k_cache, v_cache)`` as new fp64 arrays; q_rot and the
    stored entries are rounded to ``dtype``.  Positions outside the cache are
    a caller error (IndexError).

    Shared-prefix pages (the ferrox-models index's `prefix_cache`: sequences
    that share a leading run of tokens share its pages): with ``cow_src``
    (paged only), sequence b with cow_src[b] >= 0 first gets slots
    0 .. seq_lens[b] % P - 1 of every kv head of page cow_src[b] copied, k and
    v, into its own page block_table[b, seq_lens[b] // P] (copy on write of the
    boundary page it shared); the source page is not modified.
    """
    q = np.asarray(q, F64)
    k_new = np.asarray(k_new, F64)
    v_new = np.asarray(v_new, F64)
    kc = np.array(k_cache, dtype=F64, copy=True)
    vc = np.array(v_cache, dtype=F64, copy=True)
    B, T = q.shape[0], q.shape[1]
    Hkv = k_new.shape[2]
    page_size = kc.shape[2] if block_table is not None else None
    pos = np.asarray(seq_lens, dtype=np.int64)[:, None] + np.arange(T)[None, :]  # [B, T]
    q_rot, k_rot, v_st = rotate_new_tokens(q, k_new, v_new, seq_lens, base, dtype,
                                           interleaved, rotary_dim)
    if cow_src is not None:
        for b in range(B):
            src = int(cow_src[b])
            n = int(seq_lens[b]) % page_size
            if src < 0 or n == 0:
                continue
            dst = int(block_table[b, int(seq_lens[b]) // page_size])
            kc[dst, :, :n] = kc[src, :, :n]
            vc[dst, :, :n] = vc[src, :, :n]
    for b in range(B):
        for i in range(T):
            p = int(pos[b, i])
            if block_table is None:
                kc[b, :, p, :] = k_rot[b, i]
                vc[b, :, p, :] = v_st[b, i]
            else:
                page, slot = _slot(b, p, kc.shape, block_table, page_size)
                if page < 0:
                    raise IndexError("unallocated page")
                kc[page, :, slot, :] = k_rot[b, i]
                vc[page, :, slot, :] = v_st[b, i]
    return q_rot, kc, vc


# ----------------------------------------------------------------------------
# Attention (generate.rs `mha_decode_t` and `cpu::mha_causal`): softmax of
# scale * q.k over the visible keys, weights applied to v.
# ----------------------------------------------------------------------------
def attend(q_rows, K, V, scale: float, visible) -> np.ndarray:
    """Rows ``q_rows [R, D]`` against ``K, V [N, D]``; row r sees keys
    0 .. visible[r]-1.  Plain definition: s = scale * q K^T, masked keys get
    -inf, out = softmax(s) V (max subtracted before exp, a no-op in exact
    arithmetic)."""
    q_rows = np.asarray(q_rows, F64)
    K = np.asarray(K, F64)
    V = np.asarray(V, F64)
    s = F64(scale) * (q_rows @ K.T)                       # [R, N]
    t = np.arange(K.shape[0])[None, :]
    s = np.where(t < np.asarray(visible)[:, None], s, -np.inf)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=1, keepdims=True)
    return p @ V


def gather_tokens(cache, b: int, h: int, n: int, block_table=None) -> np.ndarray:
    """Tokens 0..n-1 of sequence b, kv head h, from either cache layout."""
    cache = np.asarray(cache)
    if block_table is None:
        return np.asarray(cache[b, h, :n], F64)
    P = cache.shape[2]
    t = np.arange(n)
    pages = np.asarray(block_table)[b, t // P].astype(np.int64)
    return np.asarray(cache[pages, h, t % P], F64)


def decode_attention_rows(q_rot, k_cache, v_cache, seq_lens, scale: float, b: int,
                          heads, block_table=None) -> np.ndarray:
    """Decode output for sequence b and the listed q heads: ``[T, len(heads), D]``.

    Each q head h reads kv head h // g; new token i sees the L_b + i + 1
    positions 0 .. L_b + i.
    """
    q_rot = np.asarray(q_rot)
    T, Hq, D = q_rot.shape[1], q_rot.shape[2], q_rot.shape[3]
    Hkv = k_cache.shape[1]
    g = Hq // Hkv
    L = int(seq_lens[b])
    N = L + T
    out = np.empty((T, len(heads), D), F64)
    by_kv = {}
    for j, h in enumerate(heads):
        by_kv.setdefault(h // g, []).append((j, h))
    for hk, hs in by_kv.items():
        K = gather_tokens(k_cache, b, hk, N, block_table)
        V = gather_tokens(v_cache, b, hk, N, block_table)
        for (j, h) in hs:
            out[:, j] = attend(np.asarray(q_rot[b, :, h], F64), K, V, scale,
                               L + np.arange(T) + 1)
    return out


def decode_attention(q_rot, k_cache, v_cache, seq_lens, scale: float,
                     block_table=None) -> np.ndarray:
    """Full decode output ``[B, T, Hq, D]`` (fp64)."""
    q_rot = np.asarray(q_rot)
    B, T, Hq, D = q_rot.shape
    out = np.empty((B, T, Hq, D), F64)
    for b in range(B):
        out[b] = decode_attention_rows(q_rot, k_cache, v_cache, seq_lens, scale, b,
                                       list(range(Hq)), block_table)
    return out


# ----------------------------------------------------------------------------
# Sequence-sharded decode: the split-K of "Flash Decoding" (ferrum-sampler 0.7.0
# README, Key Optimizations) with the key ranges held by different devices.
# Each shard returns, per query row, the attention over its own keys,
# normalised, and the log-sum-exp of their scores; the merge weights shard s
# by 2^(lse_s - max) and renormalises.  Log-sum-exps are in base 2, the unit
# the kernels keep.
# ----------------------------------------------------------------------------
LN2 = math.log(2.0)


def attend_partial(q_rows, K, V, scale: float, visible):
    """Rows ``q_rows [R, D]`` against the first ``visible[r]`` keys of ``K, V
    [N, D]``: ``(o [R, D], lse2 [R])`` with o the softmax-weighted mean of V
    over those keys (0 when there are none) and lse2 = log2 sum_t exp(s_t),
    s = scale q.k (-inf when there are none)."""
    q_rows = np.asarray(q_rows, F64)
    K = np.asarray(K, F64)
    V = np.asarray(V, F64)
    R, D = q_rows.shape
    vis = np.asarray(visible)
    o = np.zeros((R, D), F64)
    lse = np.full(R, -np.inf)
    if K.shape[0] == 0:
        return o, lse
    s = F64(scale) * (q_rows @ K.T)
    t = np.arange(K.shape[0])[None, :]
    s = np.where(t < vis[:, None], s, -np.inf)
    for r in range(R):
        if vis[r] <= 0:
            continue
        m = s[r].max()
        p = np.exp(s[r] - m)
        l = p.sum()
        o[r] = (p @ V) / l
        lse[r] = (m + math.log(l)) / LN2
    return o, lse


def decode_attention_shard(q_rot, k_local, v_local, seq_lens, shard_start, shard_lens,
                           scale: float, block_table=None):
    """One shard of a sequence-sharded decode step: ``(o [B, T, Hq, D],
    lse2 [B, T, Hq])``.

    The shard's cache holds, for sequence b, the tokens at global positions
    shard_start[b] .. shard_start[b] + shard_lens[b] - 1 as its local tokens
    0 .. shard_lens[b] - 1 (either layout).  New token i of sequence b (global
    position seq_lens[b] + i) sees the local tokens whose global position is at
    most seq_lens[b] + i.
    """
    q_rot = np.asarray(q_rot, F64)
    B, T, Hq, D = q_rot.shape
    Hkv = k_local.shape[1]
    g = Hq // Hkv
    o = np.zeros((B, T, Hq, D), F64)
    lse = np.full((B, T, Hq), -np.inf)
    for b in range(B):
        n = int(shard_lens[b])
        vis = np.clip(int(seq_lens[b]) + np.arange(T) + 1 - int(shard_start[b]), 0, n)
        for hk in range(Hkv):
            K = gather_tokens(k_local, b, hk, n, block_table)
            V = gather_tokens(v_local, b, hk, n, block_table)
            for h in range(hk * g, (hk + 1) * g):
                o[b, :, h], lse[b, :, h] = attend_partial(q_rot[b, :, h], K, V, scale, vis)
    return o, lse


def merge_partials(o_parts, lse_parts) -> np.ndarray:
    """``o_parts [S, ..., D]``, ``lse_parts [S, ...]`` (base 2) -> the merged
    attention output ``[..., D]``: sum_s w_s o_s / sum_s w_s, w_s = 2^(lse_s - M),
    M = max_s lse_s; shards with lse = -inf weigh 0."""
    o_parts = np.asarray(o_parts, F64)
    lse_parts = np.asarray(lse_parts, F64)
    M = lse_parts.max(axis=0)
    Ms = np.where(np.isfinite(M), M, 0.0)
    w = np.where(np.isfinite(lse_parts), np.exp2(lse_parts - Ms), 0.0)
    den = w.sum(axis=0)
    num = (w[..., None] * o_parts).sum(axis=0)
    return np.where(den[..., None] > 0, num / np.where(den > 0, den, 1.0)[..., None], 0.0)


def full_causal_attention(q_raw, k_raw, v_raw, scale: float, base: float,
                          dtype: str | None = None, interleaved: bool = False,
                          rotary_dim: int = 0) -> np.ndarray:
    """Non-cached recompute over whole sequences (generate.rs `forward_cpu`).

    ``q_raw [B, N, Hq, D]``, ``k_raw / v_raw [B, N, Hkv, D]`` hold the
    unrotated tokens at positions 0..N-1.  Every token is rotated at its own
    position (rotated q and k, and v, rounded to ``dtype`` when given, as the
    cached path stores them) and causal attention runs over all N rows.
    Returns ``[B, N, Hq, D]``; the decode step corresponds to the last rows.
    """
    q_raw = np.asarray(q_raw, F64)
    k_raw = np.asarray(k_raw, F64)
    v_raw = np.asarray(v_raw, F64)
    B, N, Hq, D = q_raw.shape
    Hkv = k_raw.shape[2]
    g = Hq // Hkv
    pos = np.arange(N)[None, :, None]
    q = rope(q_raw, pos, base, interleaved, rotary_dim)
    k = rope(k_raw, pos, base, interleaved, rotary_dim)
    v = v_raw
    if dtype is not None:
        q, k, v = round_store(q, dtype), round_store(k, dtype), round_store(v, dtype)
    out = np.empty_like(q)
    visible = np.arange(N) + 1
    for b in range(B):
        for h in range(Hq):
            out[b, :, h] = attend(q[b, :, h], k[b, :, h // g], v[b, :, h // g], scale, visible)
    return out


def max_abs_diff(a, b) -> float:
    """max |a_i - b_i| over corresponding elements: the measure of the
    exactness check in generate.rs ``run``.  The two arrays must have the same
    shape (no broadcasting: every element is compared with its own
    counterpart).  A NaN anywhere makes the result NaN, so a comparison
    ``max_abs_diff(...) <= tol`` fails on it.  Empty arrays differ by 0."""
    a = np.asarray(a, F64)
    b = np.asarray(b, F64)
    if a.shape != b.shape:
        raise ValueError(f"max_abs_diff: shapes differ {a.shape} vs {b.shape}")
    return float(np.max(np.abs(a - b))) if a.size else 0.0
