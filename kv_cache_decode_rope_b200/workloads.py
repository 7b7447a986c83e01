"""Seeded synthetic inputs for the KV-cache decode step.

This module draws random numbers and lays them out; it holds none of the
method's arithmetic (no RoPE, no attention, no softmax).  Both the CUDA path
(through the tests and the bench) and the CPU oracle consume the same bytes
produced here.

Workload shapes follow the serving cases the pages describe: a tiny MHA decode
shaped like the ferric-core `examples/generate.rs` example (prefill by feeding
prompt tokens through the decode step, then single-token decode), batched GQA
decode, continuous batching over a paged pool (ferrum-sampler README, "Paged KV
attention: GPU block pool with block-table indirection" and "Continuous
batching"), multi-token speculative verification (ferrox-models index,
`speculative`; ferrite's MTP speculative decoding) and long-context decode
(ferrum-sampler README, "Flash Decoding: split-K for long-context decode").

Recipe (all draws in fp32 from ``torch.Generator`` seeded per call, then
rounded to the storage dtype by torch's round-to-nearest-even cast):

* ``uniform``: q, k, v ~ U[-0.1, 0.1].
* ``normal``: q, k, v ~ N(0, 1).
* Cached tokens of configs drawn directly ("random" cache mode) are the stored
  values: keys are taken as already rotated.
* ``peaked_frac``: for every (sequence, kv head), floor(frac * L) distinct token
  indices (a seeded permutation prefix) have their keys scaled by
  ``peaked_scale`` before the dtype cast.
* Ragged lengths: L_b = floor(exp(U(ln lo, ln hi))) clamped to [lo, hi].
* Paged pool: exactly sum_b ceil((L_b + q_len) / P) pages; block-table rows are
  consecutive slices of one seeded random permutation of the page ids; unused
  block-table entries are -1.
* Cache slots not holding a drawn token are filled with ``fill`` ("nan" makes a
  stray read poison the result; "zero" is used for timing).
"""
from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass
from typing import Optional

import torch

DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    dtype: str                      # "f32" or "bf16": q, k/v new and the caches
    paged: bool
    q_len: int
    cache_len: Optional[int]        # fixed L_b for every sequence, or None for ragged
    len_range: Optional[tuple] = None   # (lo, hi) for log-uniform ragged lengths
    page_size: int = 16
    rope_base: float = 10000.0
    dist: str = "normal"            # "normal" or "uniform"
    peaked_frac: float = 0.0
    peaked_scale: float = 4.0
    cache_mode: str = "random"      # "random": draw stored cache; "prefill": draw raw prefix tokens
    config_id: int = 0
    shared_prefix: int = 0          # paged: tokens (whole pages) every sequence shares

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    @property
    def group(self) -> int:
        return self.num_heads // self.num_kv_heads

    @property
    def rows(self) -> int:
        return self.group * self.q_len

    @property
    def torch_dtype(self):
        return DTYPES[self.dtype]

    @property
    def esize(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads (ids 1..5).  Seeds: 1000 + id for timing, 0..9 for parity.
WORKLOADS = {
    "tiny_mha": Workload("tiny_mha", 1, 8, 8, 64, "f32", False, 1, 128,
                         dist="uniform", cache_mode="prefill", config_id=1),
    "batched_gqa": Workload("batched_gqa", 32, 32, 8, 128, "bf16", False, 1, 4096,
                            config_id=2),
    "paged_cb": Workload("paged_cb", 64, 64, 8, 128, "bf16", True, 1, None,
                         len_range=(16, 32768), config_id=3),
    "mtp_verify": Workload("mtp_verify", 16, 64, 4, 128, "bf16", True, 4, 8192,
                           config_id=4),
    "long_ctx": Workload("long_ctx", 4, 32, 8, 128, "bf16", False, 1, 131072,
                         peaked_frac=0.01, peaked_scale=4.0, config_id=5),
    # shared-prefix pages (prefix cache): 64 sequences over one 8192-token
    # prefix held once in the pool, each with a private suffix of 16..1024 tokens
    "shared_prefix": Workload("shared_prefix", 64, 64, 8, 128, "bf16", True, 1, None,
                              len_range=(16, 1024), shared_prefix=8192, config_id=6),
}


def round_up(x: int, m: int) -> int:
    return (x + m - 1) // m * m


def draw_lengths(w: Workload, gen: torch.Generator) -> torch.Tensor:
    """Cached lengths L_b before the step (int64 on the host)."""
    if w.cache_len is not None:
        return torch.full((w.batch,), w.cache_len, dtype=torch.int64)
    lo, hi = w.len_range
    u = torch.rand(w.batch, generator=gen, dtype=torch.float64)
    lens = torch.floor(torch.exp(math.log(lo) + u * (math.log(hi) - math.log(lo))))
    return lens.clamp(lo, hi).to(torch.int64) + w.shared_prefix


def page_table(w: Workload, lens, gen: torch.Generator):
    """Block table of a paged workload: each sequence's pages are consecutive
    slices of one seeded permutation of the pool; with a shared prefix the
    first shared_prefix / P entries of every row are the same pages.
    Returns (block_table int32 [B, max_pages], num_pages)."""
    P, T = w.page_size, w.q_len
    n_sh = w.shared_prefix // P
    own = [(int(L) + T + P - 1) // P - n_sh for L in lens]
    num_pages = n_sh + sum(own)
    perm = torch.randperm(num_pages, generator=gen).to(torch.int32)
    bt = torch.full((w.batch, n_sh + max(own)), -1, dtype=torch.int32)
    off = n_sh
    for b, n in enumerate(own):
        bt[b, :n_sh] = perm[:n_sh]
        bt[b, n_sh:n_sh + n] = perm[off:off + n]
        off += n
    return bt, num_pages


def _draw(shape, w: Workload, gen: torch.Generator) -> torch.Tensor:
    if w.dist == "uniform":
        return torch.rand(shape, generator=gen, dtype=torch.float32) * 0.2 - 0.1
    return torch.randn(shape, generator=gen, dtype=torch.float32)


def _fill_value(fill: str):
    return float("nan") if fill == "nan" else 0.0


def make_inputs(w: Workload, seed: int, fill: str = "nan") -> dict:
    """Build one decode step's inputs on the host (CPU tensors).

    Layouts: q ``[B, q_len, Hq, D]``; k_new, v_new ``[B, q_len, Hkv, D]``;
    contiguous caches ``[B, Hkv, capacity, D]``; paged caches
    ``[num_pages, Hkv, P, D]`` with ``block_table [B, max_pages_per_seq]``
    int32; ``seq_lens [B]`` int32 = tokens cached before the step.
    In "prefill" cache mode the prefix is returned raw (``q_prefix``,
    ``k_prefix``, ``v_prefix``, shaped like q/k_new/v_new with L tokens) and
    the caches hold only the fill value.
    """
    gen = torch.Generator().manual_seed(seed)
    B, Hq, Hkv, D, T = w.batch, w.num_heads, w.num_kv_heads, w.head_dim, w.q_len
    dt = w.torch_dtype
    lens = draw_lengths(w, gen)
    out = {"workload": w, "seed": seed}
    out["q"] = _draw((B, T, Hq, D), w, gen).to(dt)
    out["k_new"] = _draw((B, T, Hkv, D), w, gen).to(dt)
    out["v_new"] = _draw((B, T, Hkv, D), w, gen).to(dt)
    out["seq_lens"] = lens.to(torch.int32)
    fv = _fill_value(fill)
    P = w.page_size

    if w.paged:
        bt, num_pages = page_table(w, lens, gen)
        k_cache = torch.full((num_pages, Hkv, P, D), fv, dtype=dt)
        v_cache = torch.full((num_pages, Hkv, P, D), fv, dtype=dt)
        out["block_table"] = bt
        out["num_pages"] = num_pages
        out["max_pages_per_seq"] = bt.shape[1]
    else:
        cap = round_up(int(lens.max()) + T, 16)
        k_cache = torch.full((B, Hkv, cap, D), fv, dtype=dt)
        v_cache = torch.full((B, Hkv, cap, D), fv, dtype=dt)
        out["block_table"] = None
        out["max_seq_len"] = cap

    if w.cache_mode == "prefill":
        Lmax = int(lens.max())
        out["q_prefix"] = _draw((B, Lmax, Hq, D), w, gen).to(dt)
        out["k_prefix"] = _draw((B, Lmax, Hkv, D), w, gen).to(dt)
        out["v_prefix"] = _draw((B, Lmax, Hkv, D), w, gen).to(dt)
    else:
        for b in range(B):
            L = int(lens[b])
            t_lo = w.shared_prefix if b > 0 else 0   # the shared prefix is drawn once
            for h in range(Hkv):
                k = _draw((L - t_lo, D), w, gen)
                v = _draw((L - t_lo, D), w, gen)
                if w.peaked_frac > 0:
                    n_peak = int(math.floor(w.peaked_frac * L))
                    idx = torch.randperm(L, generator=gen)[:n_peak]
                    k[idx] *= w.peaked_scale
                k = k.to(dt)
                v = v.to(dt)
                if w.paged:
                    t = torch.arange(t_lo, L)
                    pages = out["block_table"][b, t // P].long()
                    k_cache[pages, h, t % P] = k
                    v_cache[pages, h, t % P] = v
                else:
                    k_cache[b, h, :L] = k
                    v_cache[b, h, :L] = v
    out["k_cache"] = k_cache
    out["v_cache"] = v_cache
    return out


def logical_kv(inp: dict, b: int, h: int, n: int, which: str = "k") -> torch.Tensor:
    """Tokens 0..n-1 of sequence b, kv head h, gathered from either cache layout
    (indexing only).  Returns ``[n, D]`` in the cache dtype."""
    cache = inp["k_cache"] if which == "k" else inp["v_cache"]
    bt = inp.get("block_table")
    if bt is None:
        return cache[b, h, :n]
    P = cache.shape[2]
    rows = []
    for t0 in range(0, n, P):
        page = int(bt[b, t0 // P])
        rows.append(cache[page, h, :min(P, n - t0)])
    return torch.cat(rows, 0)


def make_inputs_device(w: Workload, seed: int, device="cuda") -> dict:
    """The same layout and distributions as ``make_inputs``, drawn directly on
    the device with a seeded CUDA generator (used for timing, where copying
    gigabytes from the host would only slow set-up).  Unused cache slots are
    zero.  Lengths and the page permutation are drawn on the host as in
    ``make_inputs``."""
    hgen = torch.Generator().manual_seed(seed)
    dgen = torch.Generator(device=device).manual_seed(seed)
    B, Hq, Hkv, D, T = w.batch, w.num_heads, w.num_kv_heads, w.head_dim, w.q_len
    dt = w.torch_dtype
    lens = draw_lengths(w, hgen)

    def draw(shape):
        if w.dist == "uniform":
            return torch.rand(shape, generator=dgen, device=device) * 0.2 - 0.1
        return torch.randn(shape, generator=dgen, device=device)

    out = {"workload": w, "seed": seed, "seq_lens": lens.to(torch.int32).to(device)}
    out["q"] = draw((B, T, Hq, D)).to(dt)
    out["k_new"] = draw((B, T, Hkv, D)).to(dt)
    out["v_new"] = draw((B, T, Hkv, D)).to(dt)
    P = w.page_size
    if w.paged:
        bt, num_pages = page_table(w, lens, hgen)
        k_cache = torch.zeros((num_pages, Hkv, P, D), dtype=dt, device=device)
        v_cache = torch.zeros_like(k_cache)
        out.update(block_table=bt.to(device), num_pages=num_pages, max_pages_per_seq=bt.shape[1])
    else:
        cap = round_up(int(lens.max()) + T, 16)
        k_cache = torch.zeros((B, Hkv, cap, D), dtype=dt, device=device)
        v_cache = torch.zeros_like(k_cache)
        out.update(block_table=None, max_seq_len=cap)
    for b in range(B):
        L = int(lens[b])
        t_lo = w.shared_prefix if b > 0 else 0   # the shared prefix is drawn once
        for h in range(Hkv):
            k = draw((L - t_lo, D))
            v = draw((L - t_lo, D))
            if w.peaked_frac > 0:
                n_peak = int(math.floor(w.peaked_frac * L))
                idx = torch.randperm(L, generator=dgen, device=device)[:n_peak]
                k[idx] *= w.peaked_scale
            if w.paged:
                t = torch.arange(t_lo, L, device=device)
                pages = out["block_table"][b, t // P].long()
                k_cache[pages, h, t % P] = k.to(dt)
                v_cache[pages, h, t % P] = v.to(dt)
            else:
                k_cache[b, h, :L] = k.to(dt)
                v_cache[b, h, :L] = v.to(dt)
    out["k_cache"] = k_cache
    out["v_cache"] = v_cache
    return out


def step_bytes(w: Workload, seq_lens, out_esize: int) -> dict:
    """Algorithmic bytes one decode step must move (the unit of the GB/s
    figures).  ``decode``: every attended K and V row once, q read, out
    written.  ``append``: q read + written, k_new and v_new read, k and v
    written to the cache, the length (and page) indices read."""
    lens = [int(x) for x in seq_lens]
    B, T, Hq, Hkv, D, es = w.batch, w.q_len, w.num_heads, w.num_kv_heads, w.head_dim, w.esize
    # a shared prefix is stored once: its rows count once (the repeated reads
    # of it by every sequence are cache hits, not HBM traffic the method needs)
    sp = w.shared_prefix
    kv = (sp + sum(L + T - sp for L in lens)) * Hkv * 2 * D * es
    kv_logical = sum(L + T for L in lens) * Hkv * 2 * D * es
    q = B * T * Hq * D * es
    out = B * T * Hq * D * out_esize
    idx = B * 4
    if w.paged:
        idx += sum((L + T + w.page_size - 1) // w.page_size for L in lens) * 4
    decode = kv + q + out + idx
    append = 2 * q + 4 * B * T * Hkv * D * es + B * 4 + (B * T * 4 if w.paged else 0)
    return {"decode": decode, "append": append, "step": decode + append, "kv": kv,
            "kv_logical": kv_logical}
