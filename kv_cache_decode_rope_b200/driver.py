"""Decode-step driver: the autoregressive loop over per-layer KV caches.

This is the loop of ferric-core 0.1.0, examples/generate.rs (module doc
comment and `step_gpu`): every layer keeps its own K/V cache, the prompt is fed
through the same decode step as generated tokens ("prefill = decode"), and
each step rotates the new tokens, appends their k and v and attends the whole
cache.  As the ferrum-sampler 0.7.0 README ("Performance") describes for its
CUDA runner, the step of every layer is captured once into a CUDA graph and
replayed afterwards, which removes the per-step launch cost; inside the graph
the library's kernels chain with programmatic dependent launch.

Everything here is host-side bookkeeping around one library call per layer
(`kvd_decode_step`): buffers, the page pool, graph capture and the advance of
`seq_lens`.  The projections that produce q, k and v are outside this package;
a step takes them as inputs.
"""
from __future__ import annotations

from typing import Dict, Optional

import torch

from . import decode_step, workspace_size


class DecodeLoop:
    """Per-layer caches and the decode-step loop.

    Parameters: ``n_layers`` caches of ``capacity`` tokens for ``batch``
    sequences with ``num_heads`` / ``num_kv_heads`` heads of ``head_dim``.
    ``paged`` stores them in a pool of ``page_size``-token pages (each sequence
    gets its pages from one seeded permutation of the pool, shared by all
    layers' pools); otherwise each layer has a contiguous cache.

    ``step(q, k, v)`` takes ``q [n_layers, B, T, Hq, D]`` and
    ``k, v [n_layers, B, T, Hkv, D]`` for T new tokens of every sequence,
    runs every layer's decode step, advances ``seq_lens`` by T on the device
    and returns ``out [n_layers, B, T, Hq, D]``.  With ``graphs=True`` the
    first step of each T runs eagerly and captures a graph; later steps of the
    same T copy their inputs into the graph's buffers and replay it.
    """

    def __init__(self, *, n_layers: int, batch: int, num_heads: int, num_kv_heads: int,
                 head_dim: int, capacity: int, dtype=torch.bfloat16, out_dtype=None,
                 paged: bool = False, page_size: int = 16, rope_base: float = 10000.0,
                 scale: Optional[float] = None, interleaved: bool = False, rotary_dim: int = 0,
                 graphs: bool = True, device="cuda", seed: int = 0):
        self.L, self.B, self.Hq, self.Hkv, self.D = n_layers, batch, num_heads, num_kv_heads, head_dim
        self.capacity = capacity
        self.dtype = dtype
        self.out_dtype = out_dtype or dtype
        self.rope_base, self.interleaved, self.rotary_dim = rope_base, interleaved, rotary_dim
        self.scale = scale if scale is not None else head_dim ** -0.5
        self.graphs = graphs
        self.device = torch.device(device)
        if paged:
            pages_per_seq = (capacity + page_size - 1) // page_size
            n_pages = batch * pages_per_seq
            gen = torch.Generator().manual_seed(seed)
            perm = torch.randperm(n_pages, generator=gen).to(torch.int32)
            self.block_table = perm.view(batch, pages_per_seq).to(self.device)
            shape = (n_pages, num_kv_heads, page_size, head_dim)
        else:
            self.block_table = None
            shape = (batch, num_kv_heads, capacity, head_dim)
        self.k_cache = [torch.zeros(shape, dtype=dtype, device=self.device) for _ in range(n_layers)]
        self.v_cache = [torch.zeros(shape, dtype=dtype, device=self.device) for _ in range(n_layers)]
        self.seq_lens = torch.zeros(batch, dtype=torch.int32, device=self.device)
        self.length = 0                      # host copy of the (common) sequence length
        self._ws: Dict[int, torch.Tensor] = {}
        self._graph: Dict[int, tuple] = {}

    # ------------------------------------------------------------------ helpers
    def _workspace(self, T: int) -> torch.Tensor:
        if T not in self._ws:
            n = workspace_size(batch=self.B, num_heads=self.Hq, num_kv_heads=self.Hkv,
                               head_dim=self.D, q_len=T, dtype=self.dtype)
            self._ws[T] = torch.empty(max(n, 16), dtype=torch.uint8, device=self.device)
        return self._ws[T]

    def _layer_step(self, l, q, k, v, out, ws):
        decode_step(q, k, v, self.k_cache[l], self.v_cache[l], self.seq_lens, self.block_table, out,
                    scale=self.scale, max_kv_len=self.capacity, workspace=ws,
                    rope_base=self.rope_base, interleaved=self.interleaved,
                    rotary_dim=self.rotary_dim)

    def _run(self, q, k, v, out, T):
        ws = self._workspace(T)
        for l in range(self.L):
            self._layer_step(l, q[l], k[l], v[l], out[l], ws)
        self.seq_lens.add_(T)

    # --------------------------------------------------------------------- API
    def reset(self):
        """Empty every cache (the stored values stay; they are never read)."""
        self.seq_lens.zero_()
        self.length = 0

    def prefill(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor) -> torch.Tensor:
        """Feed a prompt of any length through decode steps ("prefill = decode"),
        in chunks of at most 64 query rows per (sequence, kv head), the limit
        every kernel path accepts; returns the outputs of all its tokens."""
        g = self.Hq // self.Hkv
        chunk = max(1, 64 // g)
        outs = [self.step(q[:, :, t:t + chunk], k[:, :, t:t + chunk], v[:, :, t:t + chunk])
                for t in range(0, q.shape[2], chunk)]
        return torch.cat(outs, dim=2)

    def step(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor) -> torch.Tensor:
        T = q.shape[2]
        if q.shape != (self.L, self.B, T, self.Hq, self.D):
            raise ValueError("q must be [n_layers, B, T, Hq, D]")
        if k.shape != (self.L, self.B, T, self.Hkv, self.D) or v.shape != k.shape:
            raise ValueError("k, v must be [n_layers, B, T, Hkv, D]")
        if self.length + T > self.capacity:
            raise ValueError("the step would run past the cache capacity")
        self.length += T
        if not self.graphs:
            out = torch.empty((self.L, self.B, T, self.Hq, self.D), dtype=self.out_dtype,
                              device=self.device)
            self._run(q.contiguous(), k.contiguous(), v.contiguous(), out, T)
            return out
        if T not in self._graph:
            # first step of this width: run it eagerly (which also sets the
            # kernels' one-time attributes), then capture the same calls on
            # static buffers for the later steps
            bufs = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v),
                    torch.empty((self.L, self.B, T, self.Hq, self.D), dtype=self.out_dtype,
                                device=self.device))
            out = torch.empty_like(bufs[3])
            self._run(q.contiguous(), k.contiguous(), v.contiguous(), out, T)
            torch.cuda.synchronize(self.device)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self._run(*bufs, T)
            self._graph[T] = (g, bufs)
            return out
        g, (sq, sk, sv, so) = self._graph[T]
        sq.copy_(q)
        sk.copy_(k)
        sv.copy_(v)
        g.replay()
        return so.clone()
