"""KV-cache decode step on B200 (sm_100a): RoPE + KV append + GQA flash decode.

Python binding of ``libkvdecode.so`` (C ABI in ``include/kvdecode.h``).  The
functions here only marshal torch tensors into pointers and sizes; every step
of the computation runs in the library's CUDA kernels.  PyTorch supplies
device memory and the current CUDA stream.
"""
from __future__ import annotations

import ctypes
from typing import Optional

import torch

from . import _lib
from ._lib import KvdError, Params, get_lib  # noqa: F401

__all__ = ["append_rope", "decode_attention", "decode_attention_paged", "decode_step",
           "append_rope_cow", "append_rope_shard", "decode_attention_shard", "merge_partials",
           "workspace_size", "make_params", "KvdError", "version", "DecodeLoop"]

_DT = {torch.float32: _lib.KVD_F32, torch.bfloat16: _lib.KVD_BF16}


def _dtype_code(t: torch.dtype) -> int:
    if t not in _DT:
        raise TypeError(f"unsupported dtype {t}; use float32 or bfloat16")
    return _DT[t]


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors passed to the decode library must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors passed to the decode library must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def make_params(*, batch, num_heads, num_kv_heads, head_dim, q_len, dtype, scale=None,
                rope_base=10000.0, out_dtype=None, max_seq_len=0, page_size=0, num_pages=0,
                max_pages_per_seq=0, max_kv_len=0, status=None, rope_interleaved=False,
                rotary_dim=0) -> Params:
    """Build a ``kvd_params`` struct.  ``dtype``/``out_dtype`` are torch dtypes."""
    p = Params()
    p.batch, p.num_heads, p.num_kv_heads = batch, num_heads, num_kv_heads
    p.head_dim, p.q_len = head_dim, q_len
    p.scale = (head_dim ** -0.5) if scale is None else scale
    p.rope_base = rope_base
    p.dtype = _dtype_code(dtype)
    p.out_dtype = _dtype_code(out_dtype if out_dtype is not None else dtype)
    p.max_seq_len, p.page_size, p.num_pages = max_seq_len, page_size, num_pages
    p.max_pages_per_seq, p.max_kv_len = max_pages_per_seq, max_kv_len
    p.status = None if status is None else _ptr(status)
    p.rope_interleaved = 1 if rope_interleaved else 0
    p.rotary_dim = int(rotary_dim)
    return p


def _geometry(q, k_cache, block_table):
    B, T, Hq, D = q.shape
    if block_table is None:
        Bc, Hkv, S, Dc = k_cache.shape
        if Bc != B:
            raise ValueError("contiguous cache batch does not match q")
        paging = dict(max_seq_len=S)
    else:
        NPg, Hkv, P, Dc = k_cache.shape
        paging = dict(page_size=P, num_pages=NPg, max_pages_per_seq=block_table.shape[1])
        if block_table.dtype != torch.int32 or block_table.shape[0] != B:
            raise ValueError("block_table must be int32 [B, max_pages_per_seq]")
    if Dc != D:
        raise ValueError("cache head_dim does not match q")
    return B, T, Hq, Hkv, D, paging


def append_rope(q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor, k_cache: torch.Tensor,
                v_cache: torch.Tensor, seq_lens: torch.Tensor, block_table: Optional[torch.Tensor] = None,
                *, rope_base: float = 10000.0, status: Optional[torch.Tensor] = None,
                stream=None, interleaved: bool = False, rotary_dim: int = 0) -> None:
    """``kv_append_rope``: rotate q in place, append rotated k and v at
    positions seq_lens[b] + i.  Shapes as in include/kvdecode.h.
    ``interleaved`` pairs elements (2j, 2j + 1); ``rotary_dim`` (0 = head_dim)
    rotates the first rotary_dim elements only."""
    B, T, Hq, Hkv, D, paging = _geometry(q, k_cache, block_table)
    if k_new.shape != (B, T, Hkv, D) or v_new.shape != k_new.shape:
        raise ValueError("k_new / v_new must be [B, T, Hkv, D]")
    for t in (k_new, v_new, k_cache, v_cache):
        if t.dtype != q.dtype:
            raise TypeError("q, k_new, v_new and the caches must share one dtype")
    if seq_lens.dtype != torch.int32:
        raise TypeError("seq_lens must be int32")
    p = make_params(batch=B, num_heads=Hq, num_kv_heads=Hkv, head_dim=D, q_len=T, dtype=q.dtype,
                    rope_base=rope_base, status=status, rope_interleaved=interleaved,
                    rotary_dim=rotary_dim, **paging)
    rc = get_lib().kv_append_rope(ctypes.byref(p), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache),
                                  _ptr(v_cache), _ptr(seq_lens), _ptr(block_table), _stream(stream))
    _lib.check("kv_append_rope", rc)


def workspace_size(*, batch, num_heads, num_kv_heads, head_dim, q_len, dtype=torch.bfloat16) -> int:
    p = make_params(batch=batch, num_heads=num_heads, num_kv_heads=num_kv_heads, head_dim=head_dim,
                    q_len=q_len, dtype=dtype)
    return int(get_lib().kvd_workspace_size(ctypes.byref(p)))


def _decode(q, k_cache, v_cache, seq_lens, block_table, out, *, scale, max_kv_len, workspace,
            out_dtype, status, stream):
    B, T, Hq, Hkv, D, paging = _geometry(q, k_cache, block_table)
    if k_cache.dtype != q.dtype or v_cache.dtype != q.dtype or v_cache.shape != k_cache.shape:
        raise TypeError("q and the caches must share dtype; k_cache and v_cache one shape")
    if seq_lens.dtype != torch.int32:
        raise TypeError("seq_lens must be int32")
    out_dtype = out.dtype if out is not None else (out_dtype or q.dtype)
    if out is None:
        out = torch.empty((B, T, Hq, D), dtype=out_dtype, device=q.device)
    elif out.shape != (B, T, Hq, D):
        raise ValueError("out must be [B, T, Hq, D]")
    if max_kv_len is None:
        cap = paging.get("max_seq_len") or paging["page_size"] * paging["max_pages_per_seq"]
        max_kv_len = cap
    p = make_params(batch=B, num_heads=Hq, num_kv_heads=Hkv, head_dim=D, q_len=T, dtype=q.dtype,
                    scale=scale, out_dtype=out_dtype, max_kv_len=max_kv_len, status=status, **paging)
    lib = get_lib()
    need = int(lib.kvd_workspace_size(ctypes.byref(p)))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    nbytes = workspace.numel() * workspace.element_size()
    if block_table is None:
        rc = lib.decode_attention(ctypes.byref(p), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                  _ptr(seq_lens), _ptr(out), _ptr(workspace), nbytes, _stream(stream))
        _lib.check("decode_attention", rc)
    else:
        rc = lib.decode_attention_paged(ctypes.byref(p), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                        _ptr(seq_lens), _ptr(block_table), _ptr(out), _ptr(workspace),
                                        nbytes, _stream(stream))
        _lib.check("decode_attention_paged", rc)
    return out


def decode_attention(q, k_cache, v_cache, seq_lens, out=None, *, scale=None, max_kv_len=None,
                     workspace=None, out_dtype=None, status=None, stream=None) -> torch.Tensor:
    """``decode_attention`` over the contiguous cache ``[B, Hkv, S, D]``."""
    return _decode(q, k_cache, v_cache, seq_lens, None, out, scale=scale, max_kv_len=max_kv_len,
                   workspace=workspace, out_dtype=out_dtype, status=status, stream=stream)


def decode_attention_paged(q, k_cache, v_cache, seq_lens, block_table, out=None, *, scale=None,
                           max_kv_len=None, workspace=None, out_dtype=None, status=None,
                           stream=None) -> torch.Tensor:
    """``decode_attention_paged`` over the paged cache ``[num_pages, Hkv, P, D]``."""
    if block_table is None:
        raise ValueError("decode_attention_paged needs a block_table")
    return _decode(q, k_cache, v_cache, seq_lens, block_table, out, scale=scale,
                   max_kv_len=max_kv_len, workspace=workspace, out_dtype=out_dtype, status=status,
                   stream=stream)


def decode_step(q, k_new, v_new, k_cache, v_cache, seq_lens, block_table=None, out=None, *,
                scale=None, max_kv_len=None, workspace=None, out_dtype=None, rope_base=10000.0,
                interleaved=False, rotary_dim=0, status=None, stream=None) -> torch.Tensor:
    """``kvd_decode_step``: append_rope then decode_attention[_paged] in one
    library call (seq_lens is not advanced)."""
    B, T, Hq, Hkv, D, paging = _geometry(q, k_cache, block_table)
    if k_new.shape != (B, T, Hkv, D) or v_new.shape != k_new.shape:
        raise ValueError("k_new / v_new must be [B, T, Hkv, D]")
    for t in (k_new, v_new, k_cache, v_cache):
        if t.dtype != q.dtype:
            raise TypeError("q, k_new, v_new and the caches must share one dtype")
    if seq_lens.dtype != torch.int32:
        raise TypeError("seq_lens must be int32")
    out_dtype = out.dtype if out is not None else (out_dtype or q.dtype)
    if out is None:
        out = torch.empty((B, T, Hq, D), dtype=out_dtype, device=q.device)
    elif out.shape != (B, T, Hq, D):
        raise ValueError("out must be [B, T, Hq, D]")
    if max_kv_len is None:
        max_kv_len = paging.get("max_seq_len") or paging["page_size"] * paging["max_pages_per_seq"]
    p = make_params(batch=B, num_heads=Hq, num_kv_heads=Hkv, head_dim=D, q_len=T, dtype=q.dtype,
                    scale=scale, out_dtype=out_dtype, max_kv_len=max_kv_len, status=status,
                    rope_base=rope_base, rope_interleaved=interleaved, rotary_dim=rotary_dim,
                    **paging)
    lib = get_lib()
    if workspace is None:
        need = int(lib.kvd_workspace_size(ctypes.byref(p)))
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    nbytes = workspace.numel() * workspace.element_size()
    rc = lib.kvd_decode_step(ctypes.byref(p), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache),
                             _ptr(v_cache), _ptr(seq_lens), _ptr(block_table), _ptr(out),
                             _ptr(workspace), nbytes, _stream(stream))
    _lib.check("kvd_decode_step", rc)
    return out


def append_rope_cow(q, k_new, v_new, k_cache, v_cache, seq_lens, block_table, cow_src, *,
                    rope_base: float = 10000.0, interleaved: bool = False, rotary_dim: int = 0,
                    status=None, stream=None) -> None:
    """``kv_append_rope_cow``: append_rope on a paged cache, first copying the
    slots before seq_lens[b] of shared page cow_src[b] (>= 0) into the
    sequence's own page block_table[b, seq_lens[b] // page_size]."""
    if cow_src.dtype != torch.int32:
        raise TypeError("cow_src must be int32")
    B, T, Hq, Hkv, D, paging = _geometry(q, k_cache, block_table)
    p = make_params(batch=B, num_heads=Hq, num_kv_heads=Hkv, head_dim=D, q_len=T, dtype=q.dtype,
                    rope_base=rope_base, status=status, rope_interleaved=interleaved,
                    rotary_dim=rotary_dim, **paging)
    rc = get_lib().kv_append_rope_cow(ctypes.byref(p), _ptr(q), _ptr(k_new), _ptr(v_new),
                                      _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens),
                                      _ptr(block_table), _ptr(cow_src), _stream(stream))
    _lib.check("kv_append_rope_cow", rc)


def append_rope_shard(q, k_new, v_new, k_cache, v_cache, seq_lens, shard_start, block_table=None,
                      *, rope_base: float = 10000.0, interleaved: bool = False, rotary_dim: int = 0,
                      status=None, stream=None) -> None:
    """``kv_append_rope_shard``: rotate q (and k) at the global positions
    seq_lens[b] + i and store k, v at local slot seq_lens[b] + i - shard_start[b]
    when the shard holds it.  ``k_cache = v_cache = None`` rotates q only."""
    if shard_start.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise TypeError("seq_lens and shard_start must be int32")
    rotate_only = k_cache is None and v_cache is None
    B, T, Hq, D = q.shape
    if rotate_only:
        Hkv = k_new.shape[2] if k_new is not None else Hq
        paging = dict(max_seq_len=1)
        if block_table is not None:
            raise ValueError("rotate-only mode takes no block_table")
    else:
        B, T, Hq, Hkv, D, paging = _geometry(q, k_cache, block_table)
    p = make_params(batch=B, num_heads=Hq, num_kv_heads=Hkv, head_dim=D, q_len=T, dtype=q.dtype,
                    rope_base=rope_base, status=status, rope_interleaved=interleaved,
                    rotary_dim=rotary_dim, **paging)
    rc = get_lib().kv_append_rope_shard(
        ctypes.byref(p), _ptr(q), None if rotate_only else _ptr(k_new),
        None if rotate_only else _ptr(v_new), None if rotate_only else _ptr(k_cache),
        None if rotate_only else _ptr(v_cache), _ptr(seq_lens), _ptr(shard_start),
        _ptr(block_table), _stream(stream))
    _lib.check("kv_append_rope_shard", rc)


def decode_attention_shard(q, k_cache, v_cache, seq_lens, shard_start, shard_lens, block_table=None,
                           *, scale=None, max_kv_len=None, workspace=None, out=None, out_lse=None,
                           status=None, stream=None):
    """``decode_attention_shard``: this shard's (o [B,T,Hq,D] fp32, lse2 [B,T,Hq]
    fp32) over its tokens of each sequence."""
    B, T, Hq, Hkv, D, paging = _geometry(q, k_cache, block_table)
    for t in (seq_lens, shard_start, shard_lens):
        if t.dtype != torch.int32:
            raise TypeError("seq_lens, shard_start and shard_lens must be int32")
    if out is None:
        out = torch.empty((B, T, Hq, D), dtype=torch.float32, device=q.device)
    if out_lse is None:
        out_lse = torch.empty((B, T, Hq), dtype=torch.float32, device=q.device)
    if max_kv_len is None:
        max_kv_len = paging.get("max_seq_len") or paging["page_size"] * paging["max_pages_per_seq"]
    p = make_params(batch=B, num_heads=Hq, num_kv_heads=Hkv, head_dim=D, q_len=T, dtype=q.dtype,
                    scale=scale, out_dtype=torch.float32, max_kv_len=max_kv_len, status=status,
                    **paging)
    lib = get_lib()
    if workspace is None:
        need = int(lib.kvd_workspace_size(ctypes.byref(p)))
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    nbytes = workspace.numel() * workspace.element_size()
    rc = lib.decode_attention_shard(ctypes.byref(p), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                    _ptr(seq_lens), _ptr(shard_start), _ptr(shard_lens),
                                    _ptr(block_table), _ptr(out), _ptr(out_lse), _ptr(workspace),
                                    nbytes, _stream(stream))
    _lib.check("decode_attention_shard", rc)
    return out, out_lse


def merge_partials(part_o, part_lse, out=None, *, out_dtype=None, stream=None) -> torch.Tensor:
    """``kvd_merge_partials``: part_o [S,B,T,Hq,D] fp32, part_lse [S,B,T,Hq] fp32
    -> the merged attention output [B,T,Hq,D]."""
    S, B, T, Hq, D = part_o.shape
    if part_lse.shape != (S, B, T, Hq) or part_o.dtype != torch.float32 \
            or part_lse.dtype != torch.float32:
        raise ValueError("part_o [S,B,T,Hq,D] and part_lse [S,B,T,Hq], both fp32")
    out_dtype = out.dtype if out is not None else (out_dtype or torch.float32)
    if out is None:
        out = torch.empty((B, T, Hq, D), dtype=out_dtype, device=part_o.device)
    p = make_params(batch=B, num_heads=Hq, num_kv_heads=Hq, head_dim=D, q_len=T,
                    dtype=torch.float32, out_dtype=out_dtype)
    rc = get_lib().kvd_merge_partials(ctypes.byref(p), _ptr(part_o), _ptr(part_lse), S, _ptr(out),
                                      _stream(stream))
    _lib.check("kvd_merge_partials", rc)
    return out


def version() -> int:
    return int(get_lib().kvd_version())


from .driver import DecodeLoop  # noqa: E402  (uses decode_step above)
