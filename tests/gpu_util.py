"""Helpers for the GPU parity tests: run one decode step through the library's
C ABI (via the binding), and run the same step through the fp64 oracle."""
from __future__ import annotations

import numpy as np
import torch

import kv_cache_decode_rope_b200 as kvd
import oracle

BF16_TOL = 2e-3     # max |gpu - oracle| with bf16 inputs (the exactness bound of generate.rs `run`)
F32_TOL = 1e-5      # fp32 inputs


def log_error(tag: str, value: float) -> None:
    """Append a measured error to $KVD_ERROR_LOG (if set) for the design notes."""
    import os
    path = os.environ.get("KVD_ERROR_LOG")
    if path:
        with open(path, "a") as f:
            f.write(f"{tag}\t{value:.3e}\n")


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().float().numpy().astype(np.float64)


def tol_for(w) -> float:
    return F32_TOL if w.dtype == "f32" else BF16_TOL


def to_device(inp: dict) -> dict:
    d = {}
    for k in ("q", "k_new", "v_new", "k_cache", "v_cache", "seq_lens", "block_table"):
        v = inp.get(k)
        d[k] = None if v is None else v.cuda()
    return d


def max_kv_len(inp: dict) -> int:
    return int(inp["seq_lens"].max()) + inp["workload"].q_len


def gpu_append(inp: dict, d: dict, status=None) -> None:
    w = inp["workload"]
    kvd.append_rope(d["q"], d["k_new"], d["v_new"], d["k_cache"], d["v_cache"], d["seq_lens"],
                    d["block_table"], rope_base=w.rope_base, status=status)


def gpu_decode(inp: dict, d: dict, out_dtype=torch.float32, status=None, mkl=None):
    w = inp["workload"]
    mkl = mkl or max_kv_len(inp)
    if d["block_table"] is None:
        return kvd.decode_attention(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"], scale=w.scale,
                                    max_kv_len=mkl, out_dtype=out_dtype, status=status)
    return kvd.decode_attention_paged(d["q"], d["k_cache"], d["v_cache"], d["seq_lens"],
                                      d["block_table"], scale=w.scale, max_kv_len=mkl,
                                      out_dtype=out_dtype, status=status)


def gpu_step(inp: dict, out_dtype=torch.float32, status=None):
    d = to_device(inp)
    gpu_append(inp, d, status)
    out = gpu_decode(inp, d, out_dtype, status)
    torch.cuda.synchronize()
    return d, out


def oracle_step(inp: dict):
    """Oracle append + decode on the host copy of the same inputs (fp64)."""
    w = inp["workload"]
    bt = None if inp["block_table"] is None else inp["block_table"].numpy()
    q_rot, kc, vc = oracle.append_rope(np64(inp["q"]), np64(inp["k_new"]), np64(inp["v_new"]),
                                       np64(inp["k_cache"]), np64(inp["v_cache"]),
                                       inp["seq_lens"].numpy(), w.rope_base, w.dtype, bt)
    out = oracle.decode_attention(q_rot, kc, vc, inp["seq_lens"].numpy(), w.scale, bt)
    return q_rot, kc, vc, out


def oracle_rows(inp: dict, samples):
    """Oracle outputs for sampled (b, i, h) rows of a step, built without
    copying the whole cache: the unit's cached prefix (host bytes from the
    generator) followed by the oracle-rotated new tokens."""
    w = inp["workload"]
    q_rot, k_rot, v_st = oracle.rotate_new_tokens(np64(inp["q"]), np64(inp["k_new"]),
                                                  np64(inp["v_new"]), inp["seq_lens"].numpy(),
                                                  w.rope_base, w.dtype)
    bt = None if inp["block_table"] is None else inp["block_table"].numpy()
    if bt is not None:   # one fp32 view of the pool (exact for bf16), gathered per unit
        kpool = inp["k_cache"].float().numpy()
        vpool = inp["v_cache"].float().numpy()
    g = w.group
    res = {}
    by_unit = {}
    for (b, i, h) in samples:
        by_unit.setdefault((b, h // g), []).append((b, i, h))
    for (b, hk), rows in by_unit.items():
        L = int(inp["seq_lens"][b])
        if bt is not None:
            Kp = oracle.gather_tokens(kpool, b, hk, L, bt)
            Vp = oracle.gather_tokens(vpool, b, hk, L, bt)
        else:
            Kp = np64(inp["k_cache"][b, hk, :L])
            Vp = np64(inp["v_cache"][b, hk, :L])
        K = np.concatenate([Kp, k_rot[b, :, hk]], 0)
        V = np.concatenate([Vp, v_st[b, :, hk]], 0)
        for (b_, i, h) in rows:
            res[(b_, i, h)] = oracle.attend(q_rot[b_, i, h][None, :], K, V, w.scale, [L + i + 1])[0]
    return res
