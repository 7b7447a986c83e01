"""Benchmark of one KV-cache decode step: RoPE + KV append + GQA flash decode.

A step is one pass of the whole path over one batch: one ``kvd_decode_step``
call, which rotates the new tokens and appends k/v (the ``kv_append_rope``
kernel), then runs split-KV attention and the log-sum-exp merge (the
``decode_attention[_paged]`` kernels); ``--step-route two-calls`` makes the
same step from the two separate calls.  Inputs are resident in HBM before
the timed region; the KV cache is larger than the 126 MB L2 for every default
workload, so no flush is needed between steps (the tiny workload is flushed).
``value`` is algorithmic bytes per step (see workloads.step_bytes) divided by
the device time of the step, summed over ranks; ``e2e`` times the same step
through the public API with the new tokens copied from pinned host memory and
the output copied back, inside the timed region.  ``roofline`` is the decode
call alone (split-KV kernel + merge), with the mean, median and p10/p90 of its
per-launch device times.  ``workloads`` repeats the device timings (decode
median/p10/p90, step, algorithmic bytes, fraction of the measured copy peak,
clocks) for every other workload in the same run.  ``cpu_baseline`` is the
fp64 oracle on the host cores, on all BLAS threads and on one.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference]

Multi-GPU: one process per GPU (torchrun); every rank runs its own copy of the
workload (independent sequences, no collective on the data path), so scaling
is weak.  Times are device times (CUDA events), max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attention achieved HBM GB/s (% of B200 peak) and µs per decode step"
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 1024 * 1024


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="batched_gqa")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="CPU time budget of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch (profiling captures of a smaller case)")
    ap.add_argument("--kernel-iters", type=int, default=0,
                    help="iterations of the per-kernel loops after the timed region (default max(K, 200))")
    ap.add_argument("--no-workloads", action="store_true",
                    help="time only --workload (default: every other workload too, in a 'workloads' object)")
    ap.add_argument("--cascade", action="store_true",
                    help="shared_prefix workload: decode as prefix-once-per-group + suffix + merge "
                         "(kv_cache_decode_rope_b200.prefix.cascade_decode)")
    ap.add_argument("--shard-seq", action="store_true",
                    help="sequence-sharded decode: every rank holds 1/N of each sequence's "
                         "positions; append + shard attention + all-gather of (o, lse) + merge "
                         "(strong scaling; contiguous workloads)")
    ap.add_argument("--driver-layers", type=int, default=0,
                    help="also time the decode-step driver (DecodeLoop) over this many layers of the "
                         "workload's geometry: one token per step, graph replay vs eager calls")
    ap.add_argument("--launch", default="graph", choices=["graph", "eager"],
                    help="replay the step's library calls from CUDA graphs (default) or call them eagerly")
    ap.add_argument("--step-route", default="one-call", choices=["one-call", "two-calls"],
                    help="a step as one kvd_decode_step call (default) or as kv_append_rope then "
                         "decode_attention[_paged]")
    return ap.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


# Sources that do not build the decode kernels (their changes leave a decode
# launch's DRAM traffic as it was).
NOT_DECODE = ("append_rope.cu", "kvd_static_ws.cu")


def kernel_source_hash() -> str:
    """Hash of the CUDA sources of the decode kernels and their launch; a
    committed ncu traffic figure is only valid for it."""
    import glob
    import hashlib
    d = os.path.join(ROOT, "kv_cache_decode_rope_b200", "csrc")
    files = sorted(glob.glob(os.path.join(d, "*.cu*"))) + sorted(glob.glob(os.path.join(d, "*.h")))
    files = [f for f in files if os.path.basename(f) not in NOT_DECODE]
    h = hashlib.sha256()
    for f in files:
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def committed_traffic(workload: str):
    """dram read+write bytes per decode launch from a committed ncu summary,
    or None when the kernels changed since that capture."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(workload)
    if not e or e.get("source_hash") != kernel_source_hash():
        return None
    return e.get("traffic_bytes_per_launch")


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""
    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, index: int):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:  # noqa: BLE001 - clocks are reported as unavailable
            self.nvml = None
        self.t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nvml.nvmlDeviceGetClockInfo(self.h, self.nvml.NVML_CLOCK_SM))
                self.reasons |= self.nvml.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.nvml:
            self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.nvml:
            self.t.join()

    def summary(self):
        if not self.nvml:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


# ------------------------------------------------------------------ CPU oracle
_UNIT_POOL = {}


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # noqa: BLE001
        return 1


def oracle_sample(w, seconds: float, seed: int):
    """Time the fp64 oracle's decode on host cores over a bounded sample of the
    workload: whole (sequence, kv head) units, one after another, until the
    time budget is spent.  Returns (GB/s of attended K/V bytes, threads used,
    text)."""
    import numpy as np
    import torch
    import oracle
    from kv_cache_decode_rope_b200.workloads import draw_lengths
    cores = blas_threads()
    gen = torch.Generator().manual_seed(seed)
    lens = draw_lengths(w, gen)
    g, D, T = w.group, w.head_dim, w.q_len
    key = (w.name, D, int(lens.max()) + T)
    if key not in _UNIT_POOL:   # one stream of K/V rows, sliced per unit (drawn once, untimed)
        rng = np.random.default_rng(seed)
        n = key[2]
        _UNIT_POOL[key] = (rng.standard_normal((n, D)).astype(np.float32).astype(np.float64),
                           rng.standard_normal((n, D)).astype(np.float32).astype(np.float64))
    K_all, V_all = _UNIT_POOL[key]
    rng = np.random.default_rng(seed + 1)
    done_bytes = 0
    units = 0
    elapsed = 0.0
    while elapsed < seconds:
        b = units % w.batch
        L = int(lens[b])
        n = L + T
        K, V = K_all[:n], V_all[:n]
        q = rng.standard_normal((T, g, D))
        s0 = time.perf_counter()
        for i in range(T):
            oracle.attend(q[i], K, V, w.scale, [L + i + 1] * g)
        elapsed += time.perf_counter() - s0
        done_bytes += n * 2 * D * w.esize
        units += 1
    return done_bytes / elapsed / 1e9, cores, (
        f"{units} (sequence, kv head) units of workload {w.name} (all {g * T} rows each), "
        f"fp64 oracle attend, {elapsed:.1f} s of CPU time")


def cpu_baseline(w, seconds: float, seed: int) -> dict:
    """The oracle on the host cores: all BLAS threads, then one thread."""
    v, cores, sample = oracle_sample(w, seconds, seed)
    res = {"value": round(v, 4), "unit": "GB/s", "cores": cores, "cores_total": os.cpu_count(),
           "kind": "oracle", "sample": sample}
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            v1, _, sample1 = oracle_sample(w, seconds / 2, seed)
        res["single_thread"] = {"value": round(v1, 4), "unit": "GB/s", "cores": 1, "sample": sample1}
    except Exception as e:  # noqa: BLE001 - reported, not fatal
        res["single_thread"] = {"unavailable": str(e)[:120]}
    return res


# ------------------------------------------------------------------ GPU bench
def pct(xs, q):
    """q-th percentile (0..100) of xs by linear interpolation."""
    xs = sorted(xs)
    if not xs:
        return None
    k = (len(xs) - 1) * q / 100.0
    lo = int(math.floor(k))
    hi = min(lo + 1, len(xs) - 1)
    return xs[lo] + (xs[hi] - xs[lo]) * (k - lo)


def dist_us(ms):
    """median, p10, p90 and mean of per-iteration times (ms) in µs."""
    return {"median": round(1e3 * statistics.median(ms), 2), "p10": round(1e3 * pct(ms, 10), 2),
            "p90": round(1e3 * pct(ms, 90), 2), "mean": round(1e3 * sum(ms) / len(ms), 2),
            "n": len(ms)}


def measure(args, w, local, rank, world, steps, kernel_iters, e2e=False, cascade=False):
    """All device timings of one workload: K steps (append + decode) as the
    timed region, then per-call loops of the decode and the append, and, for
    the headline, the end-to-end step through pinned host memory."""
    import torch
    import kv_cache_decode_rope_b200 as kvd
    from kv_cache_decode_rope_b200.workloads import make_inputs_device, step_bytes

    dev = torch.device("cuda", local)
    if w.cache_mode == "prefill":
        w = w.with_(cache_mode="random")
    inp = make_inputs_device(w, seed=1000 + w.config_id + 7919 * rank, device=dev)
    out_dtype = w.torch_dtype
    out = torch.empty((w.batch, w.q_len, w.num_heads, w.head_dim), dtype=out_dtype, device=dev)
    mkl = int(inp["seq_lens"].max()) + w.q_len
    ws = torch.empty(kvd.workspace_size(batch=w.batch, num_heads=w.num_heads,
                                        num_kv_heads=w.num_kv_heads, head_dim=w.head_dim,
                                        q_len=w.q_len, dtype=w.torch_dtype),
                     dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    bt = inp["block_table"]
    nbytes = step_bytes(w, inp["seq_lens"].cpu(), torch.empty((), dtype=out_dtype).element_size())
    cache_bytes = inp["k_cache"].numel() * inp["k_cache"].element_size() * 2
    flush = cache_bytes < 2 * L2_BYTES
    flush_buf = torch.empty(4 * L2_BYTES // 4, dtype=torch.int32, device=dev) if flush else None

    def append(q, kn, vn, seq, bt_=bt, st=status):
        kvd.append_rope(q, kn, vn, inp["k_cache"], inp["v_cache"], seq, bt_, rope_base=w.rope_base,
                        status=st)

    if cascade and not w.shared_prefix:
        raise SystemExit("--cascade needs a workload with a shared prefix")

    def decode(q, seq, bt_=bt, st=status):
        if cascade:
            from kv_cache_decode_rope_b200.prefix import cascade_decode
            cascade_decode(q, inp["k_cache"], inp["v_cache"], seq, bt_, w.shared_prefix,
                           scale=w.scale, out=out)
            return
        if bt_ is None:
            kvd.decode_attention(q, inp["k_cache"], inp["v_cache"], seq, out, scale=w.scale,
                                 max_kv_len=mkl, workspace=ws, status=st)
        else:
            kvd.decode_attention_paged(q, inp["k_cache"], inp["v_cache"], seq, bt_, out, scale=w.scale,
                                       max_kv_len=mkl, workspace=ws, status=st)

    one_call = args.step_route == "one-call" and not cascade

    def step_calls(q, kn, vn, seq, bt_=bt, st=status):
        """One step through the public API: kvd_decode_step (one library
        call; on the CUDA-core path the decode kernel appends the new tokens
        itself), or kv_append_rope then decode_attention[_paged]."""
        if one_call:
            kvd.decode_step(q, kn, vn, inp["k_cache"], inp["v_cache"], seq, bt_, out, scale=w.scale,
                            max_kv_len=mkl, workspace=ws, rope_base=w.rope_base, status=st)
        else:
            append(q, kn, vn, seq, bt_, st)
            decode(q, seq, bt_, st)

    q, kn, vn, seq = inp["q"], inp["k_new"], inp["v_new"], inp["seq_lens"]
    for _ in range(args.warmup):
        step_calls(q, kn, vn, seq)
    torch.cuda.synchronize()

    # The timed loop replays the step's library call(s) from a CUDA graph
    # captured through the same public API: the kernels, their arguments and
    # the work are those of the eager calls, but the host enqueues a step in a
    # few microseconds, so the device never idles waiting for Python, and the
    # kernels' programmatic dependent launch overlaps each kernel's set-up with
    # the tail of the one before.  Two more loops replay the decode call and
    # the append call alone to time them separately (the per-kernel figures).
    # --launch eager times plain calls instead.
    graphs = []
    if args.launch == "graph":
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            step_calls(q, kn, vn, seq)
            append(q, kn, vn, seq)
            decode(q, seq)
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        g_step, g_app, g_dec = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_step):
            step_calls(q, kn, vn, seq)
        with torch.cuda.graph(g_app):
            append(q, kn, vn, seq)
        with torch.cuda.graph(g_dec):
            decode(q, seq)
        torch.cuda.synchronize()
        graphs = [g_step, g_app, g_dec]
        run_step, run_append, run_decode = g_step.replay, g_app.replay, g_dec.replay
        for _ in range(3):
            run_step()
            run_append()
            run_decode()
        torch.cuda.synchronize()
    else:
        def run_append():
            append(q, kn, vn, seq)

        def run_decode():
            decode(q, seq)

        def run_step():
            step_calls(q, kn, vn, seq)

    def timed(fn, n, before=None):
        """Per-iteration device times (ms) of n calls of fn, each after an
        untimed call of `before` (the rest of the step), L2 flushed before each
        call when the inputs fit in it."""
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n)]
        for e0, e1 in evs:
            if before is not None:
                before()
            if flush:
                flush_buf.add_(1)
            e0.record()
            fn()
            e1.record()
        torch.cuda.synchronize()
        return [e0.elapsed_time(e1) for e0, e1 in evs]

    # The timed region: K steps back to back, bracketed by two events (an
    # event between steps would itself cost the stream several microseconds).
    # A workload that fits in L2 is flushed before every step instead, and its
    # steps are then timed one by one, the flush outside each event pair.
    K = steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K if flush else 0)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t_all0 = torch.cuda.Event(enable_timing=True)
        t_all1 = torch.cuda.Event(enable_timing=True)
        t_all0.record()
        for k in range(K):
            if flush:
                flush_buf.add_(1)
                ev[k][0].record()
            run_step()
            if flush:
                ev[k][1].record()
        t_all1.record()
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        total_ms = sum(e0.elapsed_time(e1) for e0, e1 in ev) if flush else t_all0.elapsed_time(t_all1)
        # per-step and per-kernel figures, after the timed region (clocks still sampled)
        step_ms = timed(run_step, kernel_iters)
        dec_ms = timed(run_decode, kernel_iters, before=run_append)
        app_ms = timed(run_append, kernel_iters, before=run_decode)
    if status.item() != 0:
        raise RuntimeError(f"device status flags set during the bench of {w.name}: {status.item()}")

    res = dict(one_call=one_call, total_ms=total_ms, steps=K, step_ms=step_ms, dec_ms=dec_ms, app_ms=app_ms, bytes=nbytes,
               clocks=clk.summary(), flush=flush, cache_bytes=cache_bytes, w=w, mkl=mkl)
    if not e2e:
        del graphs
        return res

    # ---- end to end: the step's inputs (q, k_new, v_new, lengths, block
    # table) staged in one pinned host buffer and copied to the device in one
    # transfer, the step through the public API, the output copied back
    segs = [q, kn, vn, seq] + ([bt] if bt is not None else [])
    offs, tot = [], 0
    for t in segs:
        offs.append(tot)
        tot += (t.numel() * t.element_size() + 255) // 256 * 256
    hbuf = torch.empty(tot, dtype=torch.uint8).pin_memory()
    dbuf = torch.empty(tot, dtype=torch.uint8, device=dev)

    def view(buf, i):
        t = segs[i]
        return buf[offs[i]:offs[i] + t.numel() * t.element_size()].view(t.dtype).view(t.shape)

    for i, t in enumerate(segs):
        view(hbuf, i).copy_(t.cpu())
    dq, dk, dv, ds = (view(dbuf, i) for i in range(4))
    dbt = view(dbuf, 4) if bt is not None else None
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h2d = tot
    d2h = hout.numel() * hout.element_size()

    def e2e_step():
        dbuf.copy_(hbuf, non_blocking=True)
        step_calls(dq, dk, dv, ds, dbt, None)
        hout.copy_(out, non_blocking=True)

    for _ in range(max(3, args.warmup)):
        e2e_step()
    torch.cuda.synchronize()
    # the same calls and copies captured once as a CUDA graph, as a serving
    # loop would replay them (--launch eager: plain calls)
    run_e2e = e2e_step
    if args.launch == "graph":
        g_e2e = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            e2e_step()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        with torch.cuda.graph(g_e2e):
            e2e_step()
        graphs.append(g_e2e)
        run_e2e = g_e2e.replay
        for _ in range(3):
            run_e2e()
        torch.cuda.synchronize()
    Ke = max(K, 20)
    if world > 1:
        torch.distributed.barrier()
    # Ke steps back to back between two events (flushed workloads: one by one)
    e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(Ke if flush else 0)]
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for k in range(Ke):
        if flush:
            flush_buf.add_(1)
            e_ev[k][0].record()
        run_e2e()
        if flush:
            e_ev[k][1].record()
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = (sum(a.elapsed_time(b) for a, b in e_ev) if flush else e0.elapsed_time(e1)) / Ke
    e2e_each = timed(run_e2e, Ke)   # per-step distribution, after the timed region
    res.update(e2e_ms=e2e_ms, e2e_each=e2e_each, e2e_steps=Ke, h2d=h2d, d2h=d2h,
               e2e_launch="CUDA graph of the copies and the step's library call(s)"
               if args.launch == "graph" else "eager calls")
    del graphs
    return res


def summarise(r, peak) -> dict:
    """The per-workload figures of one measure() result (device times)."""
    dec = dist_us(r["dec_ms"])
    step = dist_us(r["step_ms"])
    b = r["bytes"]
    # means: CUDA event times come in steps of about 2 us, so a median of
    # per-launch times is quantised while a mean over many launches is not
    gbs = b["decode"] / (dec["mean"] * 1e-6) / 1e9
    step_region_us = r["total_ms"] * 1e3 / r["steps"]
    return {"config": workload_config(r["w"], {"max_kv_len": r["mkl"]}),
            "decode_us": dec, "step_us": step, "append_us": dist_us(r["app_ms"]),
            "step_us_timed_region": round(step_region_us, 2),
            "algorithmic_bytes": {"decode": b["decode"], "step": b["step"]},
            "decode_gbs": round(gbs, 1), "frac": round(gbs / peak, 4),
            "step_frac": round(b["step"] / (step_region_us * 1e-6) / 1e9 / peak, 4),
            "l2": "flushed between iterations" if r["flush"] else "inputs larger than L2",
            "clocks": r["clocks"]}


def reduce_max(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def workload_config(w, extra=None):
    c = {"workload": w.name, "batch": w.batch, "num_heads": w.num_heads, "num_kv_heads": w.num_kv_heads,
         "head_dim": w.head_dim, "q_len": w.q_len,
         "cache": f"paged (page {w.page_size})" if w.paged else "contiguous",
         "cache_len": w.cache_len if w.cache_len is not None else f"log-uniform {w.len_range}"}
    if w.shared_prefix:
        c["shared_prefix"] = f"{w.shared_prefix} tokens in pages shared by every sequence"
    if extra:
        c.update(extra)
    return c


def time_driver(w, n_layers: int, local: int, steps: int = 50) -> dict:
    """Per-step device time of DecodeLoop over n_layers layers of the
    workload's geometry: prefill of the workload's cache length through decode
    steps, then single-token steps, replayed from the captured graph and
    run as eager calls.  Caches are the driver's own (zero-filled, then written
    by the prefill)."""
    import torch
    import kv_cache_decode_rope_b200 as kvd
    dev = torch.device("cuda", local)
    L0 = int(w.cache_len or w.len_range[1] // 4)
    cap = L0 + 2 * (steps + 8)
    res = {"layers": n_layers, "workload": w.name, "prefill_tokens": L0, "steps": steps}
    gen = torch.Generator(device=dev).manual_seed(7)

    def draw(T, H):
        return torch.randn((n_layers, w.batch, T, H, w.head_dim), generator=gen, device=dev,
                           dtype=torch.float32).to(w.torch_dtype)

    for mode in ("graph", "eager"):
        loop = kvd.DecodeLoop(n_layers=n_layers, batch=w.batch, num_heads=w.num_heads,
                              num_kv_heads=w.num_kv_heads, head_dim=w.head_dim, capacity=cap,
                              dtype=w.torch_dtype, paged=w.paged, page_size=w.page_size,
                              rope_base=w.rope_base, graphs=(mode == "graph"), device=dev)
        loop.prefill(draw(L0, w.num_heads), draw(L0, w.num_kv_heads), draw(L0, w.num_kv_heads))
        ins = [(draw(1, w.num_heads), draw(1, w.num_kv_heads), draw(1, w.num_kv_heads))
               for _ in range(steps + 4)]
        for i in range(4):
            loop.step(*ins[i])
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(4, steps + 4):
            loop.step(*ins[i])
        e1.record()
        torch.cuda.synchronize(dev)
        res[f"{mode}_us_per_step"] = round(e0.elapsed_time(e1) * 1e3 / steps, 2)
        del loop
    res["kernels_per_step"] = 3 * n_layers
    return res


def main():
    args = parse()
    rank, world, local = dist_env()
    if args.impl == "reference":
        return main_reference(args, rank, world)
    import torch
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    if args.shard_seq:
        return main_sharded(args, rank, world, local)
    from kv_cache_decode_rope_b200.workloads import WORKLOADS
    torch.cuda.set_device(local)
    K = args.steps
    kernel_iters = args.kernel_iters if args.kernel_iters > 0 else max(K, 200)
    head_w = WORKLOADS[args.workload]
    if args.batch > 0:
        head_w = head_w.with_(batch=args.batch)
    r = measure(args, head_w, local, rank, world, K, kernel_iters, e2e=True, cascade=args.cascade)
    w = r["w"]
    peak, peak_kind = measured_peaks()
    total_ms = reduce_max(r["total_ms"], world)
    dec = dist_us(r["dec_ms"])
    dec_mean_ms = reduce_max(dec["mean"] * 1e-3, world)
    dec_med_ms = reduce_max(dec["median"] * 1e-3, world)
    e2e_ms = reduce_max(r["e2e_ms"], world)
    ms_step = total_ms / K
    step_bytes = r["bytes"]["step"]
    value = world * step_bytes / (ms_step * 1e-3) / 1e9
    dec_gbs = r["bytes"]["decode"] / (dec_mean_ms * 1e-3) / 1e9
    traffic = committed_traffic(w.name)
    line = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 5),
        "us_per_step": round(ms_step * 1e3, 2),
        "pct_of_peak": round(100 * value / world / peak, 1),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic (seeded N(0,1) cache, shapes of the workload)",
        "config": workload_config(w, {
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": ("flushed between steps" if r["flush"] else
                   f"inputs larger than L2 ({r['cache_bytes'] / 2**20:.0f} MiB KV cache)"),
            "step": ("kv_append_rope + cascade decode (prefix per group + suffix + merge)" if args.cascade
                     else "kvd_decode_step (kv_append_rope + decode_attention" + ("_paged" if w.paged else "")
                     + " in one call)" if r["one_call"] else
                     "kv_append_rope + decode_attention" + ("_paged" if w.paged else "")),
            "launch": "CUDA graph replay of the step's library call(s)" if args.launch == "graph"
                      else "eager calls",
            "max_kv_len": r["mkl"]}),
        "step_us": dist_us(r["step_ms"]),
        "roofline": {
            "bound": "hbm",
            "kernel": "decode_attention (split-KV kernel + LSE merge)",
            "achieved": round(dec_gbs, 1),
            "peak": peak,
            "peak_source": f"{peak_kind} hbm_gbs",
            "unit": "GB/s",
            "frac": round(dec_gbs / peak, 4),
            "us_per_launch": round(dec_mean_ms * 1e3, 2),
            "us_per_launch_median": round(dec_med_ms * 1e3, 2),
            "us_per_launch_p10": dec["p10"],
            "us_per_launch_p90": dec["p90"],
            "launches_timed": dec["n"],
            "frac_median": round(r["bytes"]["decode"] / (dec_med_ms * 1e-3) / 1e9 / peak, 4),
            "algorithmic_bytes_per_launch": r["bytes"]["decode"],
            "traffic": traffic,
        },
        "append_us": dist_us(r["app_ms"]),
        "e2e": {"value": round(world * step_bytes / (e2e_ms * 1e-3) / 1e9, 1), "unit": "GB/s",
                "us_per_step": round(e2e_ms * 1e3, 2),
                "us_per_step_median": round(1e3 * statistics.median(r["e2e_each"]), 2),
                "steps": r["e2e_steps"], "launch": r["e2e_launch"],
                "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"]},
        "gpu_launches": (6 if args.cascade else 3) * K,
        "clocks": r["clocks"],
    }
    del r
    torch.cuda.empty_cache()
    # Every other workload of the contract, measured in the same run (device
    # times; per-GPU figures, max over ranks).  Parity-only at the tiny size.
    if not args.no_workloads and not args.cascade:
        extra = {}
        for name in ("batched_gqa", "paged_cb", "mtp_verify", "long_ctx", "tiny_mha"):
            if name == w.name:
                continue
            rw = measure(args, WORKLOADS[name], local, rank, world, K, kernel_iters)
            sm = summarise(rw, peak)
            for key in ("decode_us", "step_us"):
                for stat in ("median", "mean"):
                    sm[key][stat] = round(1e3 * reduce_max(sm[key][stat] * 1e-3, world), 2)
            sm["step_us_timed_region"] = round(1e3 * reduce_max(sm["step_us_timed_region"] * 1e-3, world), 2)
            del rw
            torch.cuda.empty_cache()
            extra[name] = sm
        line["workloads"] = extra
    if args.driver_layers > 0:
        line["driver"] = time_driver(w, args.driver_layers, local)
    if rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds, seed=1000 + w.config_id)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def main_sharded(args, rank, world, local):
    """--shard-seq: the workload's sequences cut into `world` position ranges,
    one per rank (kv_cache_decode_rope_b200.sharding); every step is the shard
    append, the shard attention, the all-gather of (o, lse) and the merge."""
    import torch
    import kv_cache_decode_rope_b200 as kvd
    from kv_cache_decode_rope_b200.sharding import gather_partials, shard_bounds
    from kv_cache_decode_rope_b200.workloads import WORKLOADS, step_bytes
    w = WORKLOADS[args.workload]
    if w.paged or w.cache_len is None:
        raise SystemExit("--shard-seq takes a contiguous workload with a fixed cache length")
    dev = torch.device("cuda", local)
    T, B, Hq, Hkv, D = w.q_len, w.batch, w.num_heads, w.num_kv_heads, w.head_dim
    N = w.cache_len + T
    C = ((N + world - 1) // world + 15) // 16 * 16          # positions per rank
    gen = torch.Generator(device=dev).manual_seed(1000 + w.config_id + 7919 * rank)
    rnd = lambda shape: torch.randn(shape, generator=gen, device=dev).to(w.torch_dtype)  # noqa: E731
    k_loc, v_loc = rnd((B, Hkv, C, D)), rnd((B, Hkv, C, D))
    q0, kn, vn = rnd((B, T, Hq, D)), rnd((B, T, Hkv, D)), rnd((B, T, Hkv, D))
    seq = torch.full((B,), w.cache_len, dtype=torch.int32, device=dev)
    start, lens = shard_bounds(seq, T, rank, C)
    q = q0.clone()
    o = torch.empty((B, T, Hq, D), dtype=torch.float32, device=dev)
    lse = torch.empty((B, T, Hq), dtype=torch.float32, device=dev)
    out = torch.empty((B, T, Hq, D), dtype=w.torch_dtype, device=dev)
    ws = torch.empty(kvd.workspace_size(batch=B, num_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                                        q_len=T, dtype=w.torch_dtype), dtype=torch.uint8, device=dev)

    def attend():
        kvd.decode_attention_shard(q, k_loc, v_loc, seq, start, lens, scale=w.scale, max_kv_len=C,
                                   workspace=ws, out=o, out_lse=lse)

    def step():
        q.copy_(q0)
        kvd.append_rope_shard(q, kn, vn, k_loc, v_loc, seq, start, rope_base=w.rope_base)
        attend()
        if world > 1:
            o_all, l_all = gather_partials(o, lse)
            kvd.merge_partials(o_all, l_all, out=out)
        else:
            kvd.merge_partials(o[None], lse[None], out=out)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    run_step, run_attend = step, attend
    graphs = []
    if world == 1 and args.launch == "graph":     # collectives stay outside graphs
        g1, g2 = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(g1):
            step()
        with torch.cuda.graph(g2):
            attend()
        graphs = [g1, g2]
        run_step, run_attend = g1.replay, g2.replay
        for _ in range(3):
            run_step()
        torch.cuda.synchronize(dev)
    K = args.steps
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(K):
            run_step()
        e1.record()
        torch.cuda.synchronize(dev)
    step_ms = e0.elapsed_time(e1) / K
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record()
    for _ in range(min(K, 200)):
        run_attend()
    a1.record()
    torch.cuda.synchronize(dev)
    att_ms = a0.elapsed_time(a1) / min(K, 200)
    step_ms = reduce_max(step_ms, world)
    att_ms = reduce_max(att_ms, world)
    del graphs
    esize = torch.empty((), dtype=w.torch_dtype).element_size()
    seq_cpu = torch.full((B,), w.cache_len, dtype=torch.int64)
    total = step_bytes(w, seq_cpu, esize)["step"]               # the whole job, all ranks
    local_kv = int(lens.to(torch.int64).sum().item()) * Hkv * 2 * D * esize
    peak, peak_kind = measured_peaks()
    att_gbs = local_kv / (att_ms * 1e-3) / 1e9
    line = {
        "metric": METRIC,
        "value": round(total / (step_ms * 1e-3) / 1e9, 1),
        "unit": "GB/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": round(step_ms, 5), "us_per_step": round(step_ms * 1e3, 2),
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic (seeded N(0,1) cache per rank, shapes of the workload)",
        "config": workload_config(w, {
            "parallelism": f"sequence-sharded x{world} ({C} positions per rank)",
            "l2": "inputs larger than L2" if local_kv > 2 * L2_BYTES else "rank's shard fits L2",
            "step": "kv_append_rope_shard + decode_attention_shard + all-gather + kvd_merge_partials",
            "launch": "CUDA graph replay" if (world == 1 and args.launch == "graph")
                      else "eager calls"}),
        "roofline": {"bound": "hbm", "kernel": "decode_attention_shard (rank 0's shard)",
                     "achieved": round(att_gbs, 1), "peak": peak,
                     "peak_source": f"{peak_kind} hbm_gbs", "unit": "GB/s",
                     "frac": round(att_gbs / peak, 4), "us_per_launch": round(att_ms * 1e3, 2),
                     "algorithmic_bytes_per_launch": local_kv, "traffic": None},
        "gpu_launches": 4 * K,      # append, shard attention, its split merge, shard merge
        "clocks": clk.summary(),
    }
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main_reference(args, rank, world):
    """The oracle as it stands, timed on the host cores (rank 0 only)."""
    if rank != 0:
        return 0
    from kv_cache_decode_rope_b200.workloads import WORKLOADS, step_bytes, draw_lengths
    import torch
    w = WORKLOADS[args.workload]
    if w.cache_mode == "prefill":
        w = w.with_(cache_mode="random")
    # bounded: the whole run stays near two minutes of CPU work whatever K is
    per_step = min(1.0, 120.0 / max(1, args.steps + args.warmup))
    vals = []
    info = None
    for k in range(args.warmup + args.steps):
        v, cores, sample = oracle_sample(w, per_step, seed=1000 + w.config_id + k)
        if k >= args.warmup:
            vals.append(v)
            info = (cores, sample)
    value = statistics.median(vals)
    lens = draw_lengths(w, torch.Generator().manual_seed(1000 + w.config_id))
    step_b = step_bytes(w, lens, w.esize)["step"]
    ms = step_b / (value * 1e9) * 1e3
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic", "config": workload_config(w),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": info[0],
                         "cores_total": os.cpu_count(), "kind": "oracle",
                         "sample": "each step: " + info[1]},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
