#!/usr/bin/env python
"""Benchmark of the iS-KV hot path on B200: streamed decode over a block-incrementally compressed
KV cache (Llama-3-8B-shaped layer: 8 kv / 32 q heads, d=128, 4096 generated tokens, b=64, w=256,
r_K=32, r_V=48, RoPE theta=5e5, bf16 rows, batch 1 per GPU).

One step = one pass of the whole hot path over one sequence batch: for each of the 4096 tokens,
append its K/V rows (window append, and a block-incremental fold of every path whenever the window
releases a block: 60 folds x 8 heads x 2 paths = 960 head-block updates) and run decode attention
of the 32 q-heads over the compressed history plus the exact window (one iskv_append_decode call
per token: the decode kernel stores the new rows in the window itself). Folds start on an internal
stream as soon as their block is complete and join the decode stream when the window releases the
block (every decode sees the same state as with folds at the trigger); the four folds of blocks
still inside the window at the end of the stream are joined at the end of the step. The step's
C-ABI calls are captured once into a CUDA graph and replayed; inputs (rows and queries of all 4096
tokens) are resident in HBM when the timed region starts; L2 is flushed (256 MiB write) before
every timed step. The fold throughput is timed separately: one append of all 4096 rows, whose 60
folds then run back to back on the caller's stream.

``--impl reference`` times the float64 CPU oracle on a bounded sample of the same workload.
Multi-GPU (torchrun): every rank streams its own independent sequence batch (weak scaling, no
collective on the data path); the step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import iskv_synth as syn  # noqa: E402

WL = syn.WORKLOADS[1]
METRIC = "decode tok/s over compressed KV"
UNIT = "tok/s"
D = 128


# ---------------------------------------------------------------------------------------------
def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=5)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--sample-every", type=int, default=16,
                   help="decode calls between event-timed samples inside the graph")
    p.add_argument("--profile-case", choices=["short", "long"], nargs="?", const="short",
                   help="run a short program for profiler captures instead of the bench: "
                        "'short' = the bench workload, 'long' = the long-context layer")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def workload_inputs(seq: int):
    """Token-major device-layout rows [T][1][H][D] for K and V, float64 values, queries."""
    T, H = WL.tokens, WL.n_kv_heads
    kd = np.empty((T, 1, H, D), np.uint16)
    vd = np.empty((T, 1, H, D), np.uint16)
    for h in range(H):
        kd[:, 0, h], _ = syn.workload_rows(WL, seq, 0, h, 0)
        vd[:, 0, h], _ = syn.workload_rows(WL, seq, 0, h, 1)
    q = syn.queries(syn.unit_seed(WL.cfg_id, seq, 0, 0, 0), (T, 1, WL.n_q_heads, D))
    return kd, vd, q


def decode_bytes(t: int, wl=None) -> int:
    """Algorithmic bytes of one decode call at t tokens (all sequences and kv-heads of the
    layer): fp32 coordinates of the compressed rows, bf16 window rows (K and V), fp32 bases, q and
    out."""
    wl = WL if wl is None else wl
    n = wl.n_c(t)
    e = t - n
    kK = kV = 0
    if n:
        f = n // wl.block
        k = [0, 0]
        for _ in range(f):
            for x, r in ((0, wl.rank_k), (1, wl.rank_v)):
                k[x] = min(r, k[x] + min(wl.block, D - k[x]))
        kK, kV = k
    per_unit = 4 * n * (kK + kV) + 2 * 2 * e * D + 4 * D * (kK + kV) + 2 * 4 * wl.group * D
    return wl.batch * wl.n_kv_heads * per_unit


class Clocks:
    """nvidia-smi sampler running during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def __enter__(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.Q}",
                                       "--format=csv,noheader,nounits", "-lms", "200"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.p is not None:
            self.p.terminate()
            try:
                self.p.wait(timeout=5)
            except Exception:
                self.p.kill()

    def summary(self):
        self.f.flush()
        rows = []
        with open(self.f.name) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.f.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return float("nan")
        sm = [num(r[1]) for r in rows]
        mx = [num(r[2]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": float(np.nanmedian(sm)), "sm_max_mhz": float(np.nanmax(mx)),
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------------------------
def oracle_sample(seq: int = 0, heads: int = 2, decodes: int = 256):
    """Times the float64 oracle on a bounded sample of the workload and extrapolates to tok/s:
    ``heads`` of the 8 kv-heads (their K and V paths and q-heads), all 4096 appends with their
    folds, and ``decodes`` of the 4096 decode steps evenly spaced in t."""
    from threadpoolctl import threadpool_info

    from oracle import OracleCache
    T, G = WL.tokens, WL.group
    kv = np.empty((1, heads, T, D))
    vv = np.empty((1, heads, T, D))
    for h in range(heads):
        kv[0, h] = syn.workload_rows(WL, seq, 0, h, 0)[1]
        vv[0, h] = syn.workload_rows(WL, seq, 0, h, 1)[1]
    q = syn.queries(syn.unit_seed(WL.cfg_id, seq, 0, 0, 0), (T, 1, WL.n_q_heads, D))
    q = q[:, :, : heads * G].astype(np.float64)
    orc = OracleCache(1, 1, heads, heads * G, D, WL.rank_k, WL.rank_v, WL.block, WL.window,
                      rope=True, rope_theta=WL.rope_theta)
    marks = sorted(set(np.linspace(1, T, decodes).round().astype(int).tolist()))
    t_app = t_dec = 0.0
    t = 0
    for m in marks:
        a = time.perf_counter()
        orc.append(0, kv[:, :, t:m], vv[:, :, t:m])
        b = time.perf_counter()
        orc.decode(0, q[m - 1])
        c = time.perf_counter()
        t_app += b - a
        t_dec += c - b
        t = m
    full = (t_app + t_dec * T / len(marks)) * (WL.n_kv_heads / heads)
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    return {
        "value": T / full,
        "unit": UNIT,
        "cores": int(threads),
        "host_cores": len(os.sched_getaffinity(0)),
        "kind": "oracle",
        "sample": (f"{heads} of {WL.n_kv_heads} kv-heads (K+V paths, {heads * G} q-heads): all "
                   f"{T} appends with their folds and {len(marks)} of {T} decode steps evenly "
                   f"spaced in t; extrapolated linearly to all heads and steps"),
        "sample_seconds": t_app + t_dec,
    }


def cpu_baseline() -> dict:
    """The oracle timed on the host with the BLAS pool as configured and with one thread (the
    oracle's matrices are small, so the pool's threads rarely help)."""
    from threadpoolctl import threadpool_limits
    cb = oracle_sample()
    out = {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")}
    out["host_cores"] = cb["host_cores"]
    with threadpool_limits(limits=1):
        out["value_1_thread"] = oracle_sample()["value"]
    return out


def run_reference(args, rank: int):
    if rank != 0:
        return
    for _ in range(args.warmup):
        oracle_sample(heads=1, decodes=48)
    vals, secs = [], []
    for _ in range(args.steps):
        s = oracle_sample(heads=1, decodes=48)
        vals.append(s["value"])
        secs.append(s["sample_seconds"])
    v = float(np.mean(vals))
    s["value"] = v
    out = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * WL.tokens / v, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WL.name, "global_batch": WL.batch * args.gpus,
                   "seq_len": WL.tokens, "parallelism": f"replicas{args.gpus}"},
        "cpu_baseline": {k: s[k] for k in ("kind", "cores", "sample", "value", "unit")},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "sample_seconds_per_step": float(np.mean(secs)),
    }
    print(json.dumps(out), flush=True)


# ---------------------------------------------------------------------------------------------
WL_LONG = syn.WORKLOADS[3]

FMA_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12    # fp32 FMA peak of the B200 at its max SM clock
HBM_NOMINAL_GBS = 7700.0                              # HBM3e nominal bandwidth (HGX figure), context

# DRAM bytes (read + write) of one launch of the split kernel as ncu counted them for the current
# kernel: the t = 4096 launch of the bench workload (--profile-case) and the long-context launch
# (--profile-case long). Set to None whenever the kernel changes until it is captured again.
TRAFFIC_T4096 = 13_453_824
TRAFFIC_LONG = 836_655_360


def long_context_decode(args, dev, flush, calls: int = 10):
    """Decode over a long compressed history: one layer of the Qwen3-8B-shaped workload (batch 8
    x 8 kv-heads, 32 q-heads, b=128, w=256, r_K=32, r_V=64) filled to 32768 tokens in one append
    (rows drawn on the GPU with the same recipe), then ``calls`` decode calls, each after an L2
    flush, timed with CUDA events: about 0.8 GB of coordinates per call, the HBM-bound regime of
    the decode kernels. Returns (microseconds per call, bytes per call)."""
    import torch

    from rank_kv_cache_isvd_b200.cache import IsKVCache
    wl = WL_LONG
    S, H, T, QH = wl.batch, wl.n_kv_heads, wl.tokens, wl.n_q_heads
    cache = IsKVCache(batch=S, n_layers=1, n_kv_heads=H, n_q_heads=QH, rank_k=wl.rank_k,
                      rank_v=wl.rank_v, block=wl.block, window=wl.window, max_tokens=T,
                      kv_dtype="bf16", rope=True, rope_theta=wl.rope_theta)
    s = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(s):
        Kr = torch.empty((S, H, T, D), dtype=torch.bfloat16, device=dev)
        Vr = torch.empty_like(Kr)
        for sq in range(S):
            for h in range(H):
                Kr[sq, h] = syn.device_rows(wl, sq, 0, h, 0, device=dev)
                Vr[sq, h] = syn.device_rows(wl, sq, 0, h, 1, device=dev)
        cache.append(0, Kr, Vr, s.cuda_stream)
        del Kr, Vr
        gen = torch.Generator(device=dev)
        gen.manual_seed(12345)
        q = torch.randn((S, QH, D), generator=gen, device=dev)
        out = torch.empty_like(q)
    s.synchronize()
    st = cache.status(s.cuda_stream)
    assert st == 0, f"device status {st} after filling the long-context layer"
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ms = []
    for i in range(args.warmup + calls):
        with torch.cuda.stream(s):
            flush.zero_()
            e0.record(s)
            cache.decode(0, q, out, s.cuda_stream)
            e1.record(s)
        s.synchronize()
        if i >= args.warmup:
            ms.append(e0.elapsed_time(e1))
    assert cache.status(s.cuda_stream) == 0 and bool(torch.isfinite(out).all())
    cache.close()
    return 1e3 * float(np.median(ms)), decode_bytes(T, wl)


WL_PREFILL = syn.WORKLOADS[4]


def prefill_and_decode(args, dev, flush, calls: int = 5):
    """One layer of the long-context workload (batch 4 x 8 kv-heads, 32 q-heads, b = 512, w = 512,
    r_K = 64, r_V = 96): the 65536-row prefill appended in one call (127 folds of 512-row blocks
    per head and path; rows drawn on the GPU), timed as a graph replay, then decode calls over
    the 65024 compressed rows. Returns (prefill ms, head-block updates, decode us, decode bytes)."""
    import torch

    from rank_kv_cache_isvd_b200.cache import IsKVCache
    wl = WL_PREFILL
    S, H, T0, QH = wl.batch, wl.n_kv_heads, wl.prefill, wl.n_q_heads
    cache = IsKVCache(batch=S, n_layers=1, n_kv_heads=H, n_q_heads=QH, rank_k=wl.rank_k,
                      rank_v=wl.rank_v, block=wl.block, window=wl.window, max_tokens=wl.tokens,
                      kv_dtype="bf16", rope=True, rope_theta=wl.rope_theta)
    s = torch.cuda.Stream(device=dev)
    sh = s.cuda_stream
    with torch.cuda.stream(s):
        Kr = torch.empty((S, H, T0, D), dtype=torch.bfloat16, device=dev)
        Vr = torch.empty_like(Kr)
        for sq in range(S):
            for h in range(H):
                Kr[sq, h] = syn.device_rows(wl, sq, 0, h, 0, T=T0, device=dev)
                Vr[sq, h] = syn.device_rows(wl, sq, 0, h, 1, T=T0, device=dev)
        cache.append(0, Kr, Vr, sh)
    s.synchronize()
    st = cache.status(sh)
    assert st == 0, f"device status {st} after the long prefill"
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        cache.reset(sh)
        cache.append(0, Kr, Vr, sh)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    pre = []
    for i in range(2):
        with torch.cuda.stream(s):
            flush.zero_()
            e0.record(s)
            g.replay()
            e1.record(s)
        s.synchronize()
        pre.append(e0.elapsed_time(e1))
    del g, Kr, Vr
    folds = wl.n_c(T0) // wl.block
    gen = torch.Generator(device=dev)
    gen.manual_seed(4242)
    q = torch.randn((S, QH, D), generator=gen, device=dev)
    out = torch.empty_like(q)
    ms = []
    for i in range(args.warmup + calls):
        with torch.cuda.stream(s):
            flush.zero_()
            e0.record(s)
            cache.decode(0, q, out, sh)
            e1.record(s)
        s.synchronize()
        if i >= args.warmup:
            ms.append(e0.elapsed_time(e1))
    assert cache.status(sh) == 0 and bool(torch.isfinite(out).all())
    cache.close()
    return (float(min(pre)), folds * S * H * 2, 1e3 * float(np.median(ms)),
            decode_bytes(T0, wl))


WL_LAYERS = syn.WORKLOADS[2]


def all_layers_decode_step(args, dev, flush, steps: int = 5):
    """One decode step of a 32-layer model: the 32-layer x 8 kv-head workload (batch 1, b=64,
    w=128, r_K=24, r_V=40) filled to 16384 tokens with one append of all layers (rows drawn on the
    GPU), then the 32 per-layer decode calls of one step captured in a CUDA graph and replayed,
    each replay after an L2 flush. Returns (microseconds per step, bytes per step)."""
    import torch

    from rank_kv_cache_isvd_b200.cache import IsKVCache
    wl = WL_LAYERS
    L, S, H, T, QH = wl.n_layers, wl.batch, wl.n_kv_heads, wl.tokens, wl.n_q_heads
    cache = IsKVCache(batch=S, n_layers=L, n_kv_heads=H, n_q_heads=QH, rank_k=wl.rank_k,
                      rank_v=wl.rank_v, block=wl.block, window=wl.window, max_tokens=T,
                      kv_dtype="bf16", rope=True, rope_theta=wl.rope_theta)
    s = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(s):
        Kr = torch.empty((L, S, H, T, D), dtype=torch.bfloat16, device=dev)
        Vr = torch.empty_like(Kr)
        for l in range(L):
            for sq in range(S):
                for h in range(H):
                    Kr[l, sq, h] = syn.device_rows(wl, sq, l, h, 0, device=dev)
                    Vr[l, sq, h] = syn.device_rows(wl, sq, l, h, 1, device=dev)
        fa0, fa1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        fa0.record(s)
        cache.append(-1, Kr, Vr, s.cuda_stream)
        fa1.record(s)
        del Kr, Vr
        gen = torch.Generator(device=dev)
        gen.manual_seed(2024)
        q = torch.randn((L, S, QH, D), generator=gen, device=dev)
        out = torch.empty_like(q)
        for l in range(L):
            cache.decode(l, q[l], out[l], s.cuda_stream)
    s.synchronize()
    st = cache.status(s.cuda_stream)
    assert st == 0, f"device status {st} after filling the 32-layer cache"
    append_ms = fa0.elapsed_time(fa1)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for l in range(L):
            cache.decode(l, q[l], out[l], s.cuda_stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ms = []
    for i in range(args.warmup + steps):
        with torch.cuda.stream(s):
            flush.zero_()
            e0.record(s)
            g.replay()
            e1.record(s)
        s.synchronize()
        if i >= args.warmup:
            ms.append(e0.elapsed_time(e1))
    assert cache.status(s.cuda_stream) == 0 and bool(torch.isfinite(out).all())
    del g
    cache.close()
    return 1e3 * float(np.median(ms)), L * decode_bytes(T, wl), append_ms


def fold_flops(wl, T: int) -> float:
    """Algorithmic flops of all folds of one append of T rows per unit (all layers, sequences,
    kv-heads, both paths): per fold 4 b d k (projection) + 4 d b^2 - 4 b^3 / 3 (residual QR, p = b)
    + 2 m n^2 + 11 n^3 (core SVD, m = k + b, n = k + p) + 2 d (k + p) r (new basis)
    + 2 n_c k r (history rotation) + 2 b d r (new rows' coordinates)."""
    b, d = wl.block, D
    units = wl.n_layers * wl.batch * wl.n_kv_heads
    total = 0.0
    for r in (wl.rank_k, wl.rank_v):
        k, n_c = 0, 0
        for _ in range(wl.n_c(T) // b):
            p = min(b, d - k)
            m, n = k + b, k + p
            total += units * (4 * b * d * k + 4 * d * b * p - 4 * p ** 3 / 3 + 2 * m * n * n
                              + 11 * n ** 3 + 2 * d * (k + p) * r + 2 * n_c * k * r + 2 * b * d * r)
            k = min(r, k + p)
            n_c += b
    return total


def max_over_ranks(x: float, world: int, device) -> float:
    """The largest of the ranks' values: a multi-GPU step lasts as long as its slowest rank."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, total_ms: float, steps: int) -> float:
    """Whole-job tokens/s: every rank streams its own sequence batch (weak scaling)."""
    return world * WL.batch * WL.tokens / (total_ms / steps / 1e3)


def fold_timing(args, dev, K, V, s, flush):
    """Milliseconds of one append of the whole stream in a single call (every fold back to back
    on the caller's stream), per replay of a captured graph."""
    import torch

    from rank_kv_cache_isvd_b200.cache import IsKVCache
    T, H = WL.tokens, WL.n_kv_heads
    fc = IsKVCache(batch=1, n_layers=1, n_kv_heads=H, n_q_heads=WL.n_q_heads, rank_k=WL.rank_k,
                   rank_v=WL.rank_v, block=WL.block, window=WL.window, max_tokens=T,
                   kv_dtype="bf16", rope=True, rope_theta=WL.rope_theta)
    Kb = K[:, 0].transpose(0, 1).contiguous()[None]                 # [1][H][T][D]
    Vb = V[:, 0].transpose(0, 1).contiguous()[None]
    sh = s.cuda_stream
    with torch.cuda.stream(s):
        fc.reset(sh)
        fc.append(0, Kb, Vb, sh)
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        fc.reset(sh)
        fc.append(0, Kb, Vb, sh)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    out = []
    for i in range(args.warmup + args.steps):
        with torch.cuda.stream(s):
            flush.zero_()
            e0.record(s)
            g.replay()
            e1.record(s)
        s.synchronize()
        if i >= args.warmup:
            out.append(e0.elapsed_time(e1))
    assert fc.status(sh) == 0
    del g
    fc.close()
    return out


def run_ours(args, rank: int, world: int, local_rank: int):
    import torch
    import torch.distributed as dist
    from cuda.bindings import runtime as rt

    import rank_kv_cache_isvd_b200 as iskv
    from rank_kv_cache_isvd_b200.cache import IsKVCache

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    T, H, QH = WL.tokens, WL.n_kv_heads, WL.n_q_heads
    kd, vd, q = workload_inputs(seq=rank)
    K = torch.from_numpy(kd.view(np.int16)).to(dev).view(torch.bfloat16)   # [T][1][H][D]
    V = torch.from_numpy(vd.view(np.int16)).to(dev).view(torch.bfloat16)
    Q = torch.from_numpy(q).to(dev)                                          # [T][1][QH][D]
    OUT = torch.empty_like(Q)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    cache = IsKVCache(batch=1, n_layers=1, n_kv_heads=H, n_q_heads=QH, rank_k=WL.rank_k,
                      rank_v=WL.rank_v, block=WL.block, window=WL.window, max_tokens=T,
                      kv_dtype="bf16", rope=True, rope_theta=WL.rope_theta, lookahead_folds=True)
    h = cache.handle
    kb, vb, qb, ob = K.data_ptr(), V.data_ptr(), Q.data_ptr(), OUT.data_ptr()
    krow = H * D * 2
    qrow = QH * D * 4

    def ev():
        err, e = rt.cudaEventCreate()
        assert err == rt.cudaError_t.cudaSuccess
        return e

    def rec(e, s):
        err, = rt.cudaEventRecordWithFlags(e, s, rt.cudaEventRecordExternal)
        assert err == rt.cudaError_t.cudaSuccess

    dec_marks = [(t, ev(), ev()) for t in range(args.sample_every - 1, T, args.sample_every)]
    dec_set = {t: (a, b) for t, a, b in dec_marks}
    fold_ts = [t for t in range(T) if WL.n_c(t + 1) > WL.n_c(t)]

    def step(stream_handle: int, timed_events: bool):
        iskv.check(iskv.iskv_reset(h, stream_handle))
        for t in range(T):
            dm = dec_set.get(t) if timed_events else None
            if dm:
                rec(dm[0], stream_handle)
            # one decode step: append token t's rows (the decode kernel stores them) and attend
            iskv.check(iskv.iskv_append_decode(h, 0, kb + t * krow, vb + t * krow, qb + t * qrow,
                                               ob + t * qrow, stream_handle))
            if dm:
                rec(dm[1], stream_handle)
        # folds started ahead for blocks the window has not released yet join the step here
        iskv.check(iskv.iskv_join(h, stream_handle))

    s = torch.cuda.Stream(device=dev)
    sh = s.cuda_stream
    # eager warm-up (function attributes, first-touch), then parity-relevant status check
    with torch.cuda.stream(s):
        step(sh, False)
    assert iskv.iskv_sync_status(h, sh) == 0, "device status after eager step"
    n0 = cache.launches()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step(sh, True)
    launches_per_step = cache.launches() - n0
    for _ in range(args.warmup):
        with torch.cuda.stream(s):
            g.replay()
    torch.cuda.synchronize(dev)

    def elapsed(a, b):
        err, ms = rt.cudaEventElapsedTime(a, b)
        assert err == rt.cudaError_t.cudaSuccess
        return ms

    if world > 1:
        dist.barrier(device_ids=[local_rank])
    torch.cuda.synchronize(dev)
    step_ms, dec_ms, dec_bytes = [], [], []
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with Clocks(local_rank) as clk:
        for _ in range(args.steps):
            with torch.cuda.stream(s):
                flush.zero_()
                e0.record(s)
                g.replay()
                e1.record(s)
            s.synchronize()
            step_ms.append(e0.elapsed_time(e1))
            for t, a, b in dec_marks:
                dec_ms.append(elapsed(a, b))
                dec_bytes.append(decode_bytes(t + 1))
    torch.cuda.synchronize(dev)
    clocks = clk.summary()
    total_ms = max_over_ranks(float(np.sum(step_ms)), world, dev)
    ms_per_step = total_ms / args.steps
    value = job_throughput(world, total_ms, args.steps)

    # ---- end to end through the public API with host buffers --------------------------------
    kh = torch.from_numpy(kd.view(np.int16)).view(torch.bfloat16).pin_memory()
    vh = torch.from_numpy(vd.view(np.int16)).view(torch.bfloat16).pin_memory()
    qh = torch.from_numpy(q).pin_memory()
    oh = torch.empty(OUT.shape, dtype=OUT.dtype).pin_memory()
    e2e_ms = []
    for i in range(args.steps + 1):
        with torch.cuda.stream(s):
            flush.zero_()
            e0.record(s)
            K.copy_(kh, non_blocking=True)
            V.copy_(vh, non_blocking=True)
            Q.copy_(qh, non_blocking=True)
            g.replay()
            oh.copy_(OUT, non_blocking=True)
            e1.record(s)
        s.synchronize()
        if i:
            e2e_ms.append(e0.elapsed_time(e1))
    e2e_total = max_over_ranks(float(np.sum(e2e_ms)), world, dev)
    e2e_value = job_throughput(world, e2e_total, args.steps)
    h2d = (kh.numel() + vh.numel()) * 2 + qh.numel() * 4
    d2h = oh.numel() * 4
    status = iskv.iskv_sync_status(h, sh)
    assert status == 0, f"device status {status}"

    # ---- fold throughput: the same 4096 rows appended in one call (60 folds back to back) ------
    fold_ms = fold_timing(args, dev, K, V, s, flush)
    # ---- decode over a long history (HBM-bound regime), rank 0 of a single-GPU run only --------
    long_us, long_bytes = (long_context_decode(args, dev, flush) if world == 1 and rank == 0
                           else (None, None))
    step_us, step_bytes, append_ms = (all_layers_decode_step(args, dev, flush)
                                      if world == 1 and rank == 0 else (None, None, None))
    pre_ms, pre_updates, pre_dec_us, pre_dec_bytes = (
        prefill_and_decode(args, dev, flush) if world == 1 and rank == 0
        else (None, None, None, None))

    # ---- roofline of the dominant kernel class --------------------------------------------------
    hbm, which = peaks()
    dec_total = float(np.mean(dec_ms)) * T          # per step, from the sampled launches
    fold_total = float(np.mean(fold_ms))
    achieved = float(np.sum(dec_bytes)) / (float(np.sum(dec_ms)) / 1e3) / 1e9
    updates = len(fold_ts) * H * 2
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": WL.name, "global_batch": world * WL.batch, "seq_len": T,
                   "kv_heads": H, "q_heads": QH, "block": WL.block, "window": WL.window,
                   "rank_k": WL.rank_k, "rank_v": WL.rank_v, "kv_dtype": "bf16",
                   "parallelism": f"replicas{world}", "l2": "flushed (256 MiB write) before each step",
                   "graph": "the step's C-ABI calls captured once into a CUDA graph"},
        "roofline": {"bound": "hbm", "kernel": "decode attention (split + combine)",
                     "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm, "frac_of_nominal": achieved / HBM_NOMINAL_GBS,
                     "traffic": TRAFFIC_T4096,
                     "traffic_launch": ("ncu count of the t = 4096 launch (--profile-case); its "
                                        f"algorithmic bytes are {decode_bytes(WL.tokens)}"),
                     "peak_source": f"{which} MEASURED_PEAKS hbm_gbs",
                     "bytes_per_launch_mean": float(np.mean(dec_bytes)),
                     "launch_us_mean": 1e3 * float(np.mean(dec_ms))},
        "fold": {"head_block_updates_per_s": updates / (fold_total / 1e3),
                 "updates_per_call": updates, "ms_per_call": fold_total,
                 "us_per_fold": 1e3 * fold_total / len(fold_ts),
                 "how": (f"one append of all {T} rows (folds on the caller's stream, with the "
                         f"history rotations and window appends), graph replay, L2 flushed; in "
                         f"the decode step the folds run ahead on an internal stream")},
        "decode_ms_per_step": dec_total,
        "roofline_long_context": None if long_us is None else {
            "bound": "hbm", "kernel": "decode attention (split + combine)",
            "workload": f"{WL_LONG.name}: one layer at t = {WL_LONG.tokens}",
            "achieved": long_bytes / (long_us / 1e6) / 1e9, "peak": hbm, "unit": "GB/s",
            "frac": long_bytes / (long_us / 1e6) / 1e9 / hbm,
            "frac_of_nominal": long_bytes / (long_us / 1e6) / 1e9 / HBM_NOMINAL_GBS,
            "traffic": TRAFFIC_LONG,
            "bytes_per_launch": long_bytes, "launch_us": long_us},
        "roofline_32_layer_step": None if step_us is None else {
            "bound": "hbm", "kernel": "decode attention (split + combine), 32 calls",
            "workload": f"{WL_LAYERS.name}: one decode step of all layers at t = {WL_LAYERS.tokens}",
            "achieved": step_bytes / (step_us / 1e6) / 1e9, "peak": hbm, "unit": "GB/s",
            "frac": step_bytes / (step_us / 1e6) / 1e9 / hbm,
            "frac_of_nominal": step_bytes / (step_us / 1e6) / 1e9 / HBM_NOMINAL_GBS,
            "traffic": None,
            "bytes_per_step": step_bytes, "step_us": step_us,
            "tok_per_s_one_sequence": 1e6 / step_us},
        "fold_all_layers": None if append_ms is None else {
            "bound": "fp32 fma", "workload": (f"{WL_LAYERS.name}: one append of all {WL_LAYERS.tokens} "
                                              f"rows of every layer (512 units per fold launch)"),
            "folds_per_unit": WL_LAYERS.n_c(WL_LAYERS.tokens) // WL_LAYERS.block,
            "append_ms": append_ms,
            "head_block_updates_per_s": (2 * WL_LAYERS.n_layers * WL_LAYERS.n_kv_heads
                                         * (WL_LAYERS.n_c(WL_LAYERS.tokens) // WL_LAYERS.block)
                                         / (append_ms / 1e3)),
            "achieved_tflops": fold_flops(WL_LAYERS, WL_LAYERS.tokens) / (append_ms / 1e3) / 1e12,
            "peak_tflops": FMA_PEAK_TFLOPS,
            "frac": fold_flops(WL_LAYERS, WL_LAYERS.tokens) / (append_ms / 1e3) / 1e12 / FMA_PEAK_TFLOPS,
            "peak_source": "148 SMs x 128 fp32 lanes x 2 x 1.965 GHz (derived from the unit counts)"},
        "long_prefill": None if pre_ms is None else {
            "workload": (f"{WL_PREFILL.name}: one layer, {WL_PREFILL.prefill}-row prefill in one "
                         "append, then decode at that length"),
            "prefill_ms": pre_ms, "head_block_updates": pre_updates,
            "head_block_updates_per_s": pre_updates / (pre_ms / 1e3),
            "decode_us": pre_dec_us, "decode_bytes": pre_dec_bytes,
            "decode_achieved_gbs": pre_dec_bytes / (pre_dec_us / 1e6) / 1e9,
            "decode_frac_of_hbm": pre_dec_bytes / (pre_dec_us / 1e6) / 1e9 / hbm},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h),
                "how": "pinned host rows+queries copied in, graph replay, outputs copied out"},
        "gpu_launches": int(launches_per_step * args.steps),
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline()
    del g
    cache.close()
    if rank == 0:
        print(json.dumps(out), flush=True)


def run_profile_case():
    """Short program for profiler captures of the bench workload's kernels with few launches
    before them: one bulk append of all 4096 tokens (60 folds per head and path, each followed by
    the history rotation), then three decode calls at t = 4096."""
    import torch

    from rank_kv_cache_isvd_b200.cache import IsKVCache
    T, H, QH = WL.tokens, WL.n_kv_heads, WL.n_q_heads
    kd, vd, q = workload_inputs(seq=0)
    K = torch.from_numpy(kd.view(np.int16)).cuda().view(torch.bfloat16)[:, 0].transpose(0, 1)
    V = torch.from_numpy(vd.view(np.int16)).cuda().view(torch.bfloat16)[:, 0].transpose(0, 1)
    Q = torch.from_numpy(q[T - 1]).cuda()
    cache = IsKVCache(batch=1, n_layers=1, n_kv_heads=H, n_q_heads=QH, rank_k=WL.rank_k,
                      rank_v=WL.rank_v, block=WL.block, window=WL.window, max_tokens=T,
                      kv_dtype="bf16", rope=True, rope_theta=WL.rope_theta)
    cache.append(0, K.contiguous()[None], V.contiguous()[None])
    for _ in range(3):
        out = cache.decode(0, Q)
    torch.cuda.synchronize()
    print(json.dumps({"profile_case": WL.name, "tokens": cache.tokens(0),
                      "status": cache.status(), "launches": cache.launches(),
                      "out_norm": float(out.norm())}))
    cache.close()


def main():
    args = parse()
    if args.profile_case == "long":
        import torch
        dev = torch.device("cuda", 0)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        args.warmup = 1
        us, nbytes = long_context_decode(args, dev, flush, calls=2)
        print(json.dumps({"profile_case": "long", "us": us, "bytes": nbytes}))
        return
    if args.profile_case:
        run_profile_case()
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
