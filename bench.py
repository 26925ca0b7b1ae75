#!/usr/bin/env python
"""Benchmark of the iS-KV hot path on B200: streamed decode over a block-incrementally compressed
KV cache, Qwen3-8B-shaped (36 layers x 8 kv-heads, 32 q-heads, d=128, batch 8 per GPU, 32768
tokens per sequence, b=128, w=256, r_K=32, r_V=64, RoPE theta=5e5, bf16 rows).

Setup (untimed): every layer's rows are drawn on the GPU (synthetic low-rank-plus-noise streams,
per-unit spectra) and the first T0 tokens of every (layer, sequence, kv-head) are appended in one
call per layer, which folds them block by block (the fill's fold throughput is reported).

One step = one fold period of the whole hot path: 128 streamed tokens, each one
``iskv_append_decode`` call per layer (window append, decode attention of the 32 q-heads over the
compressed history plus the exact window; the decode kernel stores the new rows itself). In every
step each of the 36 x 8 x 8 units folds its oldest block once per path (4608 head-block updates:
projection, residual basis, core SVD, basis update, history rotation, new rows' coordinates);
folds start on internal streams when their block is complete and join the decode stream when the
window releases the block. Inputs (rows and queries of every streamed token) are resident in HBM
when the timed region starts; every token reads about 29 GB of compressed history, far more than
L2, so no flush is needed. W warm-up steps, then K timed steps (CUDA events on the decode stream,
barrier + synchronize on both sides). ``value`` = tokens of all sequences / time.

``e2e``: K further steps through the same C-ABI calls with host buffers: each token's rows and
queries are copied from pinned host memory and its outputs copied back inside the timed region.

Dominant kernel: the decode split kernel. Its duration is measured after the timed steps, on the
same state, by a separate back-to-back run of every layer's decode call (no events between
calls), so the per-call time and the step time can be compared.

Extra keys (single GPU, rank 0): the Llama-3-8B-shaped layer streamed over 4096 tokens (graph
replay), one decode step of the 32-layer model at 16384 tokens and its all-layer fold, the
long-context layer (65536-row prefill in 512-row blocks, decode at 65K), and the single-head fp32
workload. ``--impl reference`` times the float64 CPU oracle on a bounded sample of the headline
workload. Multi-GPU (torchrun): every rank streams its own 8 sequences (weak scaling, no collective
on the data path); the step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import iskv_synth as syn  # noqa: E402

WL = syn.WORKLOADS[3]                 # the headline workload
TOK_PER_STEP = WL.block               # one fold of every unit per step
METRIC = "decode tok/s over compressed KV"
UNIT = "tok/s"
D = 128
WL_LLAMA = syn.WORKLOADS[1]
WL_LAYERS = syn.WORKLOADS[2]
WL_PREFILL = syn.WORKLOADS[4]
WL_SINGLE = syn.WORKLOADS[0]

FMA_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12    # fp32 FMA peak of the B200 at its max SM clock
HBM_NOMINAL_GBS = 7700.0                              # HBM3e nominal bandwidth (HGX figure), context
DECODE_SRC = os.path.join(ROOT, "rank_kv_cache_isvd_b200", "csrc", "decode_ws.cu")
PROFILE_DECODE = os.path.join(ROOT, "profiles", "decode_ws_qwen3-8b-layer_t32768.md")
PROFILE_DECODE_BYTES = 810811392       # algorithmic bytes of the captured launch (t = 32768)


# ---------------------------------------------------------------------------------------------
def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=4)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-extras", action="store_true", help="headline line only")
    p.add_argument("--coords", choices=["bf16", "f32"], default="f32",
                   help="storage of the coordinates C = U Sigma (bases and Sigma stay fp32)")
    p.add_argument("--profile-case", choices=["short", "long", "prefill", "joint"], nargs="?",
                   const="short",
                   help="run a short program for profiler captures instead of the bench: "
                        "'short' = the Llama-3-8B layer at 4096 tokens, 'long' = one layer of the "
                        "headline workload filled to 32768 tokens, 'prefill' = one long-context "
                        "layer (65536 rows in 512-row blocks), 'joint' = one Qwen3-8B-shaped layer "
                        "of 2 sequences with the joint factorisation of its 8 kv-heads (4096 rows, "
                        "b = 64)")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def ranks_after(wl, t: int):
    """(k_K, k_V) after the folds of t tokens (p = min(b, d - k) per fold)."""
    k = [0, 0]
    for _ in range(wl.n_c(t) // wl.block):
        for x, r in ((0, wl.rank_k), (1, wl.rank_v)):
            k[x] = min(r, k[x] + min(wl.block, D - k[x]))
    return k


def decode_bytes(t: int, wl=None, csz: int = 4) -> int:
    """Algorithmic bytes of one decode call at t tokens (all sequences and kv-heads of a layer):
    coordinates of the compressed rows (csz bytes each: 4 fp32, 2 bf16), window rows (K and V),
    fp32 bases, q and out."""
    wl = WL if wl is None else wl
    n = wl.n_c(t)
    e = t - n
    kK, kV = ranks_after(wl, t) if n else (0, 0)
    esz = 2 if wl.kv_dtype == "bf16" else 4
    per_unit = csz * n * (kK + kV) + 2 * esz * e * D + 4 * D * (kK + kV) + 2 * 4 * wl.group * D
    return wl.batch * wl.n_kv_heads * per_unit


def traffic_from_profile():
    """DRAM bytes per launch of the decode split kernel from the committed ncu summary, if it was
    taken on the current kernel source (the summary records the source's sha256); else None."""
    try:
        txt = open(PROFILE_DECODE).read()
        src = hashlib.sha256(open(DECODE_SRC, "rb").read()).hexdigest()[:16]
    except OSError:
        return None, "no profile summary"
    m = re.search(r"traffic_bytes_per_launch:\s*(\d+)\s+source_sha256_16:\s*([0-9a-f]+)", txt)
    if not m:
        return None, "no traffic line in the profile summary"
    if m.group(2) != src:
        return None, "profile summary taken on an older kernel source"
    return int(m.group(1)), ("ncu capture of the one-layer launch at t = 32768 (algorithmic "
                             f"{PROFILE_DECODE_BYTES} B), scaled by the algorithmic bytes of this launch")


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
# CPU baseline: the float64 oracle on a bounded sample of the headline workload
# ---------------------------------------------------------------------------------------------
class OracleStream:
    """The float64 oracle on one (layer, sequence, kv-head) unit of the headline workload near the
    end of its stream: filled (untimed) to 32768 - tokens rows, then streamed token by token, each
    token an append of one K and one V row (with the fold when the window releases a block) and
    the decode of the unit's 4 q-heads."""

    def __init__(self, tokens: int, seq: int = 0, layer: int = 0, head: int = 0):
        from oracle import OracleCache
        wl = WL
        self.T0 = wl.tokens - tokens
        self.kv = syn.workload_rows(wl, seq, layer, head, 0)[1][None, None]
        self.vv = syn.workload_rows(wl, seq, layer, head, 1)[1][None, None]
        self.q = syn.queries(syn.unit_seed(wl.cfg_id, seq, layer, head, 0),
                             (tokens, 1, wl.group, D)).astype(np.float64)
        self.orc = OracleCache(1, 1, 1, wl.group, D, wl.rank_k, wl.rank_v, wl.block, wl.window,
                               rope=True, rope_theta=wl.rope_theta)
        self.orc.append(0, self.kv[:, :, :self.T0], self.vv[:, :, :self.T0])
        self.i = 0

    def step(self, n: int) -> float:
        """Seconds to stream the next n tokens."""
        a = time.perf_counter()
        for _ in range(n):
            t = self.T0 + self.i
            self.orc.append(0, self.kv[:, :, t:t + 1], self.vv[:, :, t:t + 1])
            self.orc.decode(0, self.q[self.i])
            self.i += 1
        return time.perf_counter() - a


def oracle_value(sec_per_token_unit: float) -> float:
    """tok/s of the 8 sequences when every unit of a step costs sec_per_token_unit per token."""
    units = WL.n_layers * WL.batch * WL.n_kv_heads
    return WL.batch / (sec_per_token_unit * units)


def oracle_sample_text(n: int, T0: int) -> str:
    units = WL.n_layers * WL.batch * WL.n_kv_heads
    return (f"1 of {units} units ((layer, sequence, kv-head), K+V paths, {WL.group} q-heads) over "
            f"{n} streamed tokens from t = {T0} (appends, folds, decodes), after an untimed fill; "
            f"extrapolated linearly to all units")


def cpu_baseline(tokens: int = 24) -> dict:
    """The oracle timed on the host with the BLAS pool as configured, then (continuing the same
    stream) with one thread: the oracle's matrices are small, so the pool's threads rarely help."""
    from threadpoolctl import threadpool_info, threadpool_limits
    st = OracleStream(2 * tokens)
    v = oracle_value(st.step(tokens) / tokens)
    with threadpool_limits(limits=1):
        v1 = oracle_value(st.step(tokens) / tokens)
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    return {"value": v, "unit": UNIT, "cores": int(threads), "kind": "oracle",
            "sample": oracle_sample_text(tokens, st.T0),
            "host_cores": len(os.sched_getaffinity(0)), "value_1_thread": v1}


def run_reference(args, rank: int):
    if rank != 0:
        return
    from threadpoolctl import threadpool_info
    per_step = 8
    st = OracleStream((args.warmup + args.steps) * per_step)
    for _ in range(args.warmup):
        st.step(per_step)
    secs = [st.step(per_step) for _ in range(args.steps)]
    v = oracle_value(float(np.mean(secs)) / per_step)
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    out = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * WL.batch * TOK_PER_STEP / v, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WL.name, "global_batch": WL.batch * args.gpus,
                   "seq_len": WL.tokens, "tokens_per_step": TOK_PER_STEP,
                   "parallelism": f"replicas{args.gpus}"},
        "cpu_baseline": {"kind": "oracle", "cores": int(threads), "value": v, "unit": UNIT,
                         "sample": (f"each step: {oracle_sample_text(per_step, st.T0)}")},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "sample_seconds_per_step": float(np.mean(secs)),
    }
    print(json.dumps(out), flush=True)


# ---------------------------------------------------------------------------------------------
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
    """Whole-job tokens/s: every rank streams its own 8 sequences, TOK_PER_STEP tokens per step."""
    return world * WL.batch * TOK_PER_STEP / (total_ms / steps / 1e3)


def fold_flops(wl, T: int, units: int | None = None) -> float:
    """Algorithmic flops of all folds of one append of T rows per unit (all layers, sequences,
    kv-heads, both paths): per fold 4 b d k (projection) + 4 d b^2 - 4 b^3 / 3 (residual QR, p = b)
    + 2 m n^2 + 11 n^3 (core SVD, m = k + b, n = k + p) + 2 d (k + p) r (new basis)
    + 2 n_c k r (history rotation) + 2 b d r (new rows' coordinates)."""
    b, d = wl.block, D
    units = wl.n_layers * wl.batch * wl.n_kv_heads if units is None else units
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


def workload_inputs(seq: int, wl=None):
    """Token-major device-layout rows [T][1][H][D] (bf16 bits) for K and V and float32 queries
    [T][1][QH][D] of one sequence of a one-layer workload (the Llama-3-8B-shaped layer)."""
    wl = WL_LLAMA if wl is None else wl
    T, H = wl.tokens, wl.n_kv_heads
    kd = np.empty((T, 1, H, D), np.uint16)
    vd = np.empty((T, 1, H, D), np.uint16)
    for h in range(H):
        kd[:, 0, h], _ = syn.workload_rows(wl, seq, 0, h, 0)
        vd[:, 0, h], _ = syn.workload_rows(wl, seq, 0, h, 1)
    q = syn.queries(syn.unit_seed(wl.cfg_id, seq, 0, 0, 0), (T, 1, wl.n_q_heads, D))
    return kd, vd, q


def _csz(args) -> int:
    return 2 if getattr(args, "coords", "bf16") == "bf16" else 4


def _cache(wl, n_layers=None, **kw):
    from rank_kv_cache_isvd_b200.cache import IsKVCache
    args = dict(batch=wl.batch, n_layers=wl.n_layers if n_layers is None else n_layers,
                n_kv_heads=wl.n_kv_heads, n_q_heads=wl.n_q_heads, rank_k=wl.rank_k,
                rank_v=wl.rank_v, block=wl.block, window=wl.window, max_tokens=wl.tokens,
                kv_dtype=wl.kv_dtype, rope=wl.rope, rope_theta=wl.rope_theta)
    args.update(kw)
    return IsKVCache(**args)


# ---------------------------------------------------------------------------------------------
# headline: the Qwen3-8B-shaped model, streamed decode with folds
# ---------------------------------------------------------------------------------------------
def headline(args, dev, rank: int, world: int, local_rank: int):
    import torch

    import rank_kv_cache_isvd_b200 as iskv
    wl = WL
    L, S, H, QH, T = wl.n_layers, wl.batch, wl.n_kv_heads, wl.n_q_heads, wl.tokens
    n_stream = (args.warmup + 2 * args.steps) * TOK_PER_STEP
    T0 = T - n_stream
    assert wl.n_c(T0) > 0
    seqs = range(rank * S, rank * S + S)           # every rank streams its own sequences
    s = torch.cuda.Stream(device=dev)
    sh = s.cuda_stream
    cache = _cache(wl, lookahead_folds=True, coord_bf16=args.coords == "bf16")
    h = cache.handle
    SK = torch.empty((n_stream, L, S, H, D), dtype=torch.bfloat16, device=dev)
    SV = torch.empty_like(SK)
    fill_ms = 0.0
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_fill = time.perf_counter()
    with torch.cuda.stream(s):
        for l in range(L):
            K = syn.device_rows_batch(wl, seqs, l, range(H), 0, device=dev)    # [S][H][T][D]
            V = syn.device_rows_batch(wl, seqs, l, range(H), 1, device=dev)
            Kp, Vp = K[:, :, :T0].contiguous(), V[:, :, :T0].contiguous()
            e0.record(s)
            cache.append(l, Kp, Vp, sh)
            e1.record(s)
            SK[:, l] = K[:, :, T0:].permute(2, 0, 1, 3)
            SV[:, l] = V[:, :, T0:].permute(2, 0, 1, 3)
            s.synchronize()
            fill_ms += e0.elapsed_time(e1)
            del K, V, Kp, Vp
        gen = torch.Generator(device=dev)
        gen.manual_seed(31337 + rank)
        Q = torch.randn((n_stream, L, S, QH, D), generator=gen, device=dev)
        OUT = torch.empty_like(Q)
    s.synchronize()
    t_fill = time.perf_counter() - t_fill
    assert cache.status(sh) == 0, "device status after the fill"
    fill_updates = L * S * H * 2 * (wl.n_c(T0) // wl.block)

    def tokens(t_lo, t_hi, host=None):
        for t in range(t_lo, t_hi):
            if host is not None:
                SK[t].copy_(host[0][t - t_lo], non_blocking=True)
                SV[t].copy_(host[1][t - t_lo], non_blocking=True)
                Q[t].copy_(host[2][t - t_lo], non_blocking=True)
            for l in range(L):
                iskv.check(iskv.iskv_append_decode(h, l, SK[t, l].data_ptr(), SV[t, l].data_ptr(),
                                                   Q[t, l].data_ptr(), OUT[t, l].data_ptr(), sh))
            if host is not None:
                host[3][t - t_lo].copy_(OUT[t], non_blocking=True)

    pos = 0
    with torch.cuda.stream(s):
        for _ in range(args.warmup):
            tokens(pos, pos + TOK_PER_STEP)
            pos += TOK_PER_STEP
    s.synchronize()
    assert cache.status(sh) == 0, "device status after the warm-up"
    n_launch0 = cache.launches()
    if world > 1:
        import torch.distributed as dist
        dist.barrier(device_ids=[local_rank])
    torch.cuda.synchronize(dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    with Clocks(local_rank) as clk:
        torch.cuda.nvtx.range_push("timed")          # marks the timed steps for profilers
        with torch.cuda.stream(s):
            ev[0].record(s)
            for k in range(args.steps):
                tokens(pos, pos + TOK_PER_STEP)
                pos += TOK_PER_STEP
                ev[k + 1].record(s)
        s.synchronize()
        torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier(device_ids=[local_rank])
    clocks = clk.summary()
    step_ms = [ev[k].elapsed_time(ev[k + 1]) for k in range(args.steps)]
    launches = cache.launches() - n_launch0
    assert cache.status(sh) == 0, "device status after the timed steps"
    total_ms = max_over_ranks(float(np.sum(step_ms)), world, dev)
    t_now = T0 + pos

    # ---- the dominant kernel alone: every layer's decode call back to back, same state --------
    dec = []
    for _ in range(3):
        with torch.cuda.stream(s):
            e0.record(s)
            for l in range(L):
                iskv.check(iskv.iskv_decode_attn(h, l, Q[pos - 1, l].data_ptr(),
                                                 OUT[pos - 1, l].data_ptr(), sh))
            e1.record(s)
        s.synchronize()
        dec.append(e0.elapsed_time(e1) / L)
    dec_ms = float(np.median(dec))
    dec_bytes = decode_bytes(t_now, csz=_csz(args))

    # ---- end to end through the C ABI with host buffers ------------------------------------------
    lo = pos
    hi = lo + args.steps * TOK_PER_STEP
    host = (SK[lo:hi].cpu().pin_memory(), SV[lo:hi].cpu().pin_memory(),
            Q[lo:hi].cpu().pin_memory(), torch.empty(OUT[lo:hi].shape).pin_memory())
    if world > 1:
        dist.barrier(device_ids=[local_rank])
    torch.cuda.synchronize(dev)
    e2e_ms = []
    for k in range(args.steps):
        a = lo + k * TOK_PER_STEP
        hs = tuple(x[a - lo:a - lo + TOK_PER_STEP] for x in host)
        with torch.cuda.stream(s):
            e0.record(s)
            tokens(a, a + TOK_PER_STEP, host=hs)
            e1.record(s)
        s.synchronize()
        e2e_ms.append(e0.elapsed_time(e1))
    assert cache.status(sh) == 0, "device status after the end-to-end steps"
    e2e_total = max_over_ranks(float(np.sum(e2e_ms)), world, dev)
    per_tok_h2d = (SK[0].numel() + SV[0].numel()) * 2 + Q[0].numel() * 4
    per_tok_d2h = OUT[0].numel() * 4
    cache.close()
    del SK, SV, Q, OUT, host

    hbm, which = peaks()
    achieved = dec_bytes / (dec_ms / 1e3) / 1e9
    traffic, traffic_how = traffic_from_profile()
    if traffic is not None:
        # the same units per launch as the capture; traffic grows with the compressed rows read
        traffic = int(round(traffic * dec_bytes / PROFILE_DECODE_BYTES))
    ms_per_step = total_ms / args.steps
    return {
        "value": job_throughput(world, total_ms, args.steps),
        "ms_per_step": ms_per_step,
        "clocks": clocks,
        "gpu_launches": int(launches),
        "e2e": {"value": job_throughput(world, e2e_total, args.steps), "unit": UNIT,
                "h2d_bytes_per_step": int(per_tok_h2d * TOK_PER_STEP),
                "d2h_bytes_per_step": int(per_tok_d2h * TOK_PER_STEP),
                "how": ("per token: rows and queries of all layers copied from pinned host "
                        "memory, 36 append+decode calls, outputs copied back; same stream")},
        "roofline": {"bound": "hbm", "kernel": "decode attention (persistent kernel + merge), one layer call",
                     "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                     "frac_of_nominal": achieved / HBM_NOMINAL_GBS,
                     "traffic": traffic, "traffic_source": traffic_how,
                     "peak_source": f"{which} MEASURED_PEAKS hbm_gbs (copy)",
                     "bytes_per_launch": dec_bytes, "launch_us": 1e3 * dec_ms,
                     "at_tokens": t_now,
                     "how": ("36 decode calls back to back on the decode stream after the timed "
                             "steps (same cache state), CUDA events around the batch, median of 3"),
                     "decode_share_of_step": dec_ms * L * TOK_PER_STEP / ms_per_step,
                     # clock-independent size of the launch: microseconds x median SM MHz
                     "launch_mcycles": (1e3 * dec_ms * clocks["sm_mhz"] / 1e6
                                        if clocks.get("sm_mhz") else None)},
        "fold": {"head_block_updates_per_step": L * S * H * 2,
                 "fill_head_block_updates_per_s": fill_updates / (fill_ms / 1e3),
                 "fill_ms": fill_ms, "fill_folds_per_unit": wl.n_c(T0) // wl.block,
                 "fill_tflops": fold_flops(wl, T0, units=L * S * H) / (fill_ms / 1e3) / 1e12,
                 "fill_how": ("one append of T0 rows per layer (every fold of the 64 units of the "
                              "layer in one launch per block, history rotations included), CUDA "
                              "events around each append, summed over layers"),
                 "setup_wall_s": t_fill},
        "tokens": {"T0": T0, "streamed": n_stream, "end": t_now},
    }


# ---------------------------------------------------------------------------------------------
# extra keys (single GPU)
# ---------------------------------------------------------------------------------------------
def llama_layer_stream(args, dev, flush):
    """Llama-3-8B-shaped layer streamed over 4096 tokens (one iskv_append_decode per token, 60
    folds per path run ahead), captured once into a CUDA graph and replayed, L2 flushed before
    each replay; and the fold throughput of one append of the 4096 rows."""
    import torch

    import rank_kv_cache_isvd_b200 as iskv
    wl = WL_LLAMA
    T, H, QH = wl.tokens, wl.n_kv_heads, wl.n_q_heads
    kd, vd, q = workload_inputs(seq=0)
    K = torch.from_numpy(kd.view(np.int16)).to(dev).view(torch.bfloat16)   # [T][1][H][D]
    V = torch.from_numpy(vd.view(np.int16)).to(dev).view(torch.bfloat16)
    Q = torch.from_numpy(q).to(dev)
    OUT = torch.empty_like(Q)
    cache = _cache(wl, lookahead_folds=True, coord_bf16=args.coords == "bf16")
    h = cache.handle
    kb, vb, qb, ob = K.data_ptr(), V.data_ptr(), Q.data_ptr(), OUT.data_ptr()
    krow, qrow = H * D * 2, QH * D * 4
    s = torch.cuda.Stream(device=dev)
    sh = s.cuda_stream

    def step():
        iskv.check(iskv.iskv_reset(h, sh))
        for t in range(T):
            iskv.check(iskv.iskv_append_decode(h, 0, kb + t * krow, vb + t * krow, qb + t * qrow,
                                               ob + t * qrow, sh))
        iskv.check(iskv.iskv_join(h, sh))

    with torch.cuda.stream(s):
        step()
    assert iskv.iskv_sync_status(h, sh) == 0
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ms = []
    for i in range(args.warmup + args.steps):
        with torch.cuda.stream(s):
            flush.zero_()
            e0.record(s)
            g.replay()
            e1.record(s)
        s.synchronize()
        if i >= args.warmup:
            ms.append(e0.elapsed_time(e1))
    assert iskv.iskv_sync_status(h, sh) == 0
    del g
    # fold throughput: all 4096 rows in one append (60 folds per path back to back)
    Kb = K[:, 0].transpose(0, 1).contiguous()[None]
    Vb = V[:, 0].transpose(0, 1).contiguous()[None]
    fc = _cache(wl, coord_bf16=args.coords == "bf16")
    with torch.cuda.stream(s):
        fc.append(0, Kb, Vb, sh)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        fc.reset(sh)
        fc.append(0, Kb, Vb, sh)
    fms = []
    for i in range(args.warmup + args.steps):
        with torch.cuda.stream(s):
            flush.zero_()
            e0.record(s)
            g.replay()
            e1.record(s)
        s.synchronize()
        if i >= args.warmup:
            fms.append(e0.elapsed_time(e1))
    assert fc.status(sh) == 0
    del g
    fc.close()
    cache.close()
    folds = wl.n_c(T) // wl.block
    step_ms = float(np.median(ms))
    return {"workload": wl.name, "tok_per_s": T / (step_ms / 1e3), "ms_per_4096_tokens": step_ms,
            "how": "graph replay of reset + 4096 append+decode calls + join, L2 flushed",
            "fold_ms_per_append": float(np.median(fms)),
            "fold_us_per_fold": 1e3 * float(np.median(fms)) / folds,
            "fold_head_block_updates_per_s": folds * H * 2 / (float(np.median(fms)) / 1e3),
            **fold_latency_roofline(wl, float(np.median(fms)) * 1e3 / folds)}


def fold_latency_roofline(wl, fold_us: float) -> dict:
    """Latency roofline of one steady-state fold (k = r): the two paths' cores run on separate SMs,
    so a fold takes at least the slower path's core SVD cost 2 m n^2 + 11 n^3 (m = k + b,
    n = k + p) at one SM's fp32 FMA rate (128 lanes x 2 flops x 1.965 GHz)."""
    sm_flops = 128 * 2 * 1.965e9
    worst = 0.0
    for r in (wl.rank_k, wl.rank_v):
        k = min(r, D)
        p = min(wl.block, D - k)
        m, n = k + wl.block, k + p
        worst = max(worst, (2 * m * n * n + 11 * n ** 3) / sm_flops * 1e6)
    return {"fold_latency_roofline_us": worst, "fold_latency_frac": worst / fold_us}


def all_layers_decode_step(args, dev, flush, steps: int = 5):
    """32-layer x 8 kv-head workload (batch 1, b=64, w=128, r_K=24, r_V=40) filled to 16384 tokens
    with one append of all layers (every fold launch covers 512 units), then one decode step (32
    per-layer decode calls captured in a graph, replayed after L2 flushes)."""
    import torch
    wl = WL_LAYERS
    L, S, H, T, QH = wl.n_layers, wl.batch, wl.n_kv_heads, wl.tokens, wl.n_q_heads
    cache = _cache(wl, coord_bf16=args.coords == "bf16")
    s = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(s):
        Kr = torch.empty((L, S, H, T, D), dtype=torch.bfloat16, device=dev)
        Vr = torch.empty_like(Kr)
        for l in range(L):
            Kr[l] = syn.device_rows_batch(wl, range(S), l, range(H), 0, device=dev)
            Vr[l] = syn.device_rows_batch(wl, range(S), l, range(H), 1, device=dev)
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
    assert cache.status(s.cuda_stream) == 0
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
    assert cache.status(s.cuda_stream) == 0
    del g
    cache.close()
    hbm, _ = peaks()
    step_us = 1e3 * float(np.median(ms))
    nbytes = L * decode_bytes(T, wl, csz=_csz(args))
    folds = wl.n_c(T) // wl.block
    flops = fold_flops(wl, T)
    return {
        "decode_step": {"workload": f"{wl.name}: one decode step of all layers at t = {T}",
                        "step_us": step_us, "tok_per_s_one_sequence": 1e6 / step_us,
                        "bytes_per_step": nbytes,
                        "achieved_gbs": nbytes / (step_us / 1e6) / 1e9,
                        "frac": nbytes / (step_us / 1e6) / 1e9 / hbm},
        "fold_all_layers": {"bound": "fp32 fma",
                            "workload": (f"{wl.name}: one append of all {T} rows of every layer "
                                         f"(512 units per fold launch)"),
                            "folds_per_unit": folds, "append_ms": append_ms,
                            "per_fold_launch_ms": append_ms / folds,
                            "head_block_updates_per_s": 2 * L * S * H * folds / (append_ms / 1e3),
                            "achieved_tflops": flops / (append_ms / 1e3) / 1e12,
                            "peak_tflops": FMA_PEAK_TFLOPS,
                            "frac": flops / (append_ms / 1e3) / 1e12 / FMA_PEAK_TFLOPS,
                            "peak_source": "148 SMs x 128 fp32 lanes x 2 x 1.965 GHz"}}


def long_prefill(args, dev, flush, calls: int = 5):
    """One long-context layer (batch 4 x 8 kv-heads, b = 512, w = 512, r_K = 64, r_V = 96): the
    65536-row prefill appended in one call (127 folds of 512-row blocks per unit and path),
    timed as a graph replay, then decode calls over the 65024 compressed rows."""
    import torch
    wl = WL_PREFILL
    S, H, T0, QH = wl.batch, wl.n_kv_heads, wl.prefill, wl.n_q_heads
    cache = _cache(wl, n_layers=1, coord_bf16=args.coords == "bf16")
    s = torch.cuda.Stream(device=dev)
    sh = s.cuda_stream
    with torch.cuda.stream(s):
        Kr = syn.device_rows_batch(wl, range(S), 0, range(H), 0, T=T0, device=dev)
        Vr = syn.device_rows_batch(wl, range(S), 0, range(H), 1, T=T0, device=dev)
        cache.append(0, Kr, Vr, sh)
    s.synchronize()
    assert cache.status(sh) == 0
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
    stored = cache.storage_bytes(0)
    cache.close()
    hbm, _ = peaks()
    folds = wl.n_c(T0) // wl.block
    pre_ms = float(min(pre))
    dec_us = 1e3 * float(np.median(ms))
    nbytes = decode_bytes(T0, wl, csz=_csz(args))
    return {"workload": f"{wl.name}: one layer, {T0}-row prefill in one append, then decode",
            "prefill_ms": pre_ms, "head_block_updates": folds * S * H * 2,
            "head_block_updates_per_s": folds * S * H * 2 / (pre_ms / 1e3),
            "prefill_tflops": fold_flops(wl, T0, units=S * H) / (pre_ms / 1e3) / 1e12,
            "storage_bytes": stored, "compression_vs_bf16_cache": S * H * 2 * T0 * D * 2 / stored,
            "decode_us": dec_us, "decode_bytes": nbytes,
            "decode_achieved_gbs": nbytes / (dec_us / 1e6) / 1e9,
            "decode_frac_of_hbm": nbytes / (dec_us / 1e6) / 1e9 / hbm}


def long_decode_bf16(args, dev, flush, calls: int = 5):
    """The long-context layer of `long_prefill` with bf16 coordinates (the storage at which the
    compressed cache is smaller than the bf16 cache; read by the persistent decode): the 65536-row
    prefill in one append, then decode calls over the 65024 compressed rows, L2 flushed."""
    import torch
    wl = WL_PREFILL
    S, H, T0, QH = wl.batch, wl.n_kv_heads, wl.prefill, wl.n_q_heads
    cache = _cache(wl, n_layers=1, coord_bf16=True)
    s = torch.cuda.Stream(device=dev)
    sh = s.cuda_stream
    with torch.cuda.stream(s):
        Kr = syn.device_rows_batch(wl, range(S), 0, range(H), 0, T=T0, device=dev)
        Vr = syn.device_rows_batch(wl, range(S), 0, range(H), 1, T=T0, device=dev)
        cache.append(0, Kr, Vr, sh)
        del Kr, Vr
        gen = torch.Generator(device=dev)
        gen.manual_seed(4242)
        q = torch.randn((S, QH, D), generator=gen, device=dev)
        out = torch.empty_like(q)
    s.synchronize()
    assert cache.status(sh) == 0
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
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
    stored = cache.storage_bytes(0)
    cache.close()
    hbm, _ = peaks()
    dec_us = 1e3 * float(np.median(ms))
    nbytes = decode_bytes(T0, wl, csz=2)
    return {"workload": f"{wl.name}: one layer after the {T0}-row prefill, bf16 coordinates",
            "storage_bytes": stored, "compression_vs_bf16_cache": S * H * 2 * T0 * D * 2 / stored,
            "decode_us": dec_us, "decode_bytes": nbytes,
            "decode_achieved_gbs": nbytes / (dec_us / 1e6) / 1e9,
            "decode_frac_of_hbm": nbytes / (dec_us / 1e6) / 1e9 / hbm}


def joint_layer(args, dev, flush, calls: int = 5):
    """One layer of the headline model (batch 8 x 8 kv-heads, 32 q-heads, 32768 tokens) with the
    joint per-layer factorisation: the 8 kv-heads of a sequence share one factorisation of rows of
    d = 1024, at b = 64, r_K = 32, r_V = 64 (rank + block <= 128). All 32768 rows are appended in
    one call (508 folds per joint unit and path), timed as a graph replay; then decode calls at
    t = 32768 after an L2 flush (fp32 coordinates)."""
    import dataclasses

    import torch
    wl = dataclasses.replace(WL, block=64)
    S, H, T, QH = wl.batch, wl.n_kv_heads, wl.tokens, wl.n_q_heads
    cache = _cache(wl, n_layers=1, joint_heads=True)
    s = torch.cuda.Stream(device=dev)
    sh = s.cuda_stream
    with torch.cuda.stream(s):
        K = syn.device_rows_batch(wl, range(S), 0, range(H), 0, device=dev)
        V = syn.device_rows_batch(wl, range(S), 0, range(H), 1, device=dev)
        cache.append(0, K, V, sh)
    s.synchronize()
    assert cache.status(sh) == 0
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        cache.reset(sh)
        cache.append(0, K, V, sh)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    app = []
    for _ in range(2):
        with torch.cuda.stream(s):
            flush.zero_()
            e0.record(s)
            g.replay()
            e1.record(s)
        s.synchronize()
        app.append(e0.elapsed_time(e1))
    del g, K, V
    gen = torch.Generator(device=dev)
    gen.manual_seed(777)
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
    stored = cache.storage_bytes(0)
    cache.close()
    hbm, _ = peaks()
    folds = wl.n_c(T) // wl.block
    n = wl.n_c(T)
    kK, kV = wl.rank_k, wl.rank_v
    # algorithmic bytes: each sequence's shared coordinates once, every kv-head's basis slice and
    # window rows, q and out
    nbytes = S * (4 * n * (kK + kV) + H * (2 * 2 * (T - n) * D + 4 * D * (kK + kV)
                                           + 2 * 4 * wl.group * D))
    dec_us = 1e3 * float(np.median(ms))
    app_ms = float(min(app))
    return {"workload": (f"{wl.name}, joint factorisation of the 8 kv-heads (d = 1024), b = 64: "
                         f"one layer, {T} rows appended in one call, then decode"),
            "append_ms": app_ms, "folds_per_joint_unit": folds,
            "per_fold_ms": app_ms / folds,
            "joint_block_updates_per_s": 2 * S * folds / (app_ms / 1e3),
            "storage_bytes": stored, "compression_vs_bf16_cache": S * H * 2 * T * D * 2 / stored,
            "decode_us": dec_us, "decode_bytes": nbytes,
            "decode_achieved_gbs": nbytes / (dec_us / 1e6) / 1e9,
            "decode_frac_of_hbm": nbytes / (dec_us / 1e6) / 1e9 / hbm}


def layer_decode(args, dev, flush, coords: str, calls: int = 10):
    """One layer of the headline workload (batch 8 x 8 kv-heads, 32 q-heads) filled to 32768 tokens
    in one append, then decode calls, each after an L2 flush (CUDA events, median): the per-call
    decode of the headline at its end length, for bf16 and fp32 coordinates."""
    import torch
    wl = WL
    S, H, T, QH = wl.batch, wl.n_kv_heads, wl.tokens, wl.n_q_heads
    cache = _cache(wl, n_layers=1, coord_bf16=coords == "bf16")
    s = torch.cuda.Stream(device=dev)
    sh = s.cuda_stream
    with torch.cuda.stream(s):
        K = syn.device_rows_batch(wl, range(S), 0, range(H), 0, device=dev)
        V = syn.device_rows_batch(wl, range(S), 0, range(H), 1, device=dev)
        cache.append(0, K, V, sh)
        del K, V
        gen = torch.Generator(device=dev)
        gen.manual_seed(12345)
        q = torch.randn((S, QH, D), generator=gen, device=dev)
        out = torch.empty_like(q)
    s.synchronize()
    assert cache.status(sh) == 0
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
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
    stored = cache.storage_bytes(0)
    cache.close()
    hbm, _ = peaks()
    us = 1e3 * float(np.median(ms))
    nbytes = decode_bytes(T, wl, csz=2 if coords == "bf16" else 4)
    return {"coords": coords, "launch_us": us, "bytes": nbytes,
            "storage_bytes": stored, "compression_vs_bf16_cache": S * H * 2 * T * D * 2 / stored,
            "achieved_gbs": nbytes / (us / 1e6) / 1e9, "frac": nbytes / (us / 1e6) / 1e9 / hbm,
            "frac_of_nominal": nbytes / (us / 1e6) / 1e9 / HBM_NOMINAL_GBS}


def single_head(args, dev, flush):
    """Single head, fp32 rows, no RoPE (1024 compressed rows + 64 window, b=32, r=32): one append
    of the 1088 rows (32 folds per path) and one decode, each timed as a graph replay."""
    import torch
    wl = WL_SINGLE
    kd = np.stack([syn.workload_rows(wl, 0, 0, 0, x)[0] for x in (0, 1)])   # [2][T][D] fp32
    K = torch.from_numpy(kd[0]).to(dev)[None, None].contiguous()
    V = torch.from_numpy(kd[1]).to(dev)[None, None].contiguous()
    q = torch.from_numpy(syn.queries(5, (1, 1, D))).to(dev)
    out = torch.empty_like(q)
    cache = _cache(wl)
    s = torch.cuda.Stream(device=dev)
    sh = s.cuda_stream
    with torch.cuda.stream(s):
        cache.append(0, K, V, sh)
        cache.decode(0, q, out, sh)
    s.synchronize()
    res = {}
    for name, fn in (("append_us", lambda: (cache.reset(sh), cache.append(0, K, V, sh))),
                     ("decode_us", lambda: cache.decode(0, q, out, sh))):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ms = []
        for i in range(args.warmup + 10):
            with torch.cuda.stream(s):
                flush.zero_()
                e0.record(s)
                g.replay()
                e1.record(s)
            s.synchronize()
            if i >= args.warmup:
                ms.append(e0.elapsed_time(e1))
        res[name] = 1e3 * float(np.median(ms))
        del g
    assert cache.status(sh) == 0
    cache.close()
    folds = wl.n_c(wl.tokens) // wl.block
    res.update({"workload": wl.name, "folds_per_path": folds,
                "us_per_fold": res["append_us"] / folds})
    return res


# ---------------------------------------------------------------------------------------------
def run_ours(args, rank: int, world: int, local_rank: int):
    import torch

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    head = headline(args, dev, rank, world, local_rank)
    out = {
        "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": WL.name, "global_batch": world * WL.batch, "seq_len": WL.tokens,
                   "layers": WL.n_layers, "kv_heads": WL.n_kv_heads, "q_heads": WL.n_q_heads,
                   "block": WL.block, "window": WL.window, "rank_k": WL.rank_k,
                   "rank_v": WL.rank_v, "kv_dtype": WL.kv_dtype,
                   "coords": args.coords, "basis_sigma": "f32",
                   "tokens_per_step": TOK_PER_STEP, "tokens": head["tokens"],
                   "parallelism": f"replicas{world}",
                   "l2": "inputs larger than L2 (about 29 GB of compressed history per token)"},
        "roofline": head["roofline"],
        "fold": head["fold"],
        "e2e": head["e2e"],
        "gpu_launches": head["gpu_launches"],
        "clocks": head["clocks"],
    }
    if world == 1 and rank == 0 and not args.no_extras:
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        out["layer_decode_t32768"] = {c: layer_decode(args, dev, flush, c) for c in ("bf16", "f32")}
        out["single_head"] = single_head(args, dev, flush)
        out["llama3_8b_layer_stream"] = llama_layer_stream(args, dev, flush)
        out.update(all_layers_decode_step(args, dev, flush))
        out["long_prefill"] = long_prefill(args, dev, flush)
        out["long_decode_bf16"] = long_decode_bf16(args, dev, flush)
        out["joint_layer"] = joint_layer(args, dev, flush)
        del flush
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline()
    if rank == 0:
        print(json.dumps(out), flush=True)


def run_profile_case(which: str, coords: str = "bf16"):
    """Short programs for profiler captures, with few launches before the captured ones."""
    import torch
    dev = torch.device("cuda", 0)
    if which == "short":
        wl = WL_LLAMA
        T, H = wl.tokens, wl.n_kv_heads
        kd, vd, q = workload_inputs(seq=0)
        K = torch.from_numpy(kd.view(np.int16)).cuda().view(torch.bfloat16)[:, 0].transpose(0, 1)
        V = torch.from_numpy(vd.view(np.int16)).cuda().view(torch.bfloat16)[:, 0].transpose(0, 1)
        Q = torch.from_numpy(q[T - 1]).cuda()
        cache = _cache(wl, coord_bf16=coords == "bf16")
        cache.append(0, K.contiguous()[None], V.contiguous()[None])
    elif which == "joint":
        # joint factorisation of a Qwen3-8B-shaped layer's 8 kv-heads (d = 1024, b = 64), two
        # sequences, 4096 tokens appended in one call (60 folds per joint unit and path)
        import dataclasses
        wl = dataclasses.replace(WL, batch=2, tokens=4096, block=64)
        T = wl.tokens
        cache = _cache(wl, n_layers=1, coord_bf16=coords == "bf16", joint_heads=True)
        K = syn.device_rows_batch(wl, range(wl.batch), 0, range(wl.n_kv_heads), 0, T=T, device=dev)
        V = syn.device_rows_batch(wl, range(wl.batch), 0, range(wl.n_kv_heads), 1, T=T, device=dev)
        cache.append(0, K, V)
        del K, V
        gen = torch.Generator(device=dev)
        gen.manual_seed(12345)
        Q = torch.randn((wl.batch, wl.n_q_heads, D), generator=gen, device=dev)
    else:
        wl = WL if which == "long" else WL_PREFILL
        T = wl.tokens if which == "long" else wl.prefill
        cache = _cache(wl, n_layers=1, coord_bf16=coords == "bf16")
        K = syn.device_rows_batch(wl, range(wl.batch), 0, range(wl.n_kv_heads), 0, T=T, device=dev)
        V = syn.device_rows_batch(wl, range(wl.batch), 0, range(wl.n_kv_heads), 1, T=T, device=dev)
        cache.append(0, K, V)
        del K, V
        gen = torch.Generator(device=dev)
        gen.manual_seed(12345)
        Q = torch.randn((wl.batch, wl.n_q_heads, D), generator=gen, device=dev)
    for _ in range(3):
        out = cache.decode(0, Q)
    torch.cuda.synchronize()
    print(json.dumps({"profile_case": which, "workload": wl.name, "tokens": cache.tokens(0),
                      "coords": coords,
                      "decode_bytes": (None if which == "joint" else
                                       decode_bytes(cache.tokens(0), wl, csz=2 if coords == "bf16" else 4)),
                      "status": cache.status(), "launches": cache.launches(),
                      "out_norm": float(out.norm())}))
    cache.close()


def main():
    args = parse()
    if args.profile_case:
        run_profile_case(args.profile_case, args.coords)
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
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
