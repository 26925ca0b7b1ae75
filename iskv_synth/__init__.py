"""Seeded synthetic inputs for the iS-KV hot path (shared by the oracle tests, the GPU tests and
the benchmark).

This module only draws random numbers and rounds them; it holds none of the method's arithmetic
(no projection, factorisation, RoPE or attention). Both the float64 CPU oracle and the CUDA path
consume exactly the arrays produced here.

Workloads (synthetic stand-ins for the 8B-model KV traces that the iS-KV summary page evaluates on,
which are not available here):

* per (sequence, layer, kv-head, path) a row stream
  ``X = (G diag(s) H^T + noise * N(0,1)) diag(c)`` with ``G`` a ``T x d`` matrix with orthonormal
  columns, ``H`` a random ``d x d`` orthogonal matrix, spectrum ``s_i = i^-a`` (``a`` = 1.5 keys,
  0.8 values unless the workload draws it per head), ``noise = 0.01`` and channel scales
  ``c_j = exp(sigma z_j)``;
* a *gapped* variant (``s_i = i^-0.5`` for ``i <= r``, ``0.01 i^-1.5`` beyond, noise ``1e-4``,
  ``G`` scaled by ``sqrt(T)``) whose singular-value gap at the rank budget is large, so that
  subspaces are well defined in float32;
* queries ``q ~ N(0, 1)``.

Rows are rounded to bf16 (round to nearest even from float32) for the bf16 workloads; the oracle
receives the float64 values of those bf16 numbers, the GPU receives their bits.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

__all__ = [
    "Workload",
    "WORKLOADS",
    "unit_seed",
    "kv_rows",
    "to_bf16",
    "queries",
    "workload_rows",
    "joint_workload_rows",
    "device_rows",
    "device_rows_batch",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and schedule of one synthetic workload."""

    name: str
    batch: int
    n_layers: int
    n_kv_heads: int
    n_q_heads: int
    head_dim: int
    rank_k: int
    rank_v: int
    block: int
    window: int
    tokens: int            # total tokens per sequence (prefill + generated)
    prefill: int           # rows appended in one call before decoding starts (0 = pure streaming)
    kv_dtype: str          # "bf16" or "f32": dtype of appended rows and of the exact window
    rope: bool
    rope_theta: float
    decay_k: tuple         # (lo, hi) of the spectrum exponent; lo == hi means fixed
    decay_v: tuple
    channel_sigma: float
    cfg_id: int

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    def n_c(self, t: int) -> int:
        """Compressed rows after ``t`` tokens (fold when the window holds window+block rows)."""
        return self.block * (max(0, t - self.window) // self.block)


WORKLOADS = {
    0: Workload("single head d=128 fp32, n=1024 + 64 window, b=32 r=32", 1, 1, 1, 1, 128, 32, 32,
                32, 64, 1088, 0, "f32", False, 5e5, (1.5, 1.5), (0.8, 0.8), 0.0, 0),
    1: Workload("Llama-3-8B layer: 8 kv / 32 q heads, 4096 tokens, b=64 w=256 rK=32 rV=48", 1, 1,
                8, 32, 128, 32, 48, 64, 256, 4096, 0, "bf16", True, 5e5, (1.5, 1.5), (0.8, 0.8),
                0.5, 1),
    2: Workload("32 layers x 8 kv heads, 16384 streamed tokens, b=64 w=128 rK=24 rV=40", 1, 32, 8,
                32, 128, 24, 40, 64, 128, 16384, 0, "bf16", True, 5e5, (1.5, 1.5), (0.8, 0.8),
                0.5, 2),
    3: Workload("Qwen3-8B: 36 layers x 8 kv heads, batch 8, 32768 tokens, b=128 w=256 rK=32 rV=64",
                8, 36, 8, 32, 128, 32, 64, 128, 256, 32768, 0, "bf16", True, 5e5, (1.0, 2.0),
                (0.5, 1.0), 0.5, 3),
    4: Workload("long context: 32 layers x 8 kv, batch 4, 65536 prefill + 2048 decode, b=512 w=512 "
                "rK=64 rV=96", 4, 32, 8, 32, 128, 64, 96, 512, 512, 65536 + 2048, 65536, "bf16",
                True, 5e5, (1.5, 1.5), (0.8, 0.8), 0.5, 4),
}


def unit_seed(cfg_id: int, seq: int, layer: int, head: int, kv: int) -> int:
    """Seed of one (sequence, layer, kv-head, path) row stream; ``kv`` is 0 for K, 1 for V."""
    return 1_000_003 * cfg_id + 10_007 * seq + 101 * layer + 2 * head + kv


def _decay(wl: Workload, seed: int, kv: int) -> float:
    lo, hi = wl.decay_k if kv == 0 else wl.decay_v
    if lo == hi:
        return float(lo)
    return float(np.random.default_rng([seed, 17]).uniform(lo, hi))


def kv_rows(T: int, d: int, seed: int, decay: float, noise: float = 0.01,
            channel_sigma: float = 0.0, variant: str = "literal", rank: int | None = None,
            scale: float = 1.0) -> np.ndarray:
    """float64 ``T x d`` synthetic low-rank-plus-noise rows (before any rounding).

    Draw order (fixed): Gaussian for G, Gaussian for H, noise, channel scales.
    """
    rng = np.random.default_rng(seed)
    g = rng.standard_normal((T, d))
    h = rng.standard_normal((d, d))
    G = np.linalg.qr(g)[0]
    H = np.linalg.qr(h)[0]
    i = np.arange(1, d + 1, dtype=np.float64)
    if variant == "literal":
        s = i ** (-decay)
    elif variant == "gapped":
        if rank is None:
            raise ValueError("gapped variant needs the rank budget")
        s = np.where(i <= rank, i ** -0.5, 0.01 * i ** -1.5)
        noise = 1e-4
        G = G * math.sqrt(T)
    elif variant == "lowrank":
        # exact rank ``rank``: no noise, top singular values i^-decay
        if rank is None:
            raise ValueError("lowrank variant needs the rank")
        s = np.where(i <= rank, i ** (-decay), 0.0)
        noise = 0.0
        G = G * math.sqrt(T)
    else:
        raise ValueError(variant)
    X = (G * s) @ H.T
    nz = rng.standard_normal((T, d))
    if noise:
        X = X + noise * nz
    if channel_sigma:
        X = X * np.exp(channel_sigma * rng.standard_normal(d))
    return X * scale


def to_bf16(x: np.ndarray):
    """Round to bf16 (float32 first, then round-to-nearest-even on the top 16 bits).

    Returns ``(bits, values)``: ``uint16`` bit patterns for the device and their exact float64
    values for the oracle.
    """
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    bits = u.astype(np.uint16)
    vals = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return bits, vals


def queries(seed: int, shape) -> np.ndarray:
    """float32 N(0, 1) queries of the given shape."""
    return np.random.default_rng([seed, 99]).standard_normal(shape, dtype=np.float32)


def workload_rows(wl: Workload, seq: int, layer: int, head: int, kv: int, T: int | None = None,
                  variant: str = "literal", key_scale: float = 1.0):
    """Rows of one unit of a workload, already in the workload's dtype.

    Returns ``(device_array, oracle_values)``: for bf16 workloads the ``uint16`` bits and their
    float64 values; for f32 workloads the float32 array and its float64 values.
    ``key_scale`` multiplies key rows (the peaky-softmax stress variant uses 8).
    """
    seed = unit_seed(wl.cfg_id, seq, layer, head, kv)
    T = wl.tokens if T is None else T
    rank = wl.rank_k if kv == 0 else wl.rank_v
    X = kv_rows(T, wl.head_dim, seed, _decay(wl, seed, kv), channel_sigma=wl.channel_sigma,
                variant=variant, rank=rank, scale=(key_scale if kv == 0 else 1.0))
    if wl.kv_dtype == "bf16":
        return to_bf16(X)
    f = X.astype(np.float32)
    return f, f.astype(np.float64)


def joint_workload_rows(wl: Workload, seq: int, layer: int, kv: int, T: int | None = None,
                        variant: str = "literal", key_scale: float = 1.0):
    """Rows of all kv-heads of one (sequence, layer, path), drawn as ONE low-rank-plus-noise
    matrix of ``T x (n_kv_heads d)`` rows (the :func:`kv_rows` recipe with ``d = n_kv_heads
    head_dim``, so the kv-heads share their dominant directions) and split head by head.

    Returns ``(device_array, oracle_values)``, each ``[n_kv_heads][T][head_dim]``, in the
    workload's dtype as :func:`workload_rows` does.
    """
    seed = unit_seed(wl.cfg_id, seq, layer, 1000, kv)
    T = wl.tokens if T is None else T
    H, d = wl.n_kv_heads, wl.head_dim
    rank = wl.rank_k if kv == 0 else wl.rank_v
    X = kv_rows(T, H * d, seed, _decay(wl, seed, kv), channel_sigma=wl.channel_sigma,
                variant=variant, rank=rank, scale=(key_scale if kv == 0 else 1.0))
    X = np.ascontiguousarray(X.reshape(T, H, d).transpose(1, 0, 2))
    if wl.kv_dtype == "bf16":
        return to_bf16(X)
    f = X.astype(np.float32)
    return f, f.astype(np.float64)


def device_rows(wl: Workload, seq: int, layer: int, head: int, kv: int, T: int | None = None,
                device="cuda"):
    """The literal recipe of :func:`kv_rows` drawn with torch on a GPU, for timing workloads too
    large to generate on the host in reasonable time (tens of thousands of rows per unit).

    Same distribution and structure (orthonormal ``G`` and ``H`` from QR of Gaussians, spectrum
    ``i^-a`` with the workload's exponent for this unit, noise 0.01, lognormal channel scales),
    but a different random stream: the values do not equal :func:`workload_rows`. Returns a
    ``T x d`` tensor in the workload's dtype on ``device``.
    """
    import torch
    T = wl.tokens if T is None else T
    d = wl.head_dim
    seed = unit_seed(wl.cfg_id, seq, layer, head, kv)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    g = torch.randn(T, d, generator=gen, device=device, dtype=torch.float32)
    h = torch.randn(d, d, generator=gen, device=device, dtype=torch.float32)
    G = torch.linalg.qr(g)[0]
    H = torch.linalg.qr(h)[0]
    a = _decay(wl, seed, kv)
    s = torch.arange(1, d + 1, device=device, dtype=torch.float32) ** (-a)
    X = (G * s) @ H.T + 0.01 * torch.randn(T, d, generator=gen, device=device)
    if wl.channel_sigma:
        X = X * torch.exp(wl.channel_sigma * torch.randn(d, generator=gen, device=device))
    return X.to(torch.bfloat16 if wl.kv_dtype == "bf16" else torch.float32)


def device_rows_batch(wl: Workload, seqs, layer: int, heads, kv: int, T: int | None = None,
                      device="cuda"):
    """:func:`device_rows` for several units at once: a ``[len(seqs)][len(heads)][T][d]`` tensor
    in the workload's dtype, drawn with one generator per (layer, path) and batched QRs.

    Same recipe as :func:`kv_rows` (orthonormal ``G``, orthogonal ``H``, spectrum ``i^-a`` with each
    unit's own exponent, noise 0.01, lognormal channel scales), a different random stream again.
    """
    import torch
    T = wl.tokens if T is None else T
    d = wl.head_dim
    seqs, heads = list(seqs), list(heads)
    n = len(seqs) * len(heads)
    gen = torch.Generator(device=device)
    gen.manual_seed(unit_seed(wl.cfg_id, seqs[0], layer, heads[0], kv) * 7919 + 13)
    a = torch.tensor([_decay(wl, unit_seed(wl.cfg_id, s, layer, h, kv), kv)
                      for s in seqs for h in heads], device=device, dtype=torch.float32)
    i = torch.arange(1, d + 1, device=device, dtype=torch.float32)
    s_ = i[None, :] ** (-a[:, None])                                   # [n][d]
    out = torch.empty((n, T, d), device=device,
                      dtype=torch.bfloat16 if wl.kv_dtype == "bf16" else torch.float32)
    for u in range(n):
        g = torch.randn(T, d, generator=gen, device=device, dtype=torch.float32)
        h = torch.randn(d, d, generator=gen, device=device, dtype=torch.float32)
        G = torch.linalg.qr(g)[0]
        H = torch.linalg.qr(h)[0]
        X = (G * s_[u]) @ H.T + 0.01 * torch.randn(T, d, generator=gen, device=device)
        if wl.channel_sigma:
            X = X * torch.exp(wl.channel_sigma * torch.randn(d, generator=gen, device=device))
        out[u] = X.to(out.dtype)
    return out.view(len(seqs), len(heads), T, d)
