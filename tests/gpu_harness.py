"""Helpers shared by the GPU parity tests: seeded inputs for both sides, device upload, and the
error measures named in the tolerances."""
from __future__ import annotations

import numpy as np

import iskv_synth as syn


def workload_arrays(wl, T=None, variant="literal", key_scale=1.0, layers=None, seqs=None,
                    heads=None):
    """Rows of every selected unit: ``(k_dev, k_val, v_dev, v_val)``, each ``[L][S][H][T][D]``.

    ``*_dev`` holds the device representation (bf16 bits as uint16, or float32), ``*_val`` the
    float64 values the oracle consumes."""
    T = wl.tokens if T is None else T
    layers = range(wl.n_layers) if layers is None else layers
    seqs = range(wl.batch) if seqs is None else seqs
    heads = range(wl.n_kv_heads) if heads is None else heads
    out = []
    for kv in (0, 1):
        dev, val = [], []
        for l in layers:
            dl, vl = [], []
            for s in seqs:
                ds, vs = [], []
                for h in heads:
                    d_, v_ = syn.workload_rows(wl, s, l, h, kv, T=T, variant=variant,
                                               key_scale=key_scale)
                    ds.append(d_)
                    vs.append(v_)
                dl.append(ds)
                vl.append(vs)
            dev.append(dl)
            val.append(vl)
        out += [np.asarray(dev), np.asarray(val)]
    return out[0], out[1], out[2], out[3]


def joint_workload_arrays(wl, T=None, variant="literal", key_scale=1.0, layers=None, seqs=None):
    """Like :func:`workload_arrays`, with each (layer, sequence)'s kv-heads drawn jointly
    (:func:`iskv_synth.joint_workload_rows`): ``(k_dev, k_val, v_dev, v_val)``, each
    ``[L][S][H][T][D]``."""
    layers = range(wl.n_layers) if layers is None else layers
    seqs = range(wl.batch) if seqs is None else seqs
    out = []
    for kv in (0, 1):
        dev, val = [], []
        for l in layers:
            dl, vl = [], []
            for s in seqs:
                d_, v_ = syn.joint_workload_rows(wl, s, l, kv, T=T, variant=variant,
                                                 key_scale=key_scale)
                dl.append(d_)
                vl.append(v_)
            dev.append(dl)
            val.append(vl)
        out += [np.asarray(dev), np.asarray(val)]
    return out[0], out[1], out[2], out[3]


def to_device(arr: np.ndarray):
    import torch
    if arr.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(arr)).cuda()


def rel_err(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def max_head_rel_err(out, ref) -> float:
    """max over (sequence, q-head) of ||o - o_ref|| / ||o_ref||."""
    out = np.asarray(out, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    num = np.linalg.norm(out - ref, axis=-1)
    den = np.maximum(np.linalg.norm(ref, axis=-1), 1e-300)
    return float((num / den).max())


def projector_err(B, B0) -> float:
    B = np.asarray(B, dtype=np.float64)
    B0 = np.asarray(B0, dtype=np.float64)
    return float(np.linalg.norm(B @ B.T - B0 @ B0.T))
