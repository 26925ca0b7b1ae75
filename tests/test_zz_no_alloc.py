"""The allocation-free decode entry point (iskv_decode_attn_noalloc) against the handle-based
iskv_decode_attn, through the C ABI.

Callers that cannot allocate device memory on their decode path (inside CUDA stream capture, in
engines whose memory is owned by their own pool, or in loops that cannot afford cudaMalloc's
implicit synchronisation) describe an existing cache with iskv_decode_view; the split partials go
to a fixed device array inside the library. This file is collected last so that a failure here
leaves every other test already run.
"""
import dataclasses
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import iskv_synth as syn  # noqa: E402
from gpu_harness import max_head_rel_err, to_device, workload_arrays  # noqa: E402

pytestmark = pytest.mark.gpu

ATTN_TOL = 2e-3


@pytest.fixture(autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _caller_buffers(cache, wl):
    """Caller-owned copies of one layer's cache, assembled from the public getters."""
    import rank_kv_cache_isvd_b200 as iskv
    H, d = wl.n_kv_heads, wl.head_dim
    t = cache.tokens(0)
    bufs = {}
    n_c = 0
    ks = []
    for x, r in ((0, wl.rank_k), (1, wl.rank_v)):
        coords, bases = [], []
        for h in range(H):
            C, B, _, k, n_c = cache.factors(0, 0, h, x)
            coords.append(C)
            bases.append(B)
        ks.append(k)
        bufs["coords", x] = torch.stack(coords).contiguous()          # [H][n_c][r]
        bufs["basis", x] = torch.stack(bases).contiguous()            # [H][d][r]
        rec = cache.reconstruct(0, x)[0]                               # [H][t][d] fp32
        e = t - n_c
        ring = torch.zeros((H, e, d), dtype=torch.bfloat16, device="cuda")
        for pos in range(n_c, t):
            ring[:, pos % e] = rec[:, pos].to(torch.bfloat16)         # exact: rows are bf16
        bufs["ring", x] = ring
    pos = torch.arange(t, dtype=torch.float64)
    omega = wl.rope_theta ** (-2.0 * torch.arange(d // 2, dtype=torch.float64) / d)
    ang = pos[:, None] * omega[None, :]
    bufs["rope"] = torch.stack([torch.cos(ang), torch.sin(ang)], dim=-1).float().cuda().contiguous()
    view = iskv.iskv_decode_view(
        n_c=n_c, t=t, n_max=n_c, batch=1, n_kv_heads=H, n_q_heads=wl.n_q_heads, head_dim=d,
        rank_k=wl.rank_k, rank_v=wl.rank_v, k_k=ks[0], k_v=ks[1], ring_rows=t - n_c,
        kv_dtype=iskv.ISKV_BF16,
        coords_k=bufs["coords", 0].data_ptr(), coords_v=bufs["coords", 1].data_ptr(),
        basis_k=bufs["basis", 0].data_ptr(), basis_v=bufs["basis", 1].data_ptr(),
        ring_k=bufs["ring", 0].data_ptr(), ring_v=bufs["ring", 1].data_ptr(),
        rope_cs=bufs["rope"].data_ptr())
    return view, bufs


def test_no_alloc_decode_matches_handle_decode_twice():
    import rank_kv_cache_isvd_b200 as iskv
    from rank_kv_cache_isvd_b200.cache import IsKVCache
    wl = dataclasses.replace(syn.WORKLOADS[1], n_kv_heads=2, n_q_heads=8, tokens=1500)
    kd, kv, vd, vv = workload_arrays(wl)
    cache = IsKVCache(batch=1, n_layers=1, n_kv_heads=2, n_q_heads=8, rank_k=wl.rank_k,
                      rank_v=wl.rank_v, block=wl.block, window=wl.window, max_tokens=wl.tokens,
                      kv_dtype="bf16", rope=True, rope_theta=wl.rope_theta)
    cache.append(0, to_device(kd[0]), to_device(vd[0]))
    view, bufs = _caller_buffers(cache, wl)
    outs = []
    for call in range(2):
        q = torch.from_numpy(syn.queries(40 + call, (1, 8, 128))).cuda()
        ref = cache.decode(0, q)
        out = torch.full_like(q, float("nan"))
        assert iskv.iskv_decode_attn_noalloc(view, q, out) == iskv.ISKV_OK
        torch.cuda.synchronize()
        assert torch.isfinite(out).all()
        assert max_head_rel_err(out.cpu().numpy(), ref.cpu().numpy()) <= ATTN_TOL
        outs.append((q, out.clone()))
    # the same query again gives the same bits (the shared scratch keeps no state that matters)
    q0, o0 = outs[0]
    again = torch.empty_like(q0)
    assert iskv.iskv_decode_attn_noalloc(view, q0, again) == iskv.ISKV_OK
    torch.cuda.synchronize()
    assert torch.equal(again, o0)
    assert cache.status() == 0
