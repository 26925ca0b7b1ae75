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
    """Caller-owned copies of layer 0 of a cache, assembled from the public getters: coordinates
    and bases [batch * n_kv][...], exact rows in a ring of e = t - n_c rows. With n_c = 0 the
    factor pointers are NULL."""
    import rank_kv_cache_isvd_b200 as iskv
    S, H, d = wl.batch, wl.n_kv_heads, wl.head_dim
    t = cache.tokens(0)
    bufs = {}
    n_c = 0
    ks = []
    for x, r in ((0, wl.rank_k), (1, wl.rank_v)):
        coords, bases = [], []
        for sq in range(S):
            for h in range(H):
                C, B, _, k, n_c = cache.factors(0, sq, h, x)
                coords.append(C)
                bases.append(B)
        ks.append(k)
        bufs["coords", x] = torch.stack(coords).contiguous() if n_c else None   # [S*H][n_c][r]
        bufs["basis", x] = torch.stack(bases).contiguous() if n_c else None     # [S*H][d][r]
        rec = cache.reconstruct(0, x).reshape(S * H, t, d)                      # fp32
        e = t - n_c
        ring = torch.zeros((S * H, e, d), dtype=torch.bfloat16, device="cuda")
        for pos in range(n_c, t):
            ring[:, pos % e] = rec[:, pos].to(torch.bfloat16)         # exact: rows are bf16
        bufs["ring", x] = ring
    pos = torch.arange(t, dtype=torch.float64)
    omega = wl.rope_theta ** (-2.0 * torch.arange(d // 2, dtype=torch.float64) / d)
    ang = pos[:, None] * omega[None, :]
    bufs["rope"] = torch.stack([torch.cos(ang), torch.sin(ang)], dim=-1).float().cuda().contiguous()

    def ptr(x):
        return x.data_ptr() if x is not None else None
    view = iskv.iskv_decode_view(
        n_c=n_c, t=t, n_max=n_c, batch=S, n_kv_heads=H, n_q_heads=wl.n_q_heads, head_dim=d,
        rank_k=wl.rank_k, rank_v=wl.rank_v, k_k=ks[0], k_v=ks[1], ring_rows=t - n_c,
        kv_dtype=iskv.ISKV_BF16,
        coords_k=ptr(bufs["coords", 0]), coords_v=ptr(bufs["coords", 1]),
        basis_k=ptr(bufs["basis", 0]), basis_v=ptr(bufs["basis", 1]),
        ring_k=ptr(bufs["ring", 0]), ring_v=ptr(bufs["ring", 1]),
        rope_cs=bufs["rope"].data_ptr())
    return view, bufs


def _filled_cache(wl):
    from rank_kv_cache_isvd_b200.cache import IsKVCache
    kd, kv, vd, vv = workload_arrays(wl)
    cache = IsKVCache(batch=wl.batch, n_layers=1, n_kv_heads=wl.n_kv_heads,
                      n_q_heads=wl.n_q_heads, rank_k=wl.rank_k, rank_v=wl.rank_v,
                      block=wl.block, window=wl.window, max_tokens=wl.tokens, kv_dtype="bf16",
                      rope=True, rope_theta=wl.rope_theta)
    cache.append(0, to_device(kd[0]), to_device(vd[0]))
    return cache, kv[0], vv[0]


@pytest.mark.parametrize("batch,tokens", [(1, 1500), (2, 900), (2, 200)])
def test_no_alloc_decode_matches_handle_decode_twice(batch, tokens):
    """Two calls in a row (different queries) equal the handle decode within the attention
    tolerance; batch 2 exercises the (sequence, kv-head) indexing of the view, 200 tokens a view
    with no compressed rows (NULL factor pointers)."""
    import rank_kv_cache_isvd_b200 as iskv
    wl = dataclasses.replace(syn.WORKLOADS[1], batch=batch, n_kv_heads=2, n_q_heads=8,
                             tokens=tokens)
    cache, _, _ = _filled_cache(wl)
    view, bufs = _caller_buffers(cache, wl)
    assert (view.n_c == 0) == (tokens <= wl.window)
    outs = []
    for call in range(2):
        q = torch.from_numpy(syn.queries(40 + call, (batch, 8, 128))).cuda()
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


def test_no_alloc_decode_matches_the_float64_oracle():
    """The allocation-free decode of a batch-2 cache against the float64 oracle's attention over
    the same rows (attention tolerance)."""
    import rank_kv_cache_isvd_b200 as iskv
    from oracle import OracleCache
    wl = dataclasses.replace(syn.WORKLOADS[1], batch=2, n_kv_heads=2, n_q_heads=8, tokens=900)
    cache, kv, vv = _filled_cache(wl)
    view, bufs = _caller_buffers(cache, wl)
    orc = OracleCache(2, 1, 2, 8, 128, wl.rank_k, wl.rank_v, wl.block, wl.window, rope=True,
                      rope_theta=wl.rope_theta)
    orc.append(0, kv, vv)
    q = syn.queries(77, (2, 8, 128))
    out = torch.empty((2, 8, 128), dtype=torch.float32, device="cuda")
    assert iskv.iskv_decode_attn_noalloc(view, torch.from_numpy(q).cuda(), out) == iskv.ISKV_OK
    torch.cuda.synchronize()
    assert max_head_rel_err(out.cpu().numpy(), orc.decode(0, q.astype(np.float64))) <= ATTN_TOL
