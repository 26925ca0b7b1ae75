"""GPU parity of the CUDA path (through the C ABI) against the float64 oracle on the same seeded
inputs.

Tolerances: singular values relative error <= 1e-4; subspace projector error
||B B^T - B0 B0^T||_F <= 1e-3 where the relative spectral gap at the kept rank exceeds 1e-2;
attention output relative error <= 2e-3 per q-head (max over heads); window rows, token counts,
compressed-row counts and ranks bit-exact.
"""
import dataclasses
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import iskv_synth as syn  # noqa: E402
from gpu_harness import (max_head_rel_err, projector_err, rel_err, to_device,  # noqa: E402
                         workload_arrays)
from oracle import OracleCache, fold_from_coords, n_compressed  # noqa: E402

pytestmark = pytest.mark.gpu

SIG_TOL, PROJ_TOL, ATTN_TOL, GAP = 1e-4, 1e-3, 2e-3, 1e-2
W0, W1 = syn.WORKLOADS[0], syn.WORKLOADS[1]


@pytest.fixture(autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def make_cache(wl, **kw):
    from rank_kv_cache_isvd_b200.cache import IsKVCache
    args = dict(batch=wl.batch, n_layers=wl.n_layers, n_kv_heads=wl.n_kv_heads,
                n_q_heads=wl.n_q_heads, rank_k=wl.rank_k, rank_v=wl.rank_v, block=wl.block,
                window=wl.window, max_tokens=wl.tokens, kv_dtype=wl.kv_dtype, rope=wl.rope,
                rope_theta=wl.rope_theta)
    args.update(kw)
    return IsKVCache(**args)


def make_oracle(wl, rotate=True, fixed_basis=False, coord_bf16=False):
    return OracleCache(wl.batch, wl.n_layers, wl.n_kv_heads, wl.n_q_heads, wl.head_dim,
                       wl.rank_k, wl.rank_v, wl.block, wl.window, rope=wl.rope,
                       rope_theta=wl.rope_theta, rotate=rotate, fixed_basis=fixed_basis,
                       coord_bf16=coord_bf16)


def sub(wl, **kw):
    return dataclasses.replace(wl, **kw)


def append_both(cache, orc, layer, kd, kv, vd, vv, t0, t1):
    K = to_device(kd[:, :, t0:t1])
    V = to_device(vd[:, :, t0:t1])
    cache.append(layer, K, V)
    orc.append(layer, kv[:, :, t0:t1], vv[:, :, t0:t1])


# ------------------------------------------------------------------------------------------------
def test_window_rows_bit_exact_and_decode_before_any_fold():
    wl = sub(W1, n_kv_heads=2, n_q_heads=8, tokens=300)
    kd, kv, vd, vv = workload_arrays(wl)
    cache, orc = make_cache(wl), make_oracle(wl)
    append_both(cache, orc, 0, kd[0], kv[0], vd[0], vv[0], 0, 200)
    assert cache.tokens(0) == 200
    rk = cache.reconstruct(0, 0).cpu().numpy()
    rv = cache.reconstruct(0, 1).cpu().numpy()
    assert np.array_equal(rk, kv[0][:, :, :200].astype(np.float32))
    assert np.array_equal(rv, vv[0][:, :, :200].astype(np.float32))
    q = syn.queries(7, (1, 8, 128))
    out = cache.decode(0, torch.from_numpy(q).cuda()).cpu().numpy()
    assert max_head_rel_err(out, orc.decode(0, q.astype(np.float64))) <= ATTN_TOL
    assert cache.status() == 0


# ------------------------------------------------------------------------------------------------
def _snapshot(cache, wl):
    snap = {}
    for s in range(wl.batch):
        for h in range(wl.n_kv_heads):
            for x in (0, 1):
                C, B, S, k, n = cache.factors(0, s, h, x)
                snap[s, h, x] = (C.cpu().numpy().astype(np.float64), B.cpu().numpy().astype(np.float64),
                                 S.cpu().numpy().astype(np.float64), k, n)
    return snap


@pytest.mark.parametrize("variant,wl_id", [("gapped", 1), ("literal", 1), ("gapped", 3),
                                            ("literal", 3)])
def test_fold_one_step_parity(variant, wl_id):
    """Each GPU fold, started from the GPU's own state, matches the oracle's fold. With the
    Qwen3-shaped schedule (b=128, r_K=32, r_V=64) the core has more rows than columns once k > 0
    (k + b > k + p = d), so its transpose has surplus columns that converge to zero."""
    base = syn.WORKLOADS[wl_id]
    wl = sub(base, batch=1, n_layers=1, n_kv_heads=3, n_q_heads=12, tokens=1100)
    kd, kv, vd, vv = workload_arrays(wl, variant=variant)
    cache = make_cache(wl)
    t, folds, worst = 0, 0, {"sigma": 0.0, "proj": 0.0, "recon": 0.0}
    while True:
        nc = n_compressed(t, wl.block, wl.window)
        t_fold = nc + wl.window + wl.block           # the append that reaches it folds
        if t_fold > wl.tokens:
            break
        before = _snapshot(cache, wl)
        cache.append(0, to_device(kd[0][:, :, t:t_fold]), to_device(vd[0][:, :, t:t_fold]))
        t = t_fold
        after = _snapshot(cache, wl)
        folds += 1
        for (s, h, x), (C0, B0, S0, k0, n0) in before.items():
            r = wl.rank_k if x == 0 else wl.rank_v
            F = (kv if x == 0 else vv)[0][s, h, n0:n0 + wl.block]
            Cr, Sr, Br, _ = fold_from_coords(C0[:, :k0], S0[:k0], B0[:, :k0], F, r)
            C1, B1, S1, k1, n1 = after[s, h, x]
            assert n1 == n0 + wl.block and k1 == Sr.size
            sig = np.abs(S1[:k1] - Sr) / Sr
            worst["sigma"] = max(worst["sigma"], float(sig.max()))
            M = np.vstack([C0[:, :k0] @ B0[:, :k0].T, F]) if n0 else F
            sv = np.linalg.svd(M, compute_uv=False)
            gapped = k1 < sv.size and (sv[k1 - 1] - sv[k1]) / sv[0] > GAP
            rec = rel_err(C1[:, :k1] @ B1[:, :k1].T, Cr @ Br.T)
            if gapped:
                worst["proj"] = max(worst["proj"], projector_err(B1[:, :k1], Br))
                worst["recon"] = max(worst["recon"], rec)
            assert np.abs(B1[:, :k1].T @ B1[:, :k1] - np.eye(k1)).max() <= 5e-5
    print(f"\n{variant}: {folds} folds, worst {worst}")
    assert folds == n_compressed(wl.tokens, wl.block, wl.window) // wl.block
    assert worst["sigma"] <= SIG_TOL
    assert worst["proj"] <= PROJ_TOL
    assert worst["recon"] <= SIG_TOL
    assert cache.status() == 0


# ------------------------------------------------------------------------------------------------
@pytest.mark.parametrize("key_scale", [1.0, 8.0])
def test_decode_parity_llama_layer_full(key_scale):
    """Llama-3-8B-shaped layer (8 kv / 32 q heads, 4096 tokens, b=64, w=256, rK=32, rV=48)."""
    wl = W1
    kd, kv, vd, vv = workload_arrays(wl, key_scale=key_scale)
    cache, orc = make_cache(wl), make_oracle(wl)
    checkpoints = [1, 255, 256, 319, 320, 321, 700, 2048, 4095, 4096]
    t, worst = 0, 0.0
    for i, tc in enumerate(checkpoints):
        append_both(cache, orc, 0, kd[0], kv[0], vd[0], vv[0], t, tc)
        t = tc
        assert cache.tokens(0) == t
        q = syn.queries(100 + i, (1, wl.n_q_heads, 128))
        out = cache.decode(0, torch.from_numpy(q).cuda()).cpu().numpy()
        err = max_head_rel_err(out, orc.decode(0, q.astype(np.float64)))
        worst = max(worst, err)
    print(f"\nkey_scale={key_scale}: worst attention rel err {worst:.3e}")
    assert worst <= ATTN_TOL
    for x in (0, 1):
        _, B, S, k, n = cache.factors(0, 0, 0, x)
        assert n == 3840 and k == (32 if x == 0 else 48)
    assert cache.status() == 0


def test_single_head_f32_no_rope_full():
    """Single head, d=128, fp32 rows, n=1024 compressed + 64 window, b=32, r=32, one query."""
    wl = W0
    kd, kv, vd, vv = workload_arrays(wl)
    cache, orc = make_cache(wl), make_oracle(wl)
    append_both(cache, orc, 0, kd[0], kv[0], vd[0], vv[0], 0, wl.tokens)
    q = syn.queries(5, (1, 1, 128))
    out = cache.decode(0, torch.from_numpy(q).cuda()).cpu().numpy()
    assert max_head_rel_err(out, orc.decode(0, q.astype(np.float64))) <= ATTN_TOL
    _, _, S, k, n = cache.factors(0, 0, 0, 0)
    assert n == 1024 and k == 32
    assert cache.status() == 0


def test_gapped_end_to_end_sigma_and_projector():
    wl = sub(W1, n_kv_heads=2, n_q_heads=8, tokens=2000)
    kd, kv, vd, vv = workload_arrays(wl, variant="gapped")
    cache, orc = make_cache(wl), make_oracle(wl)
    append_both(cache, orc, 0, kd[0], kv[0], vd[0], vv[0], 0, wl.tokens)
    for h in range(2):
        for x in (0, 1):
            C, B, S, k, n = cache.factors(0, 0, h, x)
            u = orc.unit(0, 0, h, x)
            S, B = S.cpu().numpy(), B.cpu().numpy()
            assert k == u.k and n == u.n
            assert np.max(np.abs(S[:k] - u.sigma) / u.sigma) <= SIG_TOL
            assert projector_err(B[:, :k], u.B) <= PROJ_TOL
    q = syn.queries(9, (1, 8, 128))
    out = cache.decode(0, torch.from_numpy(q).cuda()).cpu().numpy()
    assert max_head_rel_err(out, orc.decode(0, q.astype(np.float64))) <= ATTN_TOL


def test_stale_coordinates_mode_matches_oracle():
    wl = sub(W1, n_kv_heads=1, n_q_heads=4, tokens=900)
    kd, kv, vd, vv = workload_arrays(wl, variant="gapped")
    cache, orc = make_cache(wl, rotate_history=False), make_oracle(wl, rotate=False)
    sync = make_oracle(wl)
    append_both(cache, orc, 0, kd[0], kv[0], vd[0], vv[0], 0, wl.tokens)
    sync.append(0, kv[0], vv[0])
    for x in (0, 1):
        rec = cache.reconstruct(0, x).cpu().numpy()[0, 0]
        ref = orc.unit(0, 0, 0, x).reconstruct()
        n = orc.unit(0, 0, 0, x).n
        assert rel_err(rec[:n], ref[:n]) <= 1e-3
        drift = rel_err(ref[:n], sync.unit(0, 0, 0, x).reconstruct()[:n])
        assert drift > 1e-2          # stale coordinates do drift


@pytest.mark.parametrize("block,window,rank_k,rank_v,tokens", [
    (64, 256, 32, 48, 900),        # both paths freeze after the first fold
    (32, 64, 32, 48, 700),         # keys freeze after one fold, values adapt for two
    (256, 128, 64, 96, 1500),      # blocks above 128 rows (triangular-factor folds)
])
def test_fixed_basis_mode_matches_oracle(block, window, rank_k, rank_v, tokens):
    """Fixed-basis ablation: after the folds that fill the rank budget, blocks are stored as their
    coordinates in the frozen basis. Reconstructions, ranks and decode match the oracle's variant;
    the frozen basis is the one the adapting folds produced."""
    wl = sub(W1, n_kv_heads=2, n_q_heads=8, tokens=tokens, block=block, window=window,
             rank_k=rank_k, rank_v=rank_v)
    kd, kv, vd, vv = workload_arrays(wl, variant="gapped")
    cache = make_cache(wl, fixed_basis=True, lookahead_folds=True)
    orc = make_oracle(wl, fixed_basis=True)
    append_both(cache, orc, 0, kd[0], kv[0], vd[0], vv[0], 0, wl.tokens)
    for h in range(2):
        for x in (0, 1):
            u = orc.unit(0, 0, h, x)
            C, B, S, k, n = cache.factors(0, 0, h, x)
            assert k == u.k and n == u.n and n > 2 * block
            rec = cache.reconstruct(0, x).cpu().numpy()[0, h]
            assert rel_err(rec[:n], u.reconstruct()[:n]) <= 1e-3
            assert projector_err(B.cpu().numpy()[:, :k], u.B) <= PROJ_TOL
    q = syn.queries(41, (1, 8, 128))
    out = cache.decode(0, torch.from_numpy(q).cuda()).cpu().numpy()
    assert max_head_rel_err(out, orc.decode(0, q.astype(np.float64))) <= ATTN_TOL
    assert cache.status() == 0


def test_all_layers_batched_equals_per_layer():
    wl = sub(W1, n_layers=3, n_kv_heads=2, n_q_heads=8, tokens=700)
    kd, kv, vd, vv = workload_arrays(wl)
    a, b = make_cache(wl), make_cache(wl)
    for t0, t1 in [(0, 1), (1, 333), (333, 700)]:
        a.append(-1, to_device(kd[:, :, :, t0:t1]), to_device(vd[:, :, :, t0:t1]))
        for l in range(3):
            b.append(l, to_device(kd[l, :, :, t0:t1]), to_device(vd[l, :, :, t0:t1]))
    for l in range(3):
        for x in (0, 1):
            assert torch.equal(a.reconstruct(l, x), b.reconstruct(l, x))


def test_bulk_append_equals_streaming():
    wl = sub(W1, n_kv_heads=1, n_q_heads=4, tokens=800)
    kd, kv, vd, vv = workload_arrays(wl)
    a, b = make_cache(wl), make_cache(wl)
    a.append(0, to_device(kd[0]), to_device(vd[0]))
    for t in range(800):
        b.append(0, to_device(kd[0][:, :, t:t + 1]), to_device(vd[0][:, :, t:t + 1]))
    for x in (0, 1):
        assert torch.equal(a.reconstruct(0, x), b.reconstruct(0, x))
    q = torch.from_numpy(syn.queries(3, (1, 4, 128))).cuda()
    assert torch.equal(a.decode(0, q), b.decode(0, q))


def test_no_truncation_reconstructs_exactly():
    """r = d: every fold keeps all directions (after the first fold p = 0)."""
    wl = sub(W0, rank_k=128, rank_v=128, tokens=500, block=32, window=40)
    kd, kv, vd, vv = workload_arrays(wl)
    cache = make_cache(wl)
    cache.append(0, to_device(kd[0]), to_device(vd[0]))
    for x, vals in ((0, kv), (1, vv)):
        rec = cache.reconstruct(0, x).cpu().numpy()[0, 0]
        assert rel_err(rec, vals[0][0, 0]) <= 1e-5
        _, B, _, k, _ = cache.factors(0, 0, 0, x)
        B = B.cpu().numpy()
        assert k == 128 and np.abs(B.T @ B - np.eye(128)).max() <= 5e-5


def test_exact_low_rank_and_zero_rows():
    """Rank-3 rows with r = 8: exact reconstruction and orthonormal bases even though most
    singular values are zero; an all-zero block keeps the factors finite."""
    wl = sub(W0, rank_k=8, rank_v=8, tokens=400, block=16, window=16)
    X = syn.kv_rows(400, 128, 3, 1.0, variant="lowrank", rank=3).astype(np.float32)
    X[200:232] = 0.0
    Xd = X[None, None].copy()
    cache = make_cache(wl)
    cache.append(0, to_device(Xd), to_device(Xd))
    for x in (0, 1):
        rec = cache.reconstruct(0, x).cpu().numpy()[0, 0]
        assert rel_err(rec, X) <= 1e-5
        _, B, S, k, _ = cache.factors(0, 0, 0, x)
        B = B.cpu().numpy()[:, :k]
        assert np.all(np.isfinite(S.cpu().numpy()))
        assert np.abs(B.T @ B - np.eye(k)).max() <= 1e-4
    assert cache.status() == 0


def test_block_of_one_row_and_capacity_error():
    from rank_kv_cache_isvd_b200 import ISKV_ERR_CAPACITY, IsKVError
    wl = sub(W1, n_kv_heads=1, n_q_heads=2, tokens=150, block=1, window=5, rank_k=4, rank_v=6)
    kd, kv, vd, vv = workload_arrays(wl)
    cache, orc = make_cache(wl), make_oracle(wl)
    append_both(cache, orc, 0, kd[0], kv[0], vd[0], vv[0], 0, 150)
    q = syn.queries(11, (1, 2, 128))
    out = cache.decode(0, torch.from_numpy(q).cuda()).cpu().numpy()
    assert max_head_rel_err(out, orc.decode(0, q.astype(np.float64))) <= ATTN_TOL
    with pytest.raises(IsKVError) as e:
        cache.append(0, to_device(kd[0][:, :, :1]), to_device(vd[0][:, :, :1]))
    assert e.value.code == ISKV_ERR_CAPACITY
    assert cache.tokens(0) == 150


def test_fma_decode_path_for_ranks_outside_the_tensor_core_layout():
    """r_K = 30 is not a multiple of 4, so decode runs on the CUDA-core kernel; same parity."""
    wl = sub(W1, n_kv_heads=2, n_q_heads=8, tokens=900, rank_k=30, rank_v=42)
    kd, kv, vd, vv = workload_arrays(wl)
    cache, orc = make_cache(wl), make_oracle(wl)
    append_both(cache, orc, 0, kd[0], kv[0], vd[0], vv[0], 0, wl.tokens)
    q = syn.queries(13, (1, 8, 128))
    out = cache.decode(0, torch.from_numpy(q).cuda()).cpu().numpy()
    assert max_head_rel_err(out, orc.decode(0, q.astype(np.float64))) <= ATTN_TOL
    assert cache.status() == 0


def test_decode_is_repeatable_and_graph_capturable():
    """The same decode twice gives identical output (the split-merge counters re-arm), also
    when captured into a CUDA graph and replayed."""
    wl = sub(W1, n_kv_heads=2, n_q_heads=8, tokens=1500)
    kd, kv, vd, vv = workload_arrays(wl)
    cache = make_cache(wl)
    cache.append(0, to_device(kd[0]), to_device(vd[0]))
    q = torch.from_numpy(syn.queries(17, (1, 8, 128))).cuda()
    o1 = cache.decode(0, q).clone()
    o2 = cache.decode(0, q).clone()
    assert torch.equal(o1, o2)
    out = torch.empty_like(q)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        cache.decode(0, q, out, stream=s)       # warm-up on the capture stream
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        cache.decode(0, q, out, stream=s)
    out.zero_()
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, o1)
    assert cache.status() == 0


def _stream_tokens(cache, K, V, Q, t0, t1, out, stream=None):
    for t in range(t0, t1):
        cache.append(0, K[:, :, t:t + 1].contiguous(), V[:, :, t:t + 1].contiguous(), stream)
        cache.decode(0, Q[t], out[t], stream)


def test_lookahead_folds_match_synchronous_folds_bitwise():
    """Folds started early on internal streams give exactly the decode outputs and factors of
    folds run at the trigger: every token's decode is compared bit for bit."""
    wl = sub(W1, n_kv_heads=2, n_q_heads=8, tokens=1200)
    kd, kv, vd, vv = workload_arrays(wl)
    K, V = to_device(kd[0]), to_device(vd[0])
    Q = torch.from_numpy(syn.queries(23, (wl.tokens, 1, 8, 128))).cuda()
    outs = []
    for la in (False, True):
        cache = make_cache(wl, lookahead_folds=la)
        out = torch.empty_like(Q)
        _stream_tokens(cache, K, V, Q, 0, wl.tokens, out)
        assert cache.status() == 0
        fac = [cache.factors(0, 0, h, x) for h in range(2) for x in (0, 1)]
        outs.append((out, fac, cache.launches()))
        cache.close()
    (o0, f0, n0), (o1, f1, n1) = outs
    assert torch.equal(o0, o1)
    for a, b in zip(f0, f1):
        assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
        assert a[3:] == b[3:]
    # the early folds of blocks the window never released ran too
    assert n1 >= n0


def test_lookahead_stream_captures_into_a_graph():
    """A reset + 700-token append/decode segment with early folds, captured once (joined before
    the capture ends) and replayed twice, reproduces the eager synchronous outputs."""
    wl = sub(W1, n_kv_heads=2, n_q_heads=8, tokens=700)
    kd, kv, vd, vv = workload_arrays(wl)
    K, V = to_device(kd[0]), to_device(vd[0])
    Q = torch.from_numpy(syn.queries(29, (wl.tokens, 1, 8, 128))).cuda()
    ref_cache = make_cache(wl)
    ref = torch.empty_like(Q)
    _stream_tokens(ref_cache, K, V, Q, 0, wl.tokens, ref)
    torch.cuda.synchronize()
    cache = make_cache(wl, lookahead_folds=True)
    out = torch.empty_like(Q)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        _stream_tokens(cache, K, V, Q, 0, wl.tokens, out, s)    # eager warm-up
        cache.reset(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        cache.reset(s)
        _stream_tokens(cache, K, V, Q, 0, wl.tokens, out, s)
        cache.join(s)
    for _ in range(2):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
    assert cache.status(s) == 0


@pytest.mark.parametrize("cbf", [False, True])
def test_long_context_layer_sampled_units(cbf):
    """Full-size Qwen3-8B-shaped layer as the benchmark's long-context decode runs it (batch 8 x
    8 kv-heads, 32 q-heads, b=128, w=256, r_K=32, r_V=64, 32768 tokens in one append, rows drawn
    on the GPU): every output is finite and the q-heads of three sampled (sequence, kv-head)
    units match the oracle run on those units' rows alone."""
    wl = syn.WORKLOADS[3]
    S, H, T, QH, G = wl.batch, wl.n_kv_heads, wl.tokens, wl.n_q_heads, wl.group
    cache = make_cache(sub(wl, n_layers=1), coord_bf16=cbf)
    K = torch.empty((S, H, T, 128), dtype=torch.bfloat16, device="cuda")
    V = torch.empty_like(K)
    for sq in range(S):
        for h in range(H):
            K[sq, h] = syn.device_rows(wl, sq, 0, h, 0)
            V[sq, h] = syn.device_rows(wl, sq, 0, h, 1)
    cache.append(0, K, V)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(12345)
    q = torch.randn((S, QH, 128), generator=gen, device="cuda")
    out = cache.decode(0, q)
    assert cache.status() == 0 and bool(torch.isfinite(out).all())
    assert cache.tokens(0) == T
    units, o64 = [], []
    for sq, h in ((0, 0), (3, 5), (7, 7)):
        err, (orc,), (orc64,) = _sampled_unit_check(wl, q, out, [(sq, h, K[sq, h], V[sq, h])], cbf)
        print(f"\nunit (seq {sq}, kv-head {h}): attention rel err {err:.3e}")
        assert err <= ATTN_TOL
        units.append((sq, h, K[sq, h], V[sq, h], orc))
        o64.append(orc64)
    # sharp attention (logit 20) on compressed rows early, mid and late, and a window row
    sa, sb = _sharp_checks(cache, wl, 0, units, [1000, 20000, 32500, 32700], 999,
                           o64 if cbf else None)
    print(f"sharp: {sa:.3e} vs device state, {sb:.3e} vs oracle stream")
    assert sa <= ATTN_TOL and sb <= ATTN_TOL
    cache.close()


@pytest.mark.parametrize("lookahead,window,cbf", [(False, 256, False), (True, 256, False),
                                                  (False, 0, False), (True, 256, True)])
def test_fused_append_decode_equals_separate_calls(lookahead, window, cbf):
    """iskv_append_decode (the decode kernel reads the new rows itself and stores them in the
    ring) gives bit-for-bit the outputs, factors and reconstructions of iskv_append_block +
    iskv_decode_attn, across fold triggers; with window 0 it falls back to the two calls."""
    wl = sub(W1, n_kv_heads=2, n_q_heads=8, tokens=900, window=window)
    kd, kv, vd, vv = workload_arrays(wl)
    K, V = to_device(kd[0]), to_device(vd[0])
    Q = torch.from_numpy(syn.queries(31, (wl.tokens, 1, 8, 128))).cuda()
    outs = []
    for fused in (False, True):
        cache = make_cache(wl, lookahead_folds=lookahead, coord_bf16=cbf)
        out = torch.empty_like(Q)
        for t in range(wl.tokens):
            kr = K[:, :, t:t + 1].contiguous()
            vr = V[:, :, t:t + 1].contiguous()
            if fused:
                cache.append_decode(0, kr, vr, Q[t], out[t])
            else:
                cache.append(0, kr, vr)
                cache.decode(0, Q[t], out[t])
        assert cache.status() == 0 and cache.tokens(0) == wl.tokens
        rec = [cache.reconstruct(0, x) for x in (0, 1)]
        outs.append((out, rec))
        cache.close()
    (o0, r0), (o1, r1) = outs
    assert torch.equal(o0, o1)
    assert torch.equal(r0[0], r1[0]) and torch.equal(r0[1], r1[1])


def test_decode_parity_ranks_below_one_tensor_map_box():
    """32-layer-workload ranks (r_K = 24, r_V = 40, b = 64, w = 128): the key-coordinate boxes of
    the tensor-core decode are 32 columns wide, so the last 8 come from outside the 24-column
    tensor (zero fill); decode matches the oracle at several lengths."""
    base = syn.WORKLOADS[2]
    wl = sub(base, n_layers=1, n_kv_heads=2, n_q_heads=8, tokens=1500)
    kd, kv, vd, vv = workload_arrays(wl)
    cache, orc = make_cache(wl, lookahead_folds=True), make_oracle(wl)
    t, worst = 0, 0.0
    for i, tc in enumerate([100, 129, 200, 700, 1500]):
        append_both(cache, orc, 0, kd[0], kv[0], vd[0], vv[0], t, tc)
        t = tc
        q = syn.queries(200 + i, (1, wl.n_q_heads, 128))
        out = cache.decode(0, torch.from_numpy(q).cuda()).cpu().numpy()
        worst = max(worst, max_head_rel_err(out, orc.decode(0, q.astype(np.float64))))
    print(f"\nr_K=24/r_V=40: worst attention rel err {worst:.3e}")
    assert worst <= ATTN_TOL
    assert cache.status() == 0


@pytest.mark.parametrize("variant,wl_id", [("gapped", 1), ("literal", 1), ("gapped", 3),
                                            ("gapped", 4)])
def test_bf16_coordinates_fold_one_step_parity(variant, wl_id):
    """bf16 coordinates: each GPU fold, started from the GPU's own state, stores the oracle's
    rounded coordinates where the subspace is gapped; Sigma and the basis (fp32) match as in the
    fp32 mode.

    The device rounds its fp32 coordinates c_dev to nearest even, and c_dev differs from the exact
    coordinates c by the fp32 fold error, at most a subspace-angle error times the row norm. So
    |stored - c| <= 2^-8 |stored| + PROJ_TOL * |row of c|: the first term is half a bf16 step,
    the second the fp32 error. Truncation or a one-step rounding error breaks the first term for
    about half of all entries. Rounding decisions can still differ where c_dev and c fall on the
    two sides of a rounding midpoint. The expected fraction of such entries is about the fp32
    error over the bf16 step (a few percent), and it is bounded at 10 %."""
    from oracle import round_bf16
    base = syn.WORKLOADS[wl_id]
    T = 1100 if wl_id != 4 else 2100
    wl = sub(base, batch=1, n_layers=1, n_kv_heads=2, n_q_heads=8, tokens=T, prefill=0)
    kd, kv, vd, vv = workload_arrays(wl, variant=variant)
    cache = make_cache(wl, coord_bf16=True)
    t, folds = 0, 0
    worst = {"sigma": 0.0, "proj": 0.0, "mismatch": 0.0, "excess": 0.0, "bias": 0.0}
    while True:
        nc = n_compressed(t, wl.block, wl.window)
        t_fold = nc + wl.window + wl.block
        if t_fold > wl.tokens:
            break
        before = _snapshot(cache, wl)
        cache.append(0, to_device(kd[0][:, :, t:t_fold]), to_device(vd[0][:, :, t:t_fold]))
        t = t_fold
        after = _snapshot(cache, wl)
        folds += 1
        for (s_, h, x), (C0, B0, S0, k0, n0) in before.items():
            r = wl.rank_k if x == 0 else wl.rank_v
            F = (kv if x == 0 else vv)[0][s_, h, n0:n0 + wl.block]
            assert np.array_equal(C0, round_bf16(C0))           # stored values are bf16
            Cr, Sr, Br, _ = fold_from_coords(C0[:, :k0], S0[:k0], B0[:, :k0], F, r)
            C1, B1, S1, k1, n1 = after[s_, h, x]
            assert n1 == n0 + wl.block and k1 == Sr.size
            worst["sigma"] = max(worst["sigma"], float((np.abs(S1[:k1] - Sr) / Sr).max()))
            M = np.vstack([C0[:, :k0] @ B0[:, :k0].T, F]) if n0 else F
            sv = np.linalg.svd(M, compute_uv=False)
            if k1 < sv.size and (sv[k1 - 1] - sv[k1]) / sv[0] > GAP:
                worst["proj"] = max(worst["proj"], projector_err(B1[:, :k1], Br))
                E = round_bf16(Cr)
                got = C1[:, :k1].copy()
                # columns past the old rank have no sign convention: align them first
                for c in range(k0, k1):
                    if float(got[:, c] @ E[:, c]) < 0:
                        got[:, c] = -got[:, c]
                row = np.linalg.norm(Cr, axis=1, keepdims=True)
                bound = 2.0 ** -8 * np.abs(got) + PROJ_TOL * row + 1e-30
                worst["excess"] = max(worst["excess"], float((np.abs(got - Cr) / bound).max()))
                worst["mismatch"] = max(worst["mismatch"], float(np.mean(got != E)))
                # round to nearest leaves no bias toward zero relative to the bf16 step; truncation
                # would give about -0.7 here (error uniform over one step, toward zero)
                bias = float(np.sum(np.sign(got) * (got - Cr)) / (2.0 ** -8 * np.sum(np.abs(got))))
                worst["bias"] = max(worst["bias"], abs(bias))
    print(f"\nbf16 coordinates {variant} cfg {wl_id}: {folds} folds, worst {worst}")
    assert worst["sigma"] <= SIG_TOL and worst["proj"] <= PROJ_TOL
    assert worst["excess"] <= 1.0 and worst["mismatch"] <= 0.1 and worst["bias"] <= 0.25
    assert cache.status() == 0


@pytest.mark.parametrize("wl_id,tokens,key_scale", [(1, 4096, 1.0), (1, 4096, 8.0), (3, 1500, 1.0),
                                                    (4, 2148, 1.0), (2, 1500, 1.0)])
def test_bf16_coordinates_decode_parity(wl_id, tokens, key_scale):
    """bf16 coordinates: streamed decode (fused append + decode, look-ahead folds) against the
    oracle's bf16-coordinate stream at several lengths, on the shapes of the workloads."""
    base = syn.WORKLOADS[wl_id]
    wl = sub(base, batch=1, n_layers=1, n_kv_heads=2, n_q_heads=8, tokens=tokens, prefill=0)
    kd, kv, vd, vv = workload_arrays(wl, key_scale=key_scale)
    cache = make_cache(wl, coord_bf16=True, lookahead_folds=True)
    orc = make_oracle(wl, coord_bf16=True)
    orc64 = make_oracle(wl)
    K, V = to_device(kd[0]), to_device(vd[0])
    n0 = min(tokens - 200, 1000)
    append_both(cache, orc, 0, kd[0], kv[0], vd[0], vv[0], 0, n0)
    orc64.append(0, kv[0][:, :, :n0], vv[0][:, :, :n0])
    worst = worst_dev = 0.0
    for t in range(n0, tokens):
        q = syn.queries(5000 + t, (1, wl.n_q_heads, 128))
        out = cache.append_decode(0, K[:, :, t:t + 1].contiguous(), V[:, :, t:t + 1].contiguous(),
                                  torch.from_numpy(q).cuda())
        orc.append(0, kv[0][:, :, t:t + 1], vv[0][:, :, t:t + 1])
        orc64.append(0, kv[0][:, :, t:t + 1], vv[0][:, :, t:t + 1])
        if t % 37 == 0 or t == tokens - 1:
            got = out.cpu().numpy()
            q64 = q.astype(np.float64)
            worst = max(worst, _bf16_excess(got, orc.decode(0, q64), orc64.decode(0, q64)))
            # the decode alone: float64 attention over the device's own (bf16) state
            ref = np.stack([_attention_over_device_state(cache, wl, 0, 0, h, K[0, h], V[0, h],
                                                         q[0, h * wl.group:(h + 1) * wl.group]
                                                         .astype(np.float64))[0]
                            for h in range(wl.n_kv_heads)]).reshape(1, wl.n_q_heads, 128)
            worst_dev = max(worst_dev, max_head_rel_err(got, ref))
    print(f"\nbf16 coordinates cfg {wl_id} x{key_scale}: excess over the oracle's own bf16 "
          f"rounding {worst:.3e}, {worst_dev:.3e} vs the device state")
    assert worst_dev <= ATTN_TOL
    assert worst <= ATTN_TOL
    for x in (0, 1):
        rec = cache.reconstruct(0, x).cpu().numpy()[0, 0]
        u = orc.unit(0, 0, 0, x)
        assert rel_err(rec[u.n:], u.reconstruct()[u.n:]) == 0.0     # window rows exact
    assert cache.status() == 0


def test_bf16_coordinates_storage_bytes():
    """The storage count uses 2-byte coordinates and fp32 bases and Sigma."""
    wl = sub(W1, n_kv_heads=2, n_q_heads=8, tokens=900)
    kd, kv, vd, vv = workload_arrays(wl)
    a, b = make_cache(wl), make_cache(wl, coord_bf16=True)
    orc = make_oracle(wl, coord_bf16=True)
    for c in (a, b):
        c.append(0, to_device(kd[0]), to_device(vd[0]))
    orc.append(0, kv[0], vv[0])
    expect = sum(orc.unit(0, 0, h, x).storage_bytes(2) for h in range(2) for x in (0, 1))
    assert b.storage_bytes(0) == expect
    n = orc.unit(0, 0, 0, 0).n
    assert a.storage_bytes(0) - b.storage_bytes(0) == 2 * 2 * n * (wl.rank_k + wl.rank_v)


def test_two_sequences_two_layers_fused_steps_with_lookahead():
    """Batch 2 x 2 layers x 2 kv-heads, every token one fused step per layer with look-ahead
    folds (one internal stream per layer): every layer's decode matches the oracle at several
    lengths, and reconstructed keys with RoPE match the oracle's rotated keys."""
    wl = sub(W1, batch=2, n_layers=2, n_kv_heads=2, n_q_heads=8, tokens=700)
    kd, kv, vd, vv = workload_arrays(wl, variant="gapped")  # well-defined subspaces
    cache, orc = make_cache(wl, lookahead_folds=True), make_oracle(wl)
    K, V = to_device(kd), to_device(vd)                     # [L][S][H][T][D]
    checkpoints, worst = {321, 450, 700}, 0.0
    for t in range(wl.tokens):
        for l in range(wl.n_layers):
            q = syn.queries(1000 + 10 * t + l, (wl.batch, wl.n_q_heads, 128))
            out = cache.append_decode(l, K[l][:, :, t:t + 1].contiguous(),
                                      V[l][:, :, t:t + 1].contiguous(), torch.from_numpy(q).cuda())
            orc.append(l, kv[l][:, :, t:t + 1], vv[l][:, :, t:t + 1])
            if t + 1 in checkpoints:
                err = max_head_rel_err(out.cpu().numpy(), orc.decode(l, q.astype(np.float64)))
                worst = max(worst, err)
    print(f"\nbatch 2 x 2 layers, fused steps: worst attention rel err {worst:.3e}")
    assert worst <= ATTN_TOL
    for l in range(wl.n_layers):
        rk = cache.reconstruct(l, 0, apply_rope=True).cpu().numpy()
        for s in range(wl.batch):
            for h in range(wl.n_kv_heads):
                kref, _ = orc.keys_values(l, s, h)
                assert rel_err(rk[s, h], kref) <= 1e-3
    assert cache.status() == 0


@pytest.mark.parametrize("variant", ["gapped", "literal"])
def test_large_blocks_fold_through_their_triangular_factor(variant):
    """Long-context shapes (b = 512, w = 512, r_K = 64, r_V = 96): blocks above 128 rows are
    folded through the 128-row triangular factor of the block. A 2048-row prefill (3 folds) plus
    100 streamed tokens: Sigma, projectors (gapped rows) and decode match the oracle."""
    base = syn.WORKLOADS[4]
    wl = sub(base, batch=1, n_layers=1, n_kv_heads=2, n_q_heads=8, tokens=2148, prefill=2048)
    kd, kv, vd, vv = workload_arrays(wl, variant=variant)
    cache, orc = make_cache(wl, lookahead_folds=True), make_oracle(wl)
    append_both(cache, orc, 0, kd[0], kv[0], vd[0], vv[0], 0, 2048)
    K, V = to_device(kd[0]), to_device(vd[0])
    worst = 0.0
    for t in range(2048, wl.tokens):
        q = syn.queries(3000 + t, (1, wl.n_q_heads, 128))
        out = cache.append_decode(0, K[:, :, t:t + 1].contiguous(), V[:, :, t:t + 1].contiguous(),
                                  torch.from_numpy(q).cuda())
        orc.append(0, kv[0][:, :, t:t + 1], vv[0][:, :, t:t + 1])
        if t % 25 == 0 or t == wl.tokens - 1:
            worst = max(worst, max_head_rel_err(out.cpu().numpy(), orc.decode(0, q.astype(np.float64))))
    print(f"\nb=512 {variant}: worst attention rel err {worst:.3e}")
    assert worst <= ATTN_TOL
    for h in range(2):
        for x in (0, 1):
            C, B, S, k, n = cache.factors(0, 0, h, x)
            u = orc.unit(0, 0, h, x)
            assert k == u.k and n == u.n == 1536
            if variant == "gapped":
                S, B = S.cpu().numpy(), B.cpu().numpy()
                assert np.max(np.abs(S[:k] - u.sigma) / u.sigma) <= SIG_TOL
                assert projector_err(B[:, :k], u.B) <= PROJ_TOL
    assert cache.status() == 0


def _unit_oracle(wl, K, V, cbf=False):
    """Float64 oracle of one (sequence, kv-head) unit fed the unit's rows as they are on the device
    (bf16 values, exact in float64)."""
    orc = OracleCache(1, 1, 1, wl.group, 128, wl.rank_k, wl.rank_v, wl.block, wl.window,
                      rope=True, rope_theta=wl.rope_theta, coord_bf16=cbf)
    orc.append(0, K.float().cpu().numpy().astype(np.float64)[None, None],
               V.float().cpu().numpy().astype(np.float64)[None, None])
    return orc


def _bf16_excess(got, ref_b, ref_f):
    """bf16 coordinates, end to end: every fold re-rounds every coordinate, and fp32 (device) and
    float64 (oracle) arithmetic put a few values on different sides of a rounding boundary, after
    which the two bf16 streams carry independent rounding errors. Their difference is not a
    parity measure; the device's bf16 cache must instead stay as close to the float64 cache as
    the oracle's own bf16 cache does: err(device, float64) <= 2 err(oracle bf16, float64) + tol.
    Returns err(device, float64) - 2 err(oracle bf16, float64), to compare with the tolerance."""
    return max_head_rel_err(got, ref_f) - 2.0 * max_head_rel_err(ref_b, ref_f)


def _sampled_unit_check(wl, q, out, units, cbf=False):
    """Oracle run on single (sequence, kv-head) units of a full-size cache, compared on their
    q-heads. Returns (worst error, the units' oracles, their float64-coordinate oracles). With
    bf16 coordinates the error is the excess of _bf16_excess."""
    G = wl.group
    worst, oracles, oracles64 = 0.0, [], []
    for sq, h, K, V in units:
        orc = _unit_oracle(wl, K, V, cbf)
        orc64 = _unit_oracle(wl, K, V, False) if cbf else orc
        qs = q[sq, h * G:(h + 1) * G].cpu().numpy().astype(np.float64)[None]
        got = out[sq, h * G:(h + 1) * G].cpu().numpy()[None]
        if cbf:
            err = _bf16_excess(got, orc.decode(0, qs), orc64.decode(0, qs))
        else:
            err = max_head_rel_err(got, orc.decode(0, qs))
        worst = max(worst, err)
        oracles.append(orc)
        oracles64.append(orc64)
    return worst, oracles, oracles64


def _sharp(keys_rot, positions, logit=20.0):
    """Queries aligned with the (rotated) keys at `positions`, scaled so that each one's own logit
    q.k / sqrt(d) is `logit`: sharp attention that peaks on those positions."""
    return np.stack([keys_rot[p] * (logit * math.sqrt(128) / float(keys_rot[p] @ keys_rot[p]))
                     for p in positions])


def _attention_over_device_state(cache, wl, layer, seq, head, K, V, qs):
    """Float64 attention (the oracle's RoPE and softmax) over the cache's own state: compressed rows
    C B^T from the device factors promoted to float64, window rows exact. Isolates the decode
    kernels from the fold trajectory (one-step parity of the decode)."""
    from oracle import attention, rope
    t = cache.tokens(layer)
    rows = []
    for x, X in ((0, K), (1, V)):
        C, B, _, k, n = cache.factors(layer, seq, head, x)
        C = C.cpu().numpy().astype(np.float64)[:, :k]
        B = B.cpu().numpy().astype(np.float64)[:, :k]
        ex = X[n:t].float().cpu().numpy().astype(np.float64)
        rows.append(np.vstack([C @ B.T, ex]) if n else ex)
    Kr = rope(rows[0], np.arange(t), wl.rope_theta)
    return np.stack([attention(qg, Kr, rows[1]) for qg in qs]), Kr


def _sharp_checks(cache, wl, layer, units, positions, rng_seed, oracles64=None):
    """Sharp-softmax decode parity on sampled units of a full-size cache. Every q-head of a sampled
    unit gets a query aligned with one of `positions` (logit 20); the other units get random
    queries. Compares each sampled q-head with (a) float64 attention over the device state and
    (b) the unit's own float64 oracle stream. Returns the worst errors (a, b)."""
    S, QH, G = wl.batch, wl.n_q_heads, wl.group
    gen = torch.Generator(device="cuda")
    gen.manual_seed(rng_seed)
    q = torch.randn((S, QH, 128), generator=gen, device="cuda")
    refs = []
    for sq, h, K, V, orc in units:
        kref, _ = orc.keys_values(0, 0, 0)
        qs = _sharp(kref, positions)
        q[sq, h * G:(h + 1) * G] = torch.from_numpy(qs.astype(np.float32)).cuda()
        refs.append(qs)
    out = cache.decode(layer, q)
    assert cache.status() == 0 and bool(torch.isfinite(out).all())
    wa = wb = 0.0
    for i, ((sq, h, K, V, orc), qs) in enumerate(zip(units, refs)):
        qs32 = q[sq, h * G:(h + 1) * G].cpu().numpy().astype(np.float64)
        got = out[sq, h * G:(h + 1) * G].cpu().numpy()[None]
        ref_a, _ = _attention_over_device_state(cache, wl, layer, sq, h, K, V, qs32)
        wa = max(wa, max_head_rel_err(got, ref_a[None]))
        if oracles64 is None:
            wb = max(wb, max_head_rel_err(got, orc.decode(0, qs32[None])))
        else:
            wb = max(wb, _bf16_excess(got, orc.decode(0, qs32[None]),
                                      oracles64[i].decode(0, qs32[None])))
    return wa, wb


def test_32_layer_workload_full_size_sampled_units():
    """The 32-layer x 8 kv-head workload at its full length (16384 tokens, b=64, w=128, r_K=24,
    r_V=40), all layers appended in one call as the benchmark does; two sampled (layer, kv-head)
    units of the decode match the oracle run on their rows alone."""
    wl = syn.WORKLOADS[2]
    L, S, H, T = wl.n_layers, wl.batch, wl.n_kv_heads, wl.tokens
    cache = make_cache(wl)
    K = torch.empty((L, S, H, T, 128), dtype=torch.bfloat16, device="cuda")
    V = torch.empty_like(K)
    for l in range(L):
        for h in range(H):
            K[l, 0, h] = syn.device_rows(wl, 0, l, h, 0)
            V[l, 0, h] = syn.device_rows(wl, 0, l, h, 1)
    cache.append(-1, K, V)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(2024)
    worst, sa, sb = 0.0, 0.0, 0.0
    for l, h in ((0, 3), (31, 6)):
        q = torch.randn((S, wl.n_q_heads, 128), generator=gen, device="cuda")
        out = cache.decode(l, q)
        assert bool(torch.isfinite(out).all())
        err, (orc,), _ = _sampled_unit_check(wl, q, out, [(0, h, K[l, 0, h], V[l, 0, h])])
        worst = max(worst, err)
        # sharp attention (logit 20) on compressed rows early, mid and late, and a window row
        a, b = _sharp_checks(cache, wl, l, [(0, h, K[l, 0, h], V[l, 0, h], orc)],
                             [5, 9000, 16250, 16300], 77 + l)
        sa, sb = max(sa, a), max(sb, b)
    print(f"\n32-layer workload, sampled units: worst attention rel err {worst:.3e}; sharp: "
          f"{sa:.3e} vs device state, {sb:.3e} vs oracle stream")
    assert worst <= ATTN_TOL and sa <= ATTN_TOL and sb <= ATTN_TOL
    assert cache.status() == 0
    cache.close()


@pytest.mark.parametrize("cbf", [False, True])
def test_long_prefill_full_size_sampled_unit(cbf):
    """The long-context layer at its full prefill (batch 4 x 8 kv-heads, 65536 rows in one
    append, b = 512, w = 512, r_K = 64, r_V = 96): one sampled unit of the decode matches the
    oracle run on its rows alone."""
    wl = syn.WORKLOADS[4]
    S, H, T0 = wl.batch, wl.n_kv_heads, wl.prefill
    cache = make_cache(sub(wl, n_layers=1), coord_bf16=cbf)
    K = torch.empty((S, H, T0, 128), dtype=torch.bfloat16, device="cuda")
    V = torch.empty_like(K)
    for sq in range(S):
        for h in range(H):
            K[sq, h] = syn.device_rows(wl, sq, 0, h, 0, T=T0)
            V[sq, h] = syn.device_rows(wl, sq, 0, h, 1, T=T0)
    cache.append(0, K, V)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(4242)
    q = torch.randn((S, wl.n_q_heads, 128), generator=gen, device="cuda")
    out = cache.decode(0, q)
    assert cache.status() == 0 and bool(torch.isfinite(out).all())
    err, (orc,), (orc64,) = _sampled_unit_check(wl, q, out, [(2, 5, K[2, 5], V[2, 5])], cbf)
    # sharp attention on compressed rows past 60K (n_c = 65024) and on a window row
    sa, sb = _sharp_checks(cache, wl, 0, [(2, 5, K[2, 5], V[2, 5], orc)],
                           [60001, 62500, 64999, 65300], 4343, [orc64] if cbf else None)
    print(f"\nlong prefill, sampled unit: attention rel err {err:.3e}; sharp: {sa:.3e} vs "
          f"device state, {sb:.3e} vs oracle stream")
    assert err <= ATTN_TOL and sa <= ATTN_TOL and sb <= ATTN_TOL
    cache.close()


# ------------------------------------------------------------------------------------------------
def _prefill_rows(wl, planted_chunks, chunk, variant="literal"):
    """Rows of one (sequence, kv-head) unit per head with a common key direction in the slowest
    RoPE pair (channels 63 and 127), so chunk scores are near 1, and one reversed key in each
    planted chunk (its chunk scores near -1): the outlier chunks are unambiguous in fp32 and
    fp64."""
    kd, kv, vd, vv = workload_arrays(wl, variant=variant)
    K = kv[0].copy()                                   # [S][H][T][D] float64 (bf16 values)
    off = np.zeros(128)
    off[63], off[127] = 0.8, 0.6
    K = K + off * np.abs(K).max()
    for c in planted_chunks:
        K[:, :, c * chunk + chunk // 2] *= -1.0
    kbits, kvals = syn.to_bf16(K)
    return kbits[None], kvals[None], vd, vv


@pytest.mark.parametrize("cbf,variant", [(False, "gapped"), (False, "literal"), (True, "literal")])
def test_prefill_with_protection_matches_oracle(cbf, variant):
    """Prefill Compression on the long-context shapes (b = 512, w = 512, r_V = 96; r_K = 64 with
    bf16 coordinates, 32 with fp32 coordinates, whose protected decode takes r_K <= 32):
    protected key chunks and their value neighbourhoods stay exact, the other rows before the
    window get one truncated SVD, later tokens fold from the window; reconstructions and decode
    match the oracle's prefill."""
    base = syn.WORKLOADS[4]
    wl = sub(base, batch=1, n_layers=1, n_kv_heads=2, n_q_heads=8, tokens=4300, prefill=3000,
             rank_k=base.rank_k if cbf else 32)
    chunk, m, suffix, rho = 32, 3, 40, 2
    kd, kv, vd, vv = _prefill_rows(wl, [5, 31, 60], chunk, variant)
    T0 = wl.prefill
    cache = make_cache(wl, coord_bf16=cbf, lookahead_folds=True, prot_cap=512)
    orc = make_oracle(wl, coord_bf16=cbf)
    orc64 = make_oracle(wl) if cbf else orc
    K, V = to_device(kd[0]), to_device(vd[0])
    cache.prefill(0, K[:, :, :T0].contiguous(), V[:, :, :T0].contiguous(),
                  protect=(chunk, m, suffix, rho))
    orc.prefill(0, kv[0][:, :, :T0], vv[0][:, :, :T0], chunk, m, suffix, rho)
    if cbf:
        orc64.prefill(0, kv[0][:, :, :T0], vv[0][:, :, :T0], chunk, m, suffix, rho)
    assert cache.tokens(0) == T0 and cache.status() == 0
    end = T0 - wl.window
    for x, vals in ((0, kv), (1, vv)):
        rec = cache.reconstruct(0, x).cpu().numpy()[0]
        for h in range(2):
            u = orc.unit(0, 0, h, x)
            prot = u.prot_pos
            if x == 0:
                planted = set()
                for c in (5, 31, 60):
                    planted.update(range(c * chunk, (c + 1) * chunk))
                planted.update(range(end - suffix, end))
                assert set(prot.tolist()) == planted
            # protected and window rows are the exact rows, bit for bit
            assert np.array_equal(rec[h][prot], vals[0][0, h][prot].astype(np.float32))
            assert np.array_equal(rec[h][end:], vals[0][0, h][end:T0].astype(np.float32))
            comp = u.comp_pos
            err = rel_err(rec[h][comp], u.reconstruct()[comp])
            if variant == "gapped":
                assert err <= 1e-3, err
    worst = 0.0
    for t in range(T0, wl.tokens):
        q = syn.queries(7000 + t, (1, wl.n_q_heads, 128))
        out = cache.append_decode(0, K[:, :, t:t + 1].contiguous(), V[:, :, t:t + 1].contiguous(),
                                  torch.from_numpy(q).cuda())
        orc.append(0, kv[0][:, :, t:t + 1], vv[0][:, :, t:t + 1])
        if cbf:
            orc64.append(0, kv[0][:, :, t:t + 1], vv[0][:, :, t:t + 1])
        if t % 97 == 0 or t == T0 or t == wl.tokens - 1:
            q64 = q.astype(np.float64)
            if cbf:
                worst = max(worst, _bf16_excess(out.cpu().numpy(), orc.decode(0, q64),
                                                orc64.decode(0, q64)))
            else:
                worst = max(worst, max_head_rel_err(out.cpu().numpy(), orc.decode(0, q64)))
    print(f"\nprefill with protection ({variant}, bf16 coords {cbf}): worst attention rel err "
          f"{worst:.3e}, folds after the prefill {orc.unit(0, 0, 0, 0).folds - 1}")
    assert orc.unit(0, 0, 0, 0).folds >= 3
    assert worst <= ATTN_TOL
    assert cache.status() == 0


def test_prefill_without_protection_is_the_truncated_svd():
    """No protection: every row before the window enters one truncated SVD (rank r); its
    singular values and subspace match the library SVD of those rows (gapped rows)."""
    base = syn.WORKLOADS[4]
    wl = sub(base, batch=1, n_layers=1, n_kv_heads=2, n_q_heads=8, tokens=2600, prefill=2600)
    kd, kv, vd, vv = workload_arrays(wl, variant="gapped")
    cache = make_cache(wl, prot_cap=1)
    cache.prefill(0, to_device(kd[0]), to_device(vd[0]))
    end = wl.prefill - wl.window
    for x, vals in ((0, kv), (1, vv)):
        r = wl.rank_k if x == 0 else wl.rank_v
        for h in range(2):
            C, B, S, k, n = cache.factors(0, 0, h, x)
            assert n == end and k == r
            X = vals[0][0, h][:end]
            sv = np.linalg.svd(X, compute_uv=False)
            Vt = np.linalg.svd(X, full_matrices=False)[2]
            S = S.cpu().numpy()
            assert np.max(np.abs(S[:k] - sv[:k]) / sv[:k]) <= SIG_TOL
            assert projector_err(B.cpu().numpy()[:, :k], Vt[:k].T) <= PROJ_TOL
    assert cache.status() == 0
