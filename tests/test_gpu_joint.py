"""GPU parity of the joint per-layer factorisation (``joint_heads=1``: all kv-heads of a (layer,
sequence) in one factorisation over rows of length n_kv 128; iS-KV summary, "Reconstruction and
Storage", per-layer storage) against the float64 oracle's joint mode, through the C ABI.

Inputs: each (layer, sequence, path) draws its kv-heads' rows as one low-rank-plus-noise matrix
of n_kv 128 columns (``iskv_synth.joint_workload_rows``), so the heads share dominant
directions. Tolerances as in the per-head tests: singular values <= 1e-4 relative, projector
<= 1e-3 where the spectrum is gapped at the kept rank, attention <= 2e-3 per q-head.
"""
import dataclasses

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import iskv_synth as syn  # noqa: E402
from gpu_harness import (joint_workload_arrays, max_head_rel_err, projector_err,  # noqa: E402
                         rel_err, to_device)
from oracle import OracleCache, fold_from_coords, n_compressed  # noqa: E402

pytestmark = pytest.mark.gpu

SIG_TOL, PROJ_TOL, ATTN_TOL, GAP = 1e-4, 1e-3, 2e-3, 1e-2
# Llama-3-8B-shaped layer: 8 kv / 32 q heads, b = 64, w = 256, r_K = 32, r_V = 48
W1 = syn.WORKLOADS[1]


@pytest.fixture(autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def sub(wl, **kw):
    return dataclasses.replace(wl, **kw)


def make_cache(wl, **kw):
    from rank_kv_cache_isvd_b200.cache import IsKVCache
    args = dict(batch=wl.batch, n_layers=wl.n_layers, n_kv_heads=wl.n_kv_heads,
                n_q_heads=wl.n_q_heads, rank_k=wl.rank_k, rank_v=wl.rank_v, block=wl.block,
                window=wl.window, max_tokens=wl.tokens, kv_dtype=wl.kv_dtype, rope=wl.rope,
                rope_theta=wl.rope_theta, joint_heads=True)
    args.update(kw)
    return IsKVCache(**args)


def make_oracle(wl, coord_bf16=False):
    return OracleCache(wl.batch, wl.n_layers, wl.n_kv_heads, wl.n_q_heads, wl.head_dim,
                       wl.rank_k, wl.rank_v, wl.block, wl.window, rope=wl.rope,
                       rope_theta=wl.rope_theta, coord_bf16=coord_bf16, joint=True)


def joint_factors(cache, wl, layer, s, x):
    """``(C, B, sigma, k, n)`` of a joint unit; B stacks the kv-heads' 128-row slices."""
    C, _, S, k, n = cache.factors(layer, s, 0, x)
    B = np.vstack([cache.factors(layer, s, h, x)[1].cpu().numpy()
                   for h in range(wl.n_kv_heads)]).astype(np.float64)
    return C.cpu().numpy().astype(np.float64), B, S.cpu().numpy().astype(np.float64), k, n


@pytest.mark.parametrize("variant", ["gapped", "literal"])
def test_joint_fold_one_step_parity(variant):
    """Each joint fold, started from the GPU's own state, matches the oracle's fold of the
    concatenated rows (d = 4 x 128)."""
    wl = sub(W1, n_kv_heads=4, n_q_heads=16, tokens=1100)
    kd, kv, vd, vv = joint_workload_arrays(wl, variant=variant)
    cache = make_cache(wl)
    t, folds, worst = 0, 0, {"sigma": 0.0, "proj": 0.0, "recon": 0.0, "orth": 0.0}
    while True:
        nc = n_compressed(t, wl.block, wl.window)
        t_fold = nc + wl.window + wl.block
        if t_fold > wl.tokens:
            break
        before = {x: joint_factors(cache, wl, 0, 0, x) for x in (0, 1)}
        cache.append(0, to_device(kd[0][:, :, t:t_fold]), to_device(vd[0][:, :, t:t_fold]))
        t = t_fold
        folds += 1
        for x in (0, 1):
            C0, B0, S0, k0, n0 = before[x]
            r = wl.rank_k if x == 0 else wl.rank_v
            F = np.concatenate(list((kv if x == 0 else vv)[0][0, :, n0:n0 + wl.block]), axis=1)
            Cr, Sr, Br, _ = fold_from_coords(C0[:, :k0], S0[:k0], B0[:, :k0], F, r)
            C1, B1, S1, k1, n1 = joint_factors(cache, wl, 0, 0, x)
            assert n1 == n0 + wl.block and k1 == Sr.size
            worst["sigma"] = max(worst["sigma"], float((np.abs(S1[:k1] - Sr) / Sr).max()))
            M = np.vstack([C0[:, :k0] @ B0[:, :k0].T, F]) if n0 else F
            sv = np.linalg.svd(M, compute_uv=False)
            gapped = k1 < sv.size and (sv[k1 - 1] - sv[k1]) / sv[0] > GAP
            rec = rel_err(C1[:, :k1] @ B1[:, :k1].T, Cr @ Br.T)
            if gapped:
                worst["proj"] = max(worst["proj"], projector_err(B1[:, :k1], Br))
                worst["recon"] = max(worst["recon"], rec)
            worst["orth"] = max(worst["orth"],
                                float(np.abs(B1[:, :k1].T @ B1[:, :k1] - np.eye(k1)).max()))
            assert not B1[:, k1:].any()
    print(f"\n{variant}: {folds} joint folds, worst {worst}")
    assert folds == n_compressed(wl.tokens, wl.block, wl.window) // wl.block
    assert worst["sigma"] <= SIG_TOL
    assert worst["proj"] <= PROJ_TOL
    assert worst["recon"] <= SIG_TOL
    assert worst["orth"] <= 5e-5
    assert cache.status() == 0


@pytest.mark.parametrize("key_scale", [1.0, 8.0])
def test_joint_decode_parity_llama_layer(key_scale):
    """Llama-3-8B-shaped layer with one factorisation over its 8 kv-heads (d = 1024): decode
    before any fold, at fold boundaries and after many folds."""
    wl = sub(W1, tokens=2100)
    kd, kv, vd, vv = joint_workload_arrays(wl, key_scale=key_scale)
    cache, orc = make_cache(wl), make_oracle(wl)
    t, worst = 0, 0.0
    for i, tc in enumerate([1, 255, 320, 321, 700, 1500, 2100]):
        cache.append(0, to_device(kd[0][:, :, t:tc]), to_device(vd[0][:, :, t:tc]))
        orc.append(0, kv[0][:, :, t:tc], vv[0][:, :, t:tc])
        t = tc
        assert cache.tokens(0) == t
        q = syn.queries(300 + i, (1, wl.n_q_heads, 128))
        out = cache.decode(0, torch.from_numpy(q).cuda()).cpu().numpy()
        worst = max(worst, max_head_rel_err(out, orc.decode(0, q.astype(np.float64))))
    print(f"\nkey_scale={key_scale}: worst attention rel err {worst:.3e}")
    assert worst <= ATTN_TOL
    for x in (0, 1):
        _, _, _, k, n = cache.factors(0, 0, 3, x)
        u = orc.unit(0, 0, 3, x)
        assert n == u.n == 1792 and k == u.k == (32 if x == 0 else 48)
    assert cache.status() == 0


def test_joint_gapped_sigma_projector_and_storage():
    wl = sub(W1, n_kv_heads=2, n_q_heads=8, tokens=1600)
    kd, kv, vd, vv = joint_workload_arrays(wl, variant="gapped")
    cache, orc = make_cache(wl), make_oracle(wl)
    cache.append(0, to_device(kd[0]), to_device(vd[0]))
    orc.append(0, kv[0], vv[0])
    for x in (0, 1):
        _, B, S, k, n = joint_factors(cache, wl, 0, 0, x)
        u = orc.unit(0, 0, 0, x)
        assert k == u.k and n == u.n
        assert np.max(np.abs(S[:k] - u.sigma) / u.sigma) <= SIG_TOL
        assert projector_err(B[:, :k], u.B) <= PROJ_TOL
    # "Reconstruction and Storage": one factorisation per (layer, sequence) and path, d = 2 x 128
    expect = sum(orc.unit(0, 0, 0, x).storage_bytes(2) for x in (0, 1))
    assert cache.storage_bytes(0) == expect
    q = syn.queries(31, (1, 8, 128))
    out = cache.decode(0, torch.from_numpy(q).cuda()).cpu().numpy()
    assert max_head_rel_err(out, orc.decode(0, q.astype(np.float64))) <= ATTN_TOL
    assert cache.status() == 0


def test_joint_two_layers_two_sequences_lookahead_and_persistent_decode():
    """Joint units of several layers and sequences; look-ahead folds equal synchronous folds
    bitwise; a call large enough for the persistent decode (16 kv-head units x 24 tiles with
    bf16 coordinates) matches float64 attention over the device's own factors."""
    wl = sub(W1, batch=2, n_layers=2, n_kv_heads=8, n_q_heads=32, tokens=3000)
    kd, kv, vd, vv = joint_workload_arrays(wl)
    a, b = make_cache(wl), make_cache(wl, lookahead_folds=True)
    orc = make_oracle(wl)
    for layer in (0, 1):
        for c in (a, b):
            c.append(layer, to_device(kd[layer][:, :, :1900]), to_device(vd[layer][:, :, :1900]))
            for t in range(1900, 2000):
                c.append(layer, to_device(kd[layer][:, :, t:t + 1]),
                         to_device(vd[layer][:, :, t:t + 1]))
        orc.append(layer, kv[layer][:, :, :2000], vv[layer][:, :, :2000])
    for layer in (0, 1):
        q = syn.queries(40 + layer, (2, 32, 128))
        qa = torch.from_numpy(q).cuda()
        oa = a.decode(layer, qa).cpu().numpy()
        ob = b.decode(layer, qa).cpu().numpy()
        assert np.array_equal(oa, ob)
        assert max_head_rel_err(oa, orc.decode(layer, q.astype(np.float64))) <= ATTN_TOL
        for s in range(2):
            for x in (0, 1):
                Ca, Ba, Sa, ka, na = joint_factors(a, wl, layer, s, x)
                Cb, Bb, Sb, kb, nb = joint_factors(b, wl, layer, s, x)
                assert ka == kb and na == nb
                assert np.array_equal(Ca, Cb) and np.array_equal(Ba, Bb)
    assert a.status() == 0 and b.status() == 0

    # bf16 coordinates: the persistent decode, against attention over the device state
    c = make_cache(wl, n_layers=1, coord_bf16=True)
    c.append(0, to_device(kd[0]), to_device(vd[0]))
    q = syn.queries(50, (2, 32, 128))
    out = c.decode(0, torch.from_numpy(q).cuda()).cpu().numpy()
    T, G = 3000, 4
    ref = np.zeros_like(out, dtype=np.float64)
    for s in range(2):
        CK, BK, _, kK, n = joint_factors(c, wl, 0, s, 0)
        CV, BV, _, kV, _ = joint_factors(c, wl, 0, s, 1)
        for h in range(8):
            K = np.vstack([CK[:, :kK] @ BK[h * 128:(h + 1) * 128, :kK].T,
                           kv[0][s, h, n:T]])
            V = np.vstack([CV[:, :kV] @ BV[h * 128:(h + 1) * 128, :kV].T,
                           vv[0][s, h, n:T]])
            from oracle import attention, rope
            Kr = rope(K, np.arange(T), wl.rope_theta)
            for g in range(h * G, (h + 1) * G):
                ref[s, g] = attention(q[s, g].astype(np.float64), Kr, V)
    assert max_head_rel_err(out, ref) <= ATTN_TOL
    assert c.status() == 0


@pytest.mark.parametrize("lookahead", [False, True])
def test_joint_fused_append_decode_equals_separate_calls(lookahead):
    """iskv_append_decode in the joint mode gives bit for bit the outputs and reconstructions of
    iskv_append_block + iskv_decode_attn across fold triggers; the reconstruction (kv-head slices
    of the shared factorisation) matches the oracle's."""
    wl = sub(W1, n_kv_heads=2, n_q_heads=8, tokens=700)
    kd, kv, vd, vv = joint_workload_arrays(wl, variant="gapped")
    K, V = to_device(kd[0]), to_device(vd[0])
    Q = torch.from_numpy(syn.queries(61, (wl.tokens, 1, 8, 128))).cuda()
    outs = []
    for fused in (False, True):
        cache = make_cache(wl, lookahead_folds=lookahead)
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
        outs.append((out, [cache.reconstruct(0, x) for x in (0, 1)]))
        cache.close()
    (o0, r0), (o1, r1) = outs
    assert torch.equal(o0, o1)
    assert torch.equal(r0[0], r1[0]) and torch.equal(r0[1], r1[1])
    orc = make_oracle(wl)
    orc.append(0, kv[0], vv[0])
    for x in (0, 1):
        assert rel_err(r0[x].cpu().numpy(), orc.reconstruct(0, x)) <= SIG_TOL


def test_joint_stale_coordinates_mode_matches_oracle():
    """The stale-coordinate ablation on a joint factorisation: Sigma and B as the oracle's joint
    unit with rotate=False, old coordinates unrotated."""
    wl = sub(W1, n_kv_heads=2, n_q_heads=8, tokens=900)
    kd, kv, vd, vv = joint_workload_arrays(wl, variant="gapped")
    cache = make_cache(wl, rotate_history=False)
    orc = OracleCache(wl.batch, wl.n_layers, wl.n_kv_heads, wl.n_q_heads, wl.head_dim,
                      wl.rank_k, wl.rank_v, wl.block, wl.window, rope=wl.rope,
                      rope_theta=wl.rope_theta, rotate=False, joint=True)
    cache.append(0, to_device(kd[0]), to_device(vd[0]))
    orc.append(0, kv[0], vv[0])
    for x in (0, 1):
        u = orc.unit(0, 0, 0, x)
        assert rel_err(cache.reconstruct(0, x).cpu().numpy(), orc.reconstruct(0, x)) <= 1e-3
        _, B, S, k, n = joint_factors(cache, wl, 0, 0, x)
        assert k == u.k and n == u.n
        assert np.max(np.abs(S[:k] - u.sigma) / u.sigma) <= SIG_TOL
    q = syn.queries(71, (1, 8, 128))
    out = cache.decode(0, torch.from_numpy(q).cuda()).cpu().numpy()
    assert max_head_rel_err(out, orc.decode(0, q.astype(np.float64))) <= ATTN_TOL
    assert cache.status() == 0


def test_joint_full_size_layer_sampled_sequence():
    """The bench's joint layer at full size (Qwen3-8B-shaped: batch 8 x 8 kv-heads, 32 q-heads,
    32768 tokens in one append, b = 64, w = 256, r_K = 32, r_V = 64, rows drawn on the GPU): every
    output is finite and the 32 q-heads of a sampled sequence match the oracle's joint unit run on
    that sequence's rows alone."""
    wl = dataclasses.replace(syn.WORKLOADS[3], block=64)
    S, H, T, QH = wl.batch, wl.n_kv_heads, wl.tokens, wl.n_q_heads
    cache = make_cache(sub(wl, n_layers=1))
    K = syn.device_rows_batch(wl, range(S), 0, range(H), 0)
    V = syn.device_rows_batch(wl, range(S), 0, range(H), 1)
    cache.append(0, K, V)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(2024)
    q = torch.randn((S, QH, 128), generator=gen, device="cuda")
    out = cache.decode(0, q).cpu().numpy()
    assert cache.status() == 0 and np.isfinite(out).all() and cache.tokens(0) == T
    sq = 5
    orc = OracleCache(1, 1, H, QH, 128, wl.rank_k, wl.rank_v, wl.block, wl.window, rope=wl.rope,
                      rope_theta=wl.rope_theta, joint=True)
    orc.append(0, K[sq:sq + 1].float().cpu().numpy().astype(np.float64),
               V[sq:sq + 1].float().cpu().numpy().astype(np.float64))
    ref = orc.decode(0, q[sq:sq + 1].cpu().numpy().astype(np.float64))
    err = max_head_rel_err(out[sq:sq + 1], ref)
    print(f"\njoint full size, sequence {sq}: attention rel err {err:.3e}")
    assert err <= ATTN_TOL
    for x in (0, 1):
        _, _, _, k, n = cache.factors(0, sq, 0, x)
        u = orc.unit(0, 0, 0, x)
        assert n == u.n == wl.n_c(T) and k == u.k
    cache.close()
