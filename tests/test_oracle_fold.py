"""Pins of the float64 oracle's block-incremental SVD (no GPU).

Each test ties the oracle to something other than itself: the library SVD of the stacked matrix
that the page says every fold optimises (iS-KV summary, "Block-Incremental Decoding Updates"),
Eckart-Young, exactness without truncation, invariants, and closed forms of the schedule and of
the storage formula ("Reconstruction and Storage").
"""
import numpy as np
import pytest

import iskv_synth as syn
from oracle import OracleUnit, fold, fold_from_coords, n_compressed, residual_basis, svd_r


def _stream(T, d, seed, decay=1.0, noise=1e-3):
    rng = np.random.default_rng(seed)
    G = np.linalg.qr(rng.standard_normal((T, d)))[0] * np.sqrt(T)
    H = np.linalg.qr(rng.standard_normal((d, d)))[0]
    s = np.arange(1, d + 1, dtype=float) ** -decay
    return (G * s) @ H.T + noise * rng.standard_normal((T, d))


def _projector(B):
    return B @ B.T


# ---------------------------------------------------------------------------------------------
# T1: the first fold (k = 0) is the plain truncated SVD of the block
# ---------------------------------------------------------------------------------------------
def test_first_fold_is_truncated_svd_of_block():
    F = _stream(12, 10, 1)
    r = 4
    U, s, B, H, P = fold(np.zeros((0, 0)), np.zeros(0), np.zeros((10, 0)), F, r)
    Ur, sr, Br = svd_r(F, r)
    np.testing.assert_allclose(s, sr, rtol=1e-12)
    np.testing.assert_allclose(_projector(B), _projector(Br), atol=1e-10)
    np.testing.assert_allclose((U * s) @ B.T, (Ur * sr) @ Br.T, atol=1e-12)


# ---------------------------------------------------------------------------------------------
# T2: every fold equals SVD_r([previous reconstruction; F])
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("d,r,b", [(16, 4, 3), (16, 6, 8), (8, 3, 7), (12, 12, 5)])
def test_every_fold_is_svd_of_stacked_rows(d, r, b):
    X = _stream(10 * b, d, 2 + d + r + b, decay=0.7)
    U, s, B = np.zeros((0, 0)), np.zeros(0), np.zeros((d, 0))
    for f in range(10):
        F = X[f * b:(f + 1) * b]
        A = (U * s) @ B.T if U.shape[0] else np.zeros((0, d))
        M = np.vstack([A, F])
        U, s, B, H, P = fold(U, s, B, F, r)
        Um, sm, Bm = svd_r(M, r)
        kp = s.size
        np.testing.assert_allclose(s, sm[:kp], rtol=1e-10, atol=1e-13)
        full = np.linalg.svd(M, compute_uv=False)
        if kp < full.size and (full[kp - 1] - full[kp]) / full[0] > 1e-3:
            np.testing.assert_allclose(_projector(B), _projector(Bm[:, :kp]), atol=1e-9)
        np.testing.assert_allclose((U * s) @ B.T, (Um[:, :kp] * sm[:kp]) @ Bm[:, :kp].T,
                                   atol=1e-9 * max(1.0, full[0]))


def test_unit_schedule_matches_manual_folds():
    d, r, b, w = 8, 3, 4, 6
    X = _stream(50, d, 7)
    unit = OracleUnit(d, r, b, w)
    U, s, B = np.zeros((0, 0)), np.zeros(0), np.zeros((d, 0))
    nf = 0
    for t in range(1, 51):
        unit.append(X[t - 1:t])
        assert unit.n == n_compressed(t, b, w)
        while nf * b < n_compressed(t, b, w):
            U, s, B, _, _ = fold(U, s, B, X[nf * b:(nf + 1) * b], r)
            nf += 1
        np.testing.assert_allclose(unit.sigma, s, rtol=1e-12)
        rec = unit.reconstruct()
        assert rec.shape == (t, d)
        np.testing.assert_array_equal(rec[unit.n:], X[unit.n:t])     # exact window rows


# ---------------------------------------------------------------------------------------------
# T3: Eckart-Young on a single block, and optimality against random rank-r subspaces
# ---------------------------------------------------------------------------------------------
def test_eckart_young_tail_energy_single_block():
    F = _stream(20, 12, 3, decay=0.5, noise=0.05)
    r = 5
    U, s, B, _, _ = fold(np.zeros((0, 0)), np.zeros(0), np.zeros((12, 0)), F, r)
    Fh = (U * s) @ B.T
    err2 = np.linalg.norm(F - Fh) ** 2
    # orthogonal projection: ||F - F^||^2 = ||F||^2 - sum of kept sigma^2
    assert err2 == pytest.approx(np.linalg.norm(F) ** 2 - np.sum(s ** 2), rel=1e-10)
    # tail energy equals the discarded squared singular values (computed from the Gram matrix)
    lam = np.sort(np.linalg.eigvalsh(F.T @ F))[::-1]
    assert err2 == pytest.approx(lam[r:].sum(), rel=1e-8)
    # no random rank-r right subspace does better
    rng = np.random.default_rng(0)
    for _ in range(2000):
        Q = np.linalg.qr(rng.standard_normal((12, r)))[0]
        assert np.linalg.norm(F - F @ Q @ Q.T) ** 2 >= err2 * (1 - 1e-12)


# ---------------------------------------------------------------------------------------------
# T4: no truncation -> the factorisation is the full SVD of all folded rows
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("b,w", [(3, 4), (5, 0), (16, 2)])
def test_no_truncation_is_exact_full_svd(b, w):
    d = 8
    X = _stream(41, d, 11, noise=0.1)
    unit = OracleUnit(d, d, b, w)
    unit.append(X)
    n = unit.n
    assert n == n_compressed(41, b, w)
    np.testing.assert_allclose(unit.reconstruct(), X, atol=1e-12)
    sv = np.linalg.svd(X[:n], compute_uv=False)
    np.testing.assert_allclose(unit.sigma, sv[:unit.k], rtol=1e-11)
    Vt = np.linalg.svd(X[:n], full_matrices=False)[2]
    np.testing.assert_allclose(_projector(unit.B), _projector(Vt[:unit.k].T), atol=1e-10)


# ---------------------------------------------------------------------------------------------
# T5: data of exact rank q <= r reconstructs exactly
# ---------------------------------------------------------------------------------------------
def test_exact_low_rank_reconstructs():
    wl = syn.WORKLOADS[0]
    X = syn.kv_rows(300, 32, 5, 1.0, variant="lowrank", rank=3)
    unit = OracleUnit(32, 5, 16, 20)
    unit.append(X)
    rel = np.linalg.norm(unit.reconstruct() - X) / np.linalg.norm(X)
    assert rel <= 1e-12
    assert wl.head_dim == 128
    # the residual basis of a block that lies inside span(B) is empty
    E, P = residual_basis(X[:16] @ unit.B @ unit.B.T, unit.B)
    assert P.shape[1] == 0 and np.linalg.norm(E) <= 1e-12 * np.linalg.norm(X[:16])


# ---------------------------------------------------------------------------------------------
# T6: orthonormal factors; C^T C = Sigma^2
# ---------------------------------------------------------------------------------------------
def test_factors_orthonormal():
    d = 32
    X = _stream(400, d, 13, decay=0.8, noise=0.01)
    unit = OracleUnit(d, 7, 16, 24)
    unit.append(X)
    I = np.eye(unit.k)
    assert np.abs(unit.B.T @ unit.B - I).max() <= 1e-12
    assert np.abs(unit.U.T @ unit.U - I).max() <= 1e-12
    C = unit.coords()
    np.testing.assert_allclose(C.T @ C, np.diag(unit.sigma ** 2), atol=1e-10 * unit.sigma[0] ** 2)
    assert np.all(np.diff(unit.sigma) <= 0)


# ---------------------------------------------------------------------------------------------
# T7: drift of stale coordinates vs none with rotated coordinates; global error bounds
# ---------------------------------------------------------------------------------------------
def test_drift_stale_vs_rotated():
    d, r, b, w = 32, 6, 16, 16
    X = _stream(16 * 24 + w, d, 17, decay=0.4, noise=0.05)
    sync = OracleUnit(d, r, b, w, rotate=True)
    stale = OracleUnit(d, r, b, w, rotate=False)
    drifts = []
    for f in range(24):
        rows = X[: b + w] if f == 0 else X[b + w + (f - 1) * b: b + w + f * b]
        sync.append(rows)
        stale.append(rows)
        a = sync.reconstruct()[: sync.n]
        s_ = stale.reconstruct()[: stale.n]
        drifts.append(np.linalg.norm(s_ - a) / np.linalg.norm(a))
    # identical basis trajectory
    np.testing.assert_allclose(stale.sigma, sync.sigma, rtol=1e-12)
    np.testing.assert_allclose(stale.B, sync.B, atol=1e-12)
    assert drifts[0] <= 1e-12            # one fold: nothing old to rotate yet
    assert drifts[1] > 1e-3              # second fold: old coordinates are in the old basis
    assert drifts[-1] > drifts[1]        # and the stale history keeps drifting
    n = sync.n
    err = np.linalg.norm(X[:n] - sync.reconstruct()[:n])
    u, s, v = svd_r(X[:n], r)
    opt = np.linalg.norm(X[:n] - (u * s) @ v.T)
    assert err >= opt * (1 - 1e-12)      # no streaming result beats the global SVD_r


def test_error_bounded_by_sum_of_discarded_energy():
    d, r, b = 16, 4, 6
    X = _stream(60, d, 19, decay=0.6, noise=0.05)
    U, s, B = np.zeros((0, 0)), np.zeros(0), np.zeros((d, 0))
    bound = 0.0
    for f in range(10):
        F = X[f * b:(f + 1) * b]
        A = (U * s) @ B.T if U.shape[0] else np.zeros((0, d))
        M2 = np.linalg.norm(A) ** 2 + np.linalg.norm(F) ** 2
        U, s, B, _, _ = fold(U, s, B, F, r)
        bound += np.sqrt(max(M2 - np.sum(s ** 2), 0.0))
        n = (f + 1) * b
        err = np.linalg.norm(X[:n] - (U * s) @ B.T)
        assert err <= bound * (1 + 1e-10) + 1e-12


# ---------------------------------------------------------------------------------------------
# one fold started from stored coordinates equals the fold of the (U, Sigma, B) state
# ---------------------------------------------------------------------------------------------
def test_fold_from_coords_matches_fold():
    d, r, b = 16, 5, 4
    X = _stream(40, d, 23)
    U, s, B = np.zeros((0, 0)), np.zeros(0), np.zeros((d, 0))
    for f in range(6):
        U, s, B, _, _ = fold(U, s, B, X[f * b:(f + 1) * b], r)
    F = X[24:28]
    C1, s1, B1, Ht = fold_from_coords(U * s, s, B, F, r)
    U2, s2, B2, H2, _ = fold(U, s, B, F, r)
    np.testing.assert_allclose(C1, U2 * s2, atol=1e-12)
    np.testing.assert_allclose(s1, s2, rtol=1e-13)
    # history rotation identity: old coordinates times H[:k] are the top rows of U+ Sigma+
    np.testing.assert_allclose((U * s) @ Ht, (U2 * s2)[: U.shape[0]], atol=1e-12)
    # new-row coordinates are F B+
    np.testing.assert_allclose(F @ B2, (U2 * s2)[U.shape[0]:], atol=1e-12)


# ---------------------------------------------------------------------------------------------
# schedule and storage closed forms
# ---------------------------------------------------------------------------------------------
def test_schedule_closed_forms():
    assert n_compressed(4096, 64, 256) == 3840               # Llama-3-8B layer workload
    assert n_compressed(65536, 512, 512) == 65024            # long-context prefill
    assert n_compressed(65536 + 2048, 512, 512) == 65024 + 2048
    assert n_compressed(1088, 32, 64) == 1024                # single-head workload
    for t in range(0, 2000, 7):
        n = n_compressed(t, 64, 256)
        e = t - n
        assert n % 64 == 0 and (e == t if t < 256 else 256 <= e <= 256 + 63)


def test_storage_formula_counts_stored_scalars():
    d = 16
    unit = OracleUnit(d, 4, 5, 7)
    unit.append(_stream(53, d, 29))
    stored = unit.coords().size + unit.B.size + unit.sigma.size + unit.exact.size
    assert unit.storage_scalars() == stored
    assert stored == unit.k * (unit.n + d + 1) + d * (53 - unit.n)


# ---------------------------------------------------------------------------------------------
# stale coordinates, closed form: with r >= d nothing is truncated, so after the second fold the
# basis spans all stacked rows and its first k1 columns are fixed by the sign convention
# ---------------------------------------------------------------------------------------------
def test_stale_rows_closed_form_two_folds():
    d, b = 16, 4
    X = _stream(d, d, 31, decay=0.5, noise=0.05)[:2 * b]
    F1, F2 = X[:b], X[b:]
    stale = OracleUnit(d, d, b, 0, rotate=False)
    stale.append(F1)
    B1 = stale.B.copy()
    k1 = B1.shape[1]
    # first fold: B1 spans the right singular vectors of F1 (library SVD), any signs
    V1 = np.linalg.svd(F1, full_matrices=False)[2][:k1].T
    np.testing.assert_allclose(np.abs(B1.T @ V1), np.eye(k1), atol=1e-10)
    # its stored coordinates are F1 B1 (no truncation: F1 = U1 Sigma1 B1^T)
    np.testing.assert_allclose(stale.coords(), F1 @ B1, atol=1e-12)
    stale.append(F2)
    assert stale.n == 2 * b and stale.k == 2 * b
    # second basis: right singular vectors of the stacked rows (library SVD), column c < k1
    # oriented along B1's column c (the sign convention)
    V2 = np.linalg.svd(X, full_matrices=False)[2][:2 * b].T
    for c in range(k1):
        if V2[:, c] @ B1[:, c] < 0:
            V2[:, c] = -V2[:, c]
    rec = stale.reconstruct()
    # old rows keep their first-fold coordinates, now read against the new basis' first k1
    # columns; new rows are coded in the new basis, which spans them, so they come back exactly
    np.testing.assert_allclose(rec[:b], (F1 @ B1) @ V2[:, :k1].T, atol=1e-10)
    np.testing.assert_allclose(rec[b:], F2, atol=1e-10)
    # and this differs from the synchronised history, which reproduces F1
    assert np.linalg.norm(rec[:b] - F1) > 1e-3 * np.linalg.norm(F1)


# ---------------------------------------------------------------------------------------------
# fixed basis ("Ablation Study"): the update runs until the rank budget is filled, then every
# block is stored as its projection onto the frozen basis
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("d,r,b,w", [(16, 4, 6, 3), (16, 6, 4, 5), (12, 5, 5, 0)])
def test_fixed_basis_projects_later_blocks(d, r, b, w):
    X = _stream(9 * b + w, d, 37 + r + b, decay=0.5, noise=0.05)
    unit = OracleUnit(d, r, b, w, fixed_basis=True)
    unit.append(X)
    n = unit.n
    f0 = -(-min(r, d) // b)                 # folds that fill the rank budget
    # the frozen basis is the rank-r truncated SVD basis of the first f0 blocks (no truncation
    # happens before the last of them, so the regular update is the SVD of their stacked rows)
    A = X[:f0 * b]
    Vt = np.linalg.svd(A, full_matrices=False)[2]
    kf = min(r, A.shape[0], d)
    P = Vt[:kf].T @ Vt[:kf]
    np.testing.assert_allclose(unit.B @ unit.B.T, P, atol=1e-10)
    rec = unit.reconstruct()
    u, s, v = svd_r(A, r)
    np.testing.assert_allclose(rec[:f0 * b], (u * s) @ v.T, atol=1e-10)
    np.testing.assert_allclose(rec[f0 * b:n], X[f0 * b:n] @ P, atol=1e-10)
    np.testing.assert_array_equal(rec[n:], X[n:])
    # the adapting cache does better on the same rows
    sync = OracleUnit(d, r, b, w)
    sync.append(X)
    assert np.linalg.norm(sync.reconstruct()[:n] - X[:n]) < np.linalg.norm(rec[:n] - X[:n])


# ---------------------------------------------------------------------------------------------
# bf16 coordinates: every fold is the update of the stored (rounded) state, rounded again
# ---------------------------------------------------------------------------------------------
def _bf16_grid_ok(x):
    """Every value has at most 8 significant bits (a bf16 number)."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    return bool(np.all(m * 256.0 == np.round(m * 256.0)))


def test_round_bf16_is_nearest_even_on_the_bf16_grid():
    from oracle import round_bf16
    # exact values stay, halfway cases go to the even neighbour, others to the nearest
    assert round_bf16(np.array([1.0, -2.5, 0.0]))[0] == 1.0
    one_ulp = 2.0 ** -7                       # bf16 spacing in [1, 2)
    half = 1.0 + one_ulp / 2                  # halfway between 1 and 1 + ulp: even is 1
    assert round_bf16(np.array([half]))[0] == 1.0
    assert round_bf16(np.array([1.0 + 1.5 * one_ulp]))[0] == 1.0 + 2 * one_ulp
    assert round_bf16(np.array([1.0 + 0.6 * one_ulp]))[0] == 1.0 + one_ulp
    x = np.random.default_rng(0).standard_normal(10000)
    y = round_bf16(x)
    assert _bf16_grid_ok(y)
    assert np.max(np.abs(y - x) / np.abs(x)) <= 2.0 ** -8 * (1 + 1e-6)


@pytest.mark.parametrize("d,r,b,w", [(16, 4, 3, 2), (16, 6, 8, 0), (32, 8, 16, 5)])
def test_bf16_coordinates_closed_form_per_fold(d, r, b, w):
    X = _stream(12 * b + w, d, 43 + d + r, decay=0.6, noise=0.02)
    unit = OracleUnit(d, r, b, w, coord_bf16=True)
    ref = OracleUnit(d, r, b, w)
    t = 0
    while unit.folds < 10:
        C0, s0, B0, n0 = unit.coords().copy(), unit.sigma.copy(), unit.B.copy(), unit.n
        step = (w + b) if unit.folds == 0 else b
        unit.append(X[t:t + step])
        ref.append(X[t:t + step])
        t += step
        F = X[n0:n0 + b]
        # library SVD of the history's rows Sigma B^T stacked on the block gives Sigma+ and B+
        M = np.vstack([s0[:, None] * B0.T, F]) if s0.size else F
        _, sv, Vt = np.linalg.svd(M, full_matrices=False)
        kp = unit.k
        V = Vt[:kp].T
        for c in range(kp):
            # columns c < k follow the sign convention; new directions have no fixed sign
            ref_col = B0[:, c] if c < s0.size else unit.B[:, c]
            if V[:, c] @ ref_col < 0:
                V[:, c] = -V[:, c]
        np.testing.assert_allclose(unit.sigma, sv[:kp], rtol=1e-10, atol=1e-12)
        gap = kp < sv.size and (sv[kp - 1] - sv[kp]) / sv[0] > 1e-3
        if gap:
            np.testing.assert_allclose(unit.B, V, atol=1e-8)
        C = unit.coords()
        assert _bf16_grid_ok(C)
        # stored coordinates: old rows moved by H[:k] = B^T B+, new rows F B+, then rounded
        if gap:
            expect = np.vstack([C0 @ (B0.T @ V), F @ V]) if n0 else F @ V
            from oracle import round_bf16
            diff = np.abs(C - round_bf16(expect))
            ulp = np.abs(round_bf16(expect)) * 2.0 ** -7 + 1e-30
            assert np.all(diff <= ulp)                       # at most one bf16 step apart
            assert np.mean(diff > 0) <= 1e-2                 # and equal almost everywhere
    # the rounded cache stays close to the unrounded one (rounding is 2^-8 relative per value)
    n = unit.n
    rel = np.linalg.norm(unit.reconstruct()[:n] - ref.reconstruct()[:n]) / np.linalg.norm(X[:n])
    assert rel <= 2e-2
    assert unit.storage_bytes(2) == 2 * unit.k * n + 4 * unit.k * (d + 1) + 2 * d * (t - n)
