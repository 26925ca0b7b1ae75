"""Pins of the oracle's prefill with protection (iS-KV summary, "Prefill Compression", steps 1-3,
and the position map of "Reconstruction and Storage"): the chunk scores against a pure-Python
evaluation, planted outliers, the value neighbourhood against brute force, the initial
factorisation against the library SVD of the remaining rows, folds after the prefill, and decode
attention over the mixed exact / compressed positions assembled by hand."""
import math

import numpy as np
import pytest

from oracle import (OracleCache, OracleUnit, attention, chunk_scores, fold, protected_positions,
                    rope, svd_r, value_protected)


def _keys(T, d, seed):
    rng = np.random.default_rng(seed)
    G = np.linalg.qr(rng.standard_normal((T, d)))[0] * math.sqrt(T)
    return (G * np.arange(1, d + 1) ** -0.7) @ np.linalg.qr(rng.standard_normal((d, d)))[0].T


def test_chunk_scores_match_pure_python():
    K = _keys(37, 6, 1)
    chunk = 8
    got = chunk_scores(K, chunk)
    exp = []
    for c0 in range(0, 37, chunk):
        rows = [list(map(float, K[i])) for i in range(c0, min(37, c0 + chunk))]
        mean = [math.fsum(r[j] for r in rows) / len(rows) for j in range(6)]
        nm = math.sqrt(math.fsum(x * x for x in mean))
        cs = []
        for r in rows:
            nr = math.sqrt(math.fsum(x * x for x in r))
            cs.append(math.fsum(a * b for a, b in zip(r, mean)) / (nr * nm))
        exp.append(min(cs))
    np.testing.assert_allclose(got, exp, rtol=1e-12)
    assert got.size == 5                              # the last chunk holds 5 rows


def test_planted_outlier_chunks_are_protected():
    d, chunk = 8, 4
    rng = np.random.default_rng(2)
    base = rng.standard_normal(d)
    K = np.tile(base, (40, 1)) + 1e-3 * rng.standard_normal((40, d))
    K[13] = -base                                     # chunk 3 holds one reversed key
    K[29] = rng.standard_normal(d) * 3                # chunk 7 one unrelated key
    P = protected_positions(K, np.arange(40), chunk, 2, 0, None)
    assert P.tolist() == list(range(12, 16)) + list(range(28, 32))
    # the reversed key scores below the unrelated one: with m = 1 only chunk 3 is protected
    assert protected_positions(K, np.arange(40), chunk, 1, 0, None).tolist() == list(range(12, 16))
    # a suffix adds the last positions; m = 0 protects the suffix alone
    assert protected_positions(K, np.arange(40), chunk, 0, 3, None).tolist() == [37, 38, 39]
    # identical keys: every chunk scores exactly 1
    assert np.all(chunk_scores(np.tile(base, (16, 1)), 4) == pytest.approx(1.0, abs=1e-15))


def test_protection_uses_rotated_keys():
    """Keys that are equal before RoPE are not aligned after it: scores use the rotated keys."""
    d = 8
    base = np.random.default_rng(3).standard_normal(d)
    K = np.tile(base, (32, 1))
    assert chunk_scores(K, 8).min() == pytest.approx(1.0)
    Kr = rope(K, np.arange(32), 10.0)
    P = protected_positions(K, np.arange(32), 8, 1, 0, 10.0)
    c = int(np.argmin(chunk_scores(Kr, 8)))
    assert P.tolist() == list(range(8 * c, 8 * c + 8))


@pytest.mark.parametrize("rho", [0, 1, 3])
def test_value_neighbourhood_brute_force(rho):
    PK = np.array([0, 5, 6, 17, 29])
    got = value_protected(PK, rho, 0, 30).tolist()
    exp = [i for i in range(30) if any(abs(i - p) <= rho for p in PK)]
    assert got == exp


def test_prefill_factorises_the_remaining_rows_and_keeps_protected_rows_exact():
    d, r, b, w = 12, 4, 5, 6
    X = _keys(60, d, 4)
    prot = [3, 4, 20, 21, 22, 50, 57]                 # 57 lies in the window: ignored
    unit = OracleUnit(d, r, b, w)
    unit.prefill(X, prot)
    comp = [i for i in range(54) if i not in prot]
    U, s, B = svd_r(X[comp], r)
    rec = unit.reconstruct()
    np.testing.assert_allclose(rec[comp], (U * s) @ B.T, atol=1e-12)
    np.testing.assert_array_equal(rec[[3, 4, 20, 21, 22, 50]], X[[3, 4, 20, 21, 22, 50]])
    np.testing.assert_array_equal(rec[54:], X[54:])
    assert unit.n == len(comp) and unit.t == 60
    assert unit.storage_scalars() == unit.k * (unit.n + d + 1) + d * (6 + 6)
    # no protection: the prefill is the truncated SVD of every row outside the window
    plain = OracleUnit(d, r, b, w)
    plain.prefill(X, [])
    U, s, B = svd_r(X[:54], r)
    np.testing.assert_allclose(plain.reconstruct()[:54], (U * s) @ B.T, atol=1e-12)


def test_folds_after_the_prefill_take_the_oldest_window_rows():
    d, r, b, w = 10, 3, 4, 5
    X = _keys(40, d, 5)
    unit = OracleUnit(d, r, b, w)
    unit.prefill(X[:23], [2, 7, 8])
    comp = [i for i in range(18) if i not in (2, 7, 8)]
    U, s, B = svd_r(X[comp], r)
    unit.append(X[23:28])                             # window 5 + 5 rows: one fold of 18 .. 21
    U, s, B, _, _ = fold(U, s, B, X[18:22], r)
    rec = unit.reconstruct()
    np.testing.assert_allclose(rec[comp + [18, 19, 20, 21]], (U * s) @ B.T, atol=1e-10)
    np.testing.assert_array_equal(rec[[2, 7, 8]], X[[2, 7, 8]])
    np.testing.assert_array_equal(rec[22:28], X[22:28])
    assert unit.comp_pos.tolist() == comp + [18, 19, 20, 21]


def test_decode_over_a_prefilled_cache_uses_exact_rows_at_protected_positions():
    d, G, T0 = 8, 2, 48
    rng = np.random.default_rng(6)
    # keys along the slowest RoPE pair (channels 3 and 7: 0.03 rad per position at theta 100),
    # so chunks stay coherent after rotation; one key reversed
    K = np.zeros((1, 1, T0, d))
    K[0, 0, :, 3], K[0, 0, :, 7] = 1.0, 0.5
    K += 1e-3 * rng.standard_normal(K.shape)
    V = rng.standard_normal((1, 1, T0, d))
    K[0, 0, 17] *= -4.0                               # an outlier key
    cache = OracleCache(1, 1, 1, G, d, 3, 3, 4, 6, rope=True, rope_theta=100.0)
    cache.prefill(0, K, V, chunk=8, m=1, suffix=2, rho=1)
    ku, vu = cache.unit(0, 0, 0, 0), cache.unit(0, 0, 0, 1)
    assert 17 in ku.prot_pos.tolist() and {16, 17, 18} <= set(vu.prot_pos.tolist())
    assert ku.prot_pos.tolist()[-2:] == [40, 41]      # the suffix before the window
    q = rng.standard_normal((1, G, d))
    out = cache.decode(0, q)
    # by hand: rows by position, exact where protected or in the window, RoPE at the position
    Kh, Vh = ku.reconstruct(), vu.reconstruct()
    for i in range(T0):
        if i in ku.prot_pos or i >= T0 - 6:
            assert np.array_equal(Kh[i], K[0, 0, i])
        if i in vu.prot_pos or i >= T0 - 6:
            assert np.array_equal(Vh[i], V[0, 0, i])
    Kr = rope(Kh, np.arange(T0), 100.0)
    for g in range(G):
        np.testing.assert_allclose(out[0, g], attention(q[0, g], Kr, Vh), rtol=1e-12)
