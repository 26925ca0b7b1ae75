"""Pins of the oracle's decode attention and rotary embedding (no GPU).

Decode attention is plain softmax attention over the reconstructed cache (iS-KV summary,
"Reconstruction and Storage"); keys are compressed before RoPE and rotated at attention time.
"""
import cmath
import math

import numpy as np

from oracle import OracleCache, attention, rope


def test_rope_matches_complex_rotation():
    # independent formulation: channel pair (j, j + d/2) as the complex number x_j + i x_{j+d/2},
    # multiplied by exp(i pos theta^(-2j/d))
    rng = np.random.default_rng(0)
    d, theta = 16, 1e4
    X = rng.standard_normal((5, d))
    pos = np.array([0, 1, 7, 1000, 65535])
    Y = rope(X, pos, theta)
    for a in range(5):
        for j in range(d // 2):
            z = complex(X[a, j], X[a, j + d // 2]) * cmath.exp(
                1j * pos[a] * theta ** (-2.0 * j / d))
            assert abs(Y[a, j] - z.real) < 1e-9 and abs(Y[a, j + d // 2] - z.imag) < 1e-9


def test_rope_identity_norm_and_relative_position():
    rng = np.random.default_rng(1)
    d, theta = 128, 5e5
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    np.testing.assert_array_equal(rope(q[None], np.array([0]), theta)[0], q)
    for m in (3, 4095, 67583):
        np.testing.assert_allclose(np.linalg.norm(rope(q[None], np.array([m]), theta)),
                                   np.linalg.norm(q), rtol=1e-13)
    # <R(q, m), R(k, n)> depends on m - n only
    ref = rope(q[None], np.array([10]), theta)[0] @ rope(k[None], np.array([3]), theta)[0]
    for c in (0, 100, 50000):
        v = rope(q[None], np.array([c + 7]), theta)[0] @ rope(k[None], np.array([c]), theta)[0]
        assert abs(v - ref) < 1e-9


def test_attention_closed_forms():
    rng = np.random.default_rng(2)
    V = rng.standard_normal((9, 6))
    q = rng.standard_normal(6)
    # identical keys -> uniform weights -> mean of the values
    K = np.tile(rng.standard_normal(6), (9, 1))
    np.testing.assert_allclose(attention(q, K, V), V.mean(axis=0), rtol=1e-13)
    # one key aligned with q by a huge margin -> its value
    K = rng.standard_normal((9, 6)) * 1e-3
    K[4] = q * 1e3
    np.testing.assert_allclose(attention(q, K, V), V[4], rtol=1e-12)
    # two keys only: logistic weight of the logit difference
    K2 = rng.standard_normal((2, 6))
    w1 = 1.0 / (1.0 + math.exp((K2[1] - K2[0]) @ q / math.sqrt(6)))
    np.testing.assert_allclose(attention(q, K2, V[:2]), w1 * V[0] + (1 - w1) * V[1], rtol=1e-12)


def test_cache_gqa_map_and_window_only_decode():
    # before any fold the cache is exact: decode is attention over the raw rows, and q-head g
    # reads kv-head g // (n_q / n_kv)
    rng = np.random.default_rng(3)
    d = 8
    cache = OracleCache(1, 1, 2, 4, d, 2, 3, 4, 16, rope=True, rope_theta=100.0)
    K = rng.standard_normal((1, 2, 10, d))
    V = rng.standard_normal((1, 2, 10, d))
    cache.append(0, K, V)
    assert cache.unit(0, 0, 0, 0).n == 0
    q = rng.standard_normal((1, 4, d))
    out = cache.decode(0, q)
    for g in range(4):
        h = g // 2
        Kr = rope(K[0, h], np.arange(10), 100.0)
        np.testing.assert_allclose(out[0, g], attention(q[0, g], Kr, V[0, h]), rtol=1e-13)
    rec = cache.reconstruct(0, 1)
    np.testing.assert_array_equal(rec[0], V[0])


def test_decode_over_compressed_history_is_attention_over_reconstruction():
    rng = np.random.default_rng(4)
    d = 16
    cache = OracleCache(2, 1, 1, 2, d, 3, 5, 4, 6, rope=True, rope_theta=50.0)
    K = rng.standard_normal((2, 1, 30, d))
    V = rng.standard_normal((2, 1, 30, d))
    cache.append(0, K, V)
    assert cache.unit(0, 1, 0, 0).n == 24
    q = rng.standard_normal((2, 2, d))
    out = cache.decode(0, q)
    for s in range(2):
        Kt = cache.reconstruct(0, 0, apply_rope=True)[s, 0]
        Vt = cache.reconstruct(0, 1)[s, 0]
        for g in range(2):
            np.testing.assert_allclose(out[s, g], attention(q[s, g], Kt, Vt), rtol=1e-12)
