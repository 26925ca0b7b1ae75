"""Pins of the oracle's joint per-layer factorisation (all kv-heads of a (layer, sequence) in one
factorisation over rows of length n_kv d; iS-KV summary, "Reconstruction and Storage", per-layer
storage).

Each pin compares the joint unit with something fixed independently of the oracle's update: the
library SVD of the concatenated rows, exactness when the rank budget covers the data, and the
per-head mode it must reduce to with one kv-head.
"""
import numpy as np

import oracle.iskv_oracle as O


def _rows(rng, S, H, T, d, decay=0.5):
    return rng.standard_normal((S, H, T, d)) * np.arange(1, d + 1) ** -decay


def test_joint_with_one_kv_head_is_the_per_head_mode():
    rng = np.random.default_rng(1)
    d, r, b, w = 8, 3, 4, 3
    K, V = _rows(rng, 2, 1, 23, d), _rows(rng, 2, 1, 23, d)
    a = O.OracleCache(2, 1, 1, 2, d, r, r, b, w)
    j = O.OracleCache(2, 1, 1, 2, d, r, r, b, w, joint=True)
    a.append(0, K, V)
    j.append(0, K, V)
    for which in (0, 1):
        assert np.array_equal(a.reconstruct(0, which), j.reconstruct(0, which))
    q = rng.standard_normal((2, 2, d))
    assert np.array_equal(a.decode(0, q), j.decode(0, q))


def test_joint_singular_values_are_those_of_the_concatenated_history():
    # a rank budget above the data's rank: the incremental update is exact, so after every fold
    # Sigma holds the singular values of all folded rows side by side (library SVD)
    rng = np.random.default_rng(2)
    d, H, b, w = 5, 3, 4, 2
    q_rank = 6
    T = 22
    C = rng.standard_normal((T, q_rank))
    W = rng.standard_normal((q_rank, H * d))
    X = (C @ W).reshape(T, H, d).transpose(1, 0, 2)[None]        # [1][H][T][d], rank 6 jointly
    c = O.OracleCache(1, 1, H, H, d, 8, 8, b, w, joint=True)
    c.append(0, X, X)
    u = c.unit(0, 0, 0, 0)
    cat = np.concatenate([X[0, h, :u.n] for h in range(H)], axis=1)
    sv = np.linalg.svd(cat, compute_uv=False)
    assert np.allclose(np.sort(u.sigma)[::-1][:q_rank], sv[:q_rank], rtol=1e-10, atol=1e-10)
    assert np.all(np.abs(u.sigma[q_rank:]) < 1e-9)
    # and every kv-head's rows come back exactly, although no single head's rank fits the budget
    for h in range(H):
        K, _ = c.keys_values(0, 0, h)
        assert np.allclose(K, X[0, h], atol=1e-9)


def test_joint_truncation_is_shared_by_the_heads():
    # first fold with a rank budget below the block's rank: the compressed rows are the rank-r
    # truncation of the concatenated block (library SVD), not per-head truncations
    rng = np.random.default_rng(3)
    d, H, r, b, w = 6, 4, 5, 10, 3
    K = _rows(rng, 1, H, b + w, d)
    c = O.OracleCache(1, 1, H, H, d, r, r, b, w, joint=True)
    c.append(0, K, K)
    cat = np.concatenate([K[0, h, :b] for h in range(H)], axis=1)
    u, sv, vt = np.linalg.svd(cat, full_matrices=False)
    trunc = (u[:, :r] * sv[:r]) @ vt[:r]
    rec = c.reconstruct(0, 1)
    for h in range(H):
        assert np.allclose(rec[0, h, :b], trunc[:, h * d:(h + 1) * d], atol=1e-10)
        assert np.array_equal(rec[0, h, b:], K[0, h, b:])
        # a per-head truncation of the same rank differs
        uh, sh, vh = np.linalg.svd(K[0, h, :b], full_matrices=False)
        assert not np.allclose(rec[0, h, :b], (uh[:, :r] * sh[:r]) @ vh[:r], atol=1e-6)


def test_joint_storage_counts_one_factorisation_per_layer():
    # "Reconstruction and Storage": k (n + d + 1) factor scalars per path, d = n_kv head_dim
    rng = np.random.default_rng(4)
    d, H, r, b, w = 4, 2, 3, 4, 2
    K = _rows(rng, 1, H, 14, d)
    c = O.OracleCache(1, 1, H, H, d, r, r, b, w, joint=True)
    c.append(0, K, K)
    u = c.unit(0, 0, 1, 0)
    assert u is c.unit(0, 0, 0, 0)
    assert u.n == 12 and u.k == 3
    assert u.storage_scalars() == 3 * (12 + H * d + 1) + H * d * 2
