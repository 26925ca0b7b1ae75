"""Brute-force pins of the oracle on an 8 x 4 stream (n=8, d=4, b=2, r=2), no GPU, no LAPACK.

An independent pure-Python path: a cyclic two-sided Jacobi eigendecomposition of the 4 x 4 Gram
matrix of the stacked rows (iS-KV summary, "Block-Incremental Decoding Updates": each fold is the
rank-r optimum of [history; block]), nested-loop attention sums, and a random search over
orthonormal 2-planes that must find none better than the oracle's fold.
"""
import math
import random

import numpy as np

from oracle import OracleUnit, attention, fold


def _gram(rows):
    d = len(rows[0])
    return [[sum(r[i] * r[j] for r in rows) for j in range(d)] for i in range(d)]


def _jacobi_eig(A, sweeps=60):
    """Cyclic two-sided Jacobi on a symmetric list-of-lists matrix; returns (eigvals, eigvecs)."""
    n = len(A)
    A = [row[:] for row in A]
    V = [[1.0 if i == j else 0.0 for j in range(n)] for i in range(n)]
    for _ in range(sweeps):
        off = sum(A[i][j] ** 2 for i in range(n) for j in range(n) if i != j)
        if off < 1e-30:
            break
        for p in range(n - 1):
            for q in range(p + 1, n):
                if abs(A[p][q]) < 1e-300:
                    continue
                tau = (A[q][q] - A[p][p]) / (2.0 * A[p][q])
                t = (1.0 if tau >= 0 else -1.0) / (abs(tau) + math.sqrt(1.0 + tau * tau))
                c = 1.0 / math.sqrt(1.0 + t * t)
                s = t * c
                for k in range(n):
                    akp, akq = A[k][p], A[k][q]
                    A[k][p], A[k][q] = c * akp - s * akq, s * akp + c * akq
                for k in range(n):
                    apk, aqk = A[p][k], A[q][k]
                    A[p][k], A[q][k] = c * apk - s * aqk, s * apk + c * aqk
                for k in range(n):
                    vkp, vkq = V[k][p], V[k][q]
                    V[k][p], V[k][q] = c * vkp - s * vkq, s * vkp + c * vkq
    lam = [A[i][i] for i in range(n)]
    order = sorted(range(n), key=lambda i: -lam[i])
    return [lam[i] for i in order], [[V[k][i] for i in order] for k in range(n)]


def _rows(seed):
    rnd = random.Random(seed)
    base = [[rnd.gauss(0, 1) for _ in range(4)] for _ in range(3)]
    X = []
    for _ in range(8):
        w = [rnd.gauss(0, 1) * s for s in (2.0, 1.0, 0.5)]
        X.append([sum(w[a] * base[a][j] for a in range(3)) + 0.05 * rnd.gauss(0, 1)
                  for j in range(4)])
    return X


def test_bruteforce_8x4_stream():
    X = _rows(1)
    d, b, r = 4, 2, 2
    U, s, B = np.zeros((0, 0)), np.zeros(0), np.zeros((d, 0))
    recon = []          # pure-Python reconstruction of the history so far
    for f in range(4):
        F = X[f * b:(f + 1) * b]
        M = recon + F
        last_M = M
        lam, vec = _jacobi_eig(_gram(M))
        U, s, B, _, _ = fold(U, s, B, np.array(F), r)
        sig_bf = [math.sqrt(max(l, 0.0)) for l in lam[:r]]
        np.testing.assert_allclose(s, sig_bf, rtol=1e-9)
        Pb = [[sum(vec[i][c] * vec[j][c] for c in range(r)) for j in range(d)] for i in range(d)]
        np.testing.assert_allclose(B @ B.T, np.array(Pb), atol=1e-9)
        # brute-force rank-r reconstruction: project every row onto the top-r eigenvectors
        recon = [[sum(row[a] * Pb[a][j] for a in range(d)) for j in range(d)] for row in M]
        np.testing.assert_allclose((U * s) @ B.T, np.array(recon), atol=1e-9)

    # random search over orthonormal 2-planes: none beats the oracle's last fold on its own M
    Mlast = np.array(last_M)
    best_oracle = np.linalg.norm(Mlast - Mlast @ B @ B.T) ** 2
    rng = np.random.default_rng(5)
    Q = np.linalg.qr(rng.standard_normal((100_000, d, r)))[0]
    proj = np.einsum("nd,kde,kfe->knf", Mlast, Q, Q)
    errs = ((Mlast[None] - proj) ** 2).sum(axis=(1, 2))
    assert errs.min() >= best_oracle * (1 - 1e-9)
    assert errs.min() <= best_oracle * 1.25         # the search does get close


def test_bruteforce_attention_nested_loops():
    X = _rows(2)
    unit_k = OracleUnit(4, 2, 2, 2)
    unit_v = OracleUnit(4, 2, 2, 2)
    unit_k.append(np.array(X))
    unit_v.append(np.array(X[::-1]))
    K, V = unit_k.reconstruct(), unit_v.reconstruct()
    rnd = random.Random(3)
    q = [rnd.gauss(0, 1) for _ in range(4)]
    logits = [sum(q[j] * K[i][j] for j in range(4)) / 2.0 for i in range(8)]
    m = max(logits)
    w = [math.exp(l - m) for l in logits]
    tot = sum(w)
    out = [sum(w[i] * V[i][j] for i in range(8)) / tot for j in range(4)]
    np.testing.assert_allclose(attention(np.array(q), K, V), out, rtol=1e-13)
