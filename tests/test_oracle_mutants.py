"""Planted mistakes: each mutant of the oracle (a dropped term, a wrong sign, a wrong scale, an
off-by-one) must fail at least one of the pins, and the unmodified oracle must pass all of them.

The mistakes are planted in a private copy of the oracle's source on the CPU; the real module is
untouched.
"""
import cmath
import math
import pathlib
import types

import numpy as np
import pytest

import oracle.iskv_oracle as O

SRC = pathlib.Path(O.__file__).read_text()


def _load(src):
    mod = types.ModuleType("oracle_mutant")
    exec(compile(src, "oracle_mutant", "exec"), mod.__dict__)
    return mod


def _stream(T, d, seed):
    rng = np.random.default_rng(seed)
    G = np.linalg.qr(rng.standard_normal((T, d)))[0] * np.sqrt(T)
    H = np.linalg.qr(rng.standard_normal((d, d)))[0]
    return (G * np.arange(1, d + 1) ** -0.7) @ H.T + 1e-3 * rng.standard_normal((T, d))


def _pin_stacked_svd(m):
    d, r, b = 12, 4, 5
    X = _stream(40, d, 3)
    U, s, B = np.zeros((0, 0)), np.zeros(0), np.zeros((d, 0))
    for f in range(8):
        F = X[f * b:(f + 1) * b]
        A = (U * s) @ B.T if U.shape[0] else np.zeros((0, d))
        M = np.vstack([A, F])
        U, s, B, _, _ = m.fold(U, s, B, F, r)
        u, sv, vt = np.linalg.svd(M, full_matrices=False)
        ref = (u[:, :r] * sv[:r]) @ vt[:r]
        if s.size != min(r, M.shape[0], d) or not np.allclose((U * s) @ B.T, ref, atol=1e-8):
            return False
    return True


def _pin_no_truncation(m):
    d = 8
    X = _stream(37, d, 5)
    unit = m.OracleUnit(d, d, 3, 4)
    for i in range(0, 37, 3):
        unit.append(X[i:i + 3])
        if not np.all(np.isfinite(unit.sigma)) or unit.sigma.sum() > 1e6:
            return False        # diverging mutant: stop before LAPACK sees inf/nan
    return unit.n == 3 * ((37 - 4) // 3) and np.allclose(unit.reconstruct(), X, atol=1e-10)


def _pin_rope(m):
    x = np.array([[0.3, -1.2, 2.0, 0.7]])
    y = m.rope(x, np.array([5]), 100.0)[0]
    for j in range(2):
        z = complex(x[0, j], x[0, j + 2]) * cmath.exp(1j * 5 * 100.0 ** (-j / 2))
        if abs(y[j] - z.real) > 1e-12 or abs(y[j + 2] - z.imag) > 1e-12:
            return False
    return True


def _pin_attention(m):
    rng = np.random.default_rng(1)
    q, K, V = rng.standard_normal(6), rng.standard_normal((2, 6)), rng.standard_normal((2, 3))
    w1 = 1.0 / (1.0 + math.exp((K[1] - K[0]) @ q / math.sqrt(6)))
    return np.allclose(m.attention(q, K, V), w1 * V[0] + (1 - w1) * V[1], rtol=1e-12)


def _pin_schedule(m):
    return (m.n_compressed(4096, 64, 256) == 3840 and m.n_compressed(255, 64, 256) == 0
            and m.n_compressed(320, 64, 256) == 64 and m.n_compressed(319, 64, 256) == 0)


def _pin_stale_two_folds(m):
    """Stale coordinates after two untruncated folds: old rows keep their first-fold coordinates
    against the new basis' first columns, new rows come back exactly (library SVDs)."""
    d, b = 16, 4
    X = _stream(d, d, 31)[:2 * b]
    unit = m.OracleUnit(d, d, b, 0, rotate=False)
    unit.append(X[:b])
    B1 = unit.B.copy()
    k1 = B1.shape[1]
    unit.append(X[b:])
    V2 = np.linalg.svd(X, full_matrices=False)[2][:2 * b].T
    for c in range(k1):
        if V2[:, c] @ B1[:, c] < 0:
            V2[:, c] = -V2[:, c]
    rec = unit.reconstruct()
    return (np.allclose(rec[:b], (X[:b] @ B1) @ V2[:, :k1].T, atol=1e-10)
            and np.allclose(rec[b:], X[b:], atol=1e-10))


def _pin_fixed_basis(m):
    """Fixed basis: after the folds that fill the rank budget, blocks are projected onto the
    rank-r right singular subspace of the rows folded so far (library SVD)."""
    d, r, b = 16, 6, 4
    X = _stream(40, d, 41)
    unit = m.OracleUnit(d, r, b, 0, fixed_basis=True)
    unit.append(X)
    Vt = np.linalg.svd(X[:8], full_matrices=False)[2][:r]
    P = Vt.T @ Vt
    return unit.n == 40 and np.allclose(unit.reconstruct()[8:], X[8:] @ P, atol=1e-10)


def _pin_bf16_coordinates(m):
    """bf16 coordinates: stored values lie on the bf16 grid and each fold's coordinates are the
    rounded [C H[:k]; F B+] of the stored state (library SVD of [Sigma B^T; F])."""
    d, r, b = 16, 5, 6
    X = _stream(60, d, 47)
    unit = m.OracleUnit(d, r, b, 0, coord_bf16=True)
    unit.append(X[:b])
    for f in range(1, 6):
        C0, s0, B0 = unit.coords().copy(), unit.sigma.copy(), unit.B.copy()
        F = X[f * b:(f + 1) * b]
        unit.append(F)
        _, sv, Vt = np.linalg.svd(np.vstack([s0[:, None] * B0.T, F]), full_matrices=False)
        V = Vt[:unit.k].T
        for c in range(unit.k):
            if V[:, c] @ (B0[:, c] if c < s0.size else unit.B[:, c]) < 0:
                V[:, c] = -V[:, c]
        C = unit.coords()
        mant = np.frexp(C)[0] * 256.0
        if not np.all(mant == np.round(mant)):
            return False
        expect = np.vstack([C0 @ (B0.T @ V), F @ V])
        # nearest rounding to 8 significant bits moves a value by at most half a step
        if np.any(np.abs(C - expect) > 2.0 ** -8 * np.abs(expect) * (1 + 1e-4)
                  + 1e-9 * np.abs(expect).max()):
            return False
    return True


def _pin_prefill(m):
    """Prefill protection: a planted reversed key protects its chunk; the value neighbourhood
    is the brute-force dilation; the initial factorisation is the library SVD of the rows left."""
    d, chunk = 8, 4
    rng = np.random.default_rng(2)
    base = rng.standard_normal(d)
    K = np.tile(base, (40, 1)) + 1e-3 * rng.standard_normal((40, d))
    K[13] = -base
    if m.protected_positions(K, np.arange(40), chunk, 1, 0, None).tolist() != [12, 13, 14, 15]:
        return False
    PK = np.array([0, 5, 17])
    if m.value_protected(PK, 2, 0, 30).tolist() != [i for i in range(30)
                                                     if any(abs(i - p) <= 2 for p in PK)]:
        return False
    X = _stream(40, d, 9)
    unit = m.OracleUnit(d, 3, 4, 5)
    unit.prefill(X, [1, 2, 9])
    comp = [i for i in range(35) if i not in (1, 2, 9)]
    u, sv, vt = np.linalg.svd(X[comp], full_matrices=False)
    rec = unit.reconstruct()
    return (np.allclose(rec[comp], (u[:, :3] * sv[:3]) @ vt[:3], atol=1e-10)
            and np.array_equal(rec[[1, 2, 9]], X[[1, 2, 9]]))


def _pin_joint(m):
    """Joint per-layer factorisation: after the first fold the layer's compressed rows are the
    rank-r truncation (library SVD) of the kv-heads' rows side by side, and kv-head h reads its
    own d columns of it, for keys and values alike."""
    d, H, r, b, w = 6, 3, 3, 6, 2
    rng = np.random.default_rng(12)
    K = rng.standard_normal((1, H, b + w, d)) * np.arange(1, d + 1) ** -0.5
    V = rng.standard_normal((1, H, b + w, d))
    c = m.OracleCache(1, 1, H, H, d, r, r, b, w, joint=True)
    c.append(0, K, V)
    for which, X in ((0, K), (1, V)):
        cat = np.concatenate([X[0, h, :b] for h in range(H)], axis=1)
        u, sv, vt = np.linalg.svd(cat, full_matrices=False)
        trunc = (u[:, :r] * sv[:r]) @ vt[:r]
        for h in range(H):
            got = c.keys_values(0, 0, h)[which]
            if not (np.allclose(got[:b], trunc[:, h * d:(h + 1) * d], atol=1e-10)
                    and np.array_equal(got[b:], X[0, h, b:])):
                return False
    return True


PINS = [_pin_stacked_svd, _pin_no_truncation, _pin_rope, _pin_attention, _pin_schedule,
        _pin_stale_two_folds, _pin_fixed_basis, _pin_bf16_coordinates, _pin_prefill, _pin_joint]

MUTANTS = {
    "new-row identity block negated": ("Ublk[n:, k:] = np.eye(b)", "Ublk[n:, k:] = -np.eye(b)"),
    "coupling term F B dropped": ("Z[k:, :k] = F @ B", "Z[k:, :k] = 0.0 * (F @ B)"),
    "Sigma squared in the core": ("Z[:k, :k] = np.diag(sigma)", "Z[:k, :k] = np.diag(sigma ** 2)"),
    "history block of U dropped": ("Ublk[:n, :k] = U", "Ublk[:n, :k] = 0.0 * U"),
    "residual basis ignored": ("B_new = np.hstack([B, P]) @ H",
                               "B_new = np.hstack([B, 0.0 * P]) @ H"),
    "one rank too few": ("kp = min(r, k + p)", "kp = max(1, min(r, k + p) - 1)"),
    "RoPE sign": ("x2 * c + x1 * s", "x2 * c - x1 * s"),
    "RoPE frequency exponent": ("theta ** (-2.0 * np.arange(h, dtype=np.float64) / d)",
                                "theta ** (-1.0 * np.arange(h, dtype=np.float64) / d)"),
    "softmax scale 1/d": ("/ math.sqrt(q.size)", "/ q.size"),
    "fold one row early": ("max(0, t - window)", "max(0, t - window + 1)"),
    "stale: new rows coded in the old basis": (
        "self.C_stale = np.vstack([C, F @ B_new])",
        "self.C_stale = np.vstack([C, np.hstack([F @ self.B, "
        "np.zeros((F.shape[0], kp - k_old))])])"),
    "stale: old coordinates in the wrong columns": (
        "C[:, :m] = self.C_stale[:, :m]\n            self.C_stale = np.vstack([C, F @ B_new])",
        "C[:, kp - m:] = self.C_stale[:, :m]\n            self.C_stale = np.vstack([C, F @ B_new])"),
    "fixed basis: one adapting fold too few": ("self.adapt_folds = -(-min(rank, d) // block)",
                                               "self.adapt_folds = min(rank, d) // block"),
    "fixed basis: frozen one fold late": ("self.folds >= self.adapt_folds",
                                          "self.folds > self.adapt_folds"),
    "bf16: rotated coordinates left unrounded": ("                self.C_stale = rnd(C_new)",
                                                 "                self.C_stale = C_new"),
    "prefill: chunk score takes the largest cosine": ("        out.append(cos.min())",
                                                       "        out.append(cos.max())"),
    "prefill: value neighbourhood one short": ("range(max(lo, p - rho), min(hi, p + rho + 1))",
                                               "range(max(lo, p - rho), min(hi, p + rho))"),
    "prefill: protected rows factorised too": (
        "comp = np.asarray(sorted(set(range(end)) - set(prot.tolist())), dtype=np.int64)",
        "comp = np.asarray(sorted(set(range(end))), dtype=np.int64)"),
    "bf16: rounding to 7 significant bits": ("u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16\n    return (u.astype(np.uint32) << 16)",
                                             "u = (u + 0xFFFF + ((u >> 17) & 1)) >> 17\n    return (u.astype(np.uint32) << 17)"),
    "joint: kv-heads concatenated in reverse order": (
        "np.concatenate(list(K[s]), axis=1)", "np.concatenate(list(K[s])[::-1], axis=1)"),
    "joint: head slice one head late": (
        "return X[:, head * self.d:(head + 1) * self.d]",
        "return X[:, ((head + 1) % self.n_kv) * self.d:((head + 1) % self.n_kv + 1) * self.d]"),
}


def test_unmodified_oracle_passes_every_pin():
    m = _load(SRC)
    assert all(pin(m) for pin in PINS)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    old, new = MUTANTS[name]
    assert SRC.count(old) == 1, name
    m = _load(SRC.replace(old, new))
    caught = []
    for pin in PINS:
        try:
            ok = pin(m)
        except Exception:       # a crash is a failed pin too
            ok = False
        if not ok:
            caught.append(pin.__name__)
            break
    assert caught, f"mutant '{name}' passed every pin"
