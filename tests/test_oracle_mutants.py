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


PINS = [_pin_stacked_svd, _pin_no_truncation, _pin_rope, _pin_attention, _pin_schedule]

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
