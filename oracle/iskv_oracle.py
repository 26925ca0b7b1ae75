"""Float64 CPU oracle of the iS-KV hot path: block-incremental truncated SVD of a growing row set
plus decode attention over the reconstructed cache.

TEST INFRASTRUCTURE ONLY. The product package never imports, links or runs anything here; only
``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` do. It shares no
code with the CUDA path: the two meet only in the seeded inputs of ``iskv_synth``.

Source: "iS-KV: Online Low-Rank KV Cache Compression via Block-Incremental SVD" (summary page).

* section "Theoretical Foundation": the rank-budgeted objective and the truncated SVD ``SVD_r``,
  which keeps ``k = min(r, n, d)`` singular triplets with orthonormal ``U``, ``B``;
* section "Architecture Overview": per K/V path an exact window of the most recent tokens plus a
  low-rank history;
* section "Block-Incremental Decoding Updates": steps 1-3 (residual ``E = F - (F B) B^T``, residual
  basis ``P`` via QR and SVD, augmented core ``Z = [[Sigma, 0], [F B, F P]]``, core SVD
  ``(G, Sigma+, H) = SVD_r(Z)``, ``U+ = diag(U, I_b) G``, ``B+ = [B P] H``);
* section "Reconstruction and Storage": compressed rows are ``(U Sigma B^T)[j]``, the others the
  exact rows; persistent storage ``k (n + d + 1)`` factor scalars per path plus ``d e`` exact
  scalars.

Readings taken where the page is silent (each also stated at its definition):

* fold trigger: rows are appended one at a time; whenever the exact window holds ``window +
  block`` rows, its oldest ``block`` rows are folded, so ``n_c(t) = block * floor(max(0, t -
  window) / block)`` and decode at ``t`` tokens sees positions ``0 .. t-1``;
* the residual is projected twice (classical Gram-Schmidt, twice);
* ``P`` spans the numerical row space of ``E`` (singular values above ``1e-12 max(1, ||F||_2)``),
  re-orthogonalised against ``B``; ``p`` is that numerical rank;
* the retained rank after a fold is ``min(r, k + p)``; zero singular values are kept;
* RoPE pairs channel ``j`` with ``j + d/2`` at angle ``pos * theta^(-2j/d)``; keys are stored
  before RoPE and rotated at attention time, queries arrive rotated; scale ``1/sqrt(d)``; q-head
  ``g`` reads kv-head ``g // (n_q / n_kv)``;
* singular vectors are sign-ambiguous; each fold orients new basis vector ``c`` along old basis
  vector ``c`` (``H[c, c] >= 0`` for ``c < k``). Reconstructions and attention do not depend on
  it; the stale-coordinate variant does;
* the "stale coordinates" variant (``rotate=False``) updates ``Sigma`` and ``B`` exactly as above
  but keeps the old rows' coordinates ``U Sigma`` unrotated (zero-padded or truncated to the new
  rank) and reconstructs them against the new basis; new rows get ``F B+``;
* bf16 coordinates (``coord_bf16=True``; "Reconstruction and Storage" leaves the bytes per factor
  scalar beta_f open and the "Conclusion" names quantisation as the next step): the stored
  coordinates ``C = U Sigma`` (the ``k n`` scalars that grow with the history) are rounded to
  bf16 (nearest even, through float32, as a kernel rounding its fp32 results) after every fold,
  and the next fold starts from the rounded values; ``B`` and ``Sigma`` stay unrounded, because
  the update's core assumes an orthonormal ``B``;
* prefill with protection (section "Prefill Compression", steps 1-3): over the prefill rows that
  the window does not hold, keys are cut into chunks of ``chunk`` consecutive positions; chunk
  ``c`` scores ``min_{i in c} cos(k_i^rot, mean_c k^rot)`` (keys rotated at their positions; a
  zero vector's cosine counts as 1); the ``m`` lowest-scoring chunks (ties by chunk index) plus
  the ``suffix`` positions just before the window (the local suffix of the rows that would be
  compressed) are the protected key positions ``P_K``; ``P_V`` is every
  position within ``rho`` of ``P_K``. Protected rows stay exact for good; the remaining rows of the
  prefill (outside the window) get one truncated SVD; later blocks fold from the window as usual.
  Compressed rows keep their positions (the index map ``C_X`` of "Reconstruction and Storage");
* the "fixed basis" variant (``fixed_basis=True``, section "Ablation Study": bases kept fixed)
  runs the regular update for the first ``ceil(min(r, d) / block)`` blocks, which fill the rank
  budget, and then freezes ``B`` and ``Sigma``: every later block is stored as its coordinates
  ``F B`` in the frozen basis (its orthogonal projection onto ``span B``) and old coordinates stay
  as they are (the basis does not move, so nothing drifts).

* joint per-layer factorisation (``joint=True``; "Reconstruction and Storage" counts persistent
  storage per layer, and the ranks the page reports only compress when all kv-heads of a layer
  share one factorisation): the rows of all ``n_kv`` kv-heads of one (layer, sequence) at one
  position are concatenated, head by head, into one row of length ``n_kv d``; one unit per path
  factorises those rows exactly as above, and kv-head ``h`` reads columns ``h d .. h d + d - 1`` of
  its reconstruction (RoPE then per head, as in the per-head mode). Its exact window is the same
  rows, so it is the concatenation of the per-head windows.

Parity: every function here is pinned by ``tests/test_oracle_*.py`` (closed forms, library special
cases, invariants and brute force); none is "parity unpinned".
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "svd_r",
    "n_compressed",
    "residual_basis",
    "fold",
    "fold_from_coords",
    "OracleUnit",
    "OracleCache",
    "rope",
    "attention",
    "round_bf16",
    "chunk_scores",
    "protected_positions",
    "value_protected",
]


# ----------------------------------------------------------------------------------------------
# Theoretical Foundation
# ----------------------------------------------------------------------------------------------
def svd_r(X: np.ndarray, r: int):
    """Truncated SVD ``SVD_r(X) = (U, sigma, B)`` keeping ``k = min(r, n, d)`` components.

    iS-KV summary, section "Theoretical Foundation": the optimum of the rank-``r`` objective.
    """
    U, s, Vt = np.linalg.svd(np.asarray(X, dtype=np.float64), full_matrices=False)
    k = min(r, X.shape[0], X.shape[1])
    return U[:, :k], s[:k], Vt[:k].T


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Values rounded to bfloat16 (8-bit significand, round to nearest even) through float32, as
    a kernel that computes in fp32 and stores bf16 rounds them; returned as float64."""
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float64).astype(np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return (u.astype(np.uint32) << 16).view(np.float32).astype(np.float64).reshape(f.shape)


def n_compressed(t: int, block: int, window: int) -> int:
    """Rows in the low-rank history after ``t`` tokens (fold when window + block rows are exact).

    iS-KV summary, section "Architecture Overview" (exact window of the most recent ``w`` tokens)
    with the reading that a fold consumes the oldest ``block`` rows as soon as ``window + block``
    rows are exact.
    """
    return block * (max(0, t - window) // block)


# ----------------------------------------------------------------------------------------------
# Block-Incremental Decoding Updates
# ----------------------------------------------------------------------------------------------
def residual_basis(F: np.ndarray, B: np.ndarray):
    """Step 1: residual ``E = F - (F B) B^T`` and an orthonormal residual basis ``P``.

    The projection is applied twice (the page gives it once; twice keeps ``E`` orthogonal to ``B``
    to rounding). ``P`` is found "via QR and SVD": QR of ``E^T``, then the SVD of the R factor
    keeps the directions with singular value above ``1e-12 max(1, ||F||_2)``; ``P`` is finally
    re-orthogonalised against ``B``. Returns ``(E, P)`` with ``P`` of shape ``d x p``.
    """
    F = np.asarray(F, dtype=np.float64)
    d = F.shape[1]
    k = B.shape[1]
    if k:
        E = F - (F @ B) @ B.T
        E = E - (E @ B) @ B.T
    else:
        E = F.copy()
    Q, R = np.linalg.qr(E.T)                 # d x m, m x b   (m = min(d, b))
    Ur, sr, _ = np.linalg.svd(R)
    tol = 1e-12 * max(1.0, float(np.linalg.norm(F, 2)))
    p = int(np.count_nonzero(sr > tol))
    P = Q @ Ur[:, :p]
    if k and p:
        P = P - B @ (B.T @ P)
        P = np.linalg.qr(P)[0]
    return E, P.reshape(d, p)


def fold(U: np.ndarray, sigma: np.ndarray, B: np.ndarray, F: np.ndarray, r: int):
    """One block-incremental update of ``A = U diag(sigma) B^T`` with the pending block ``F``.

    iS-KV summary, section "Block-Incremental Decoding Updates", steps 1-3:
    ``Z = [[Sigma, 0], [F B, F P]]`` of size ``(k+b) x (k+p)``, ``(G, Sigma+, H) = SVD_r(Z)``,
    ``U+ = diag(U, I_b) G`` and ``B+ = [B P] H``. The retained rank is ``min(r, k + p)``.

    Returns ``(U+, sigma+, B+, H, P)``.
    """
    F = np.asarray(F, dtype=np.float64)
    b, d = F.shape
    n, k = U.shape[0], sigma.size
    _, P = residual_basis(F, B)
    p = P.shape[1]
    Z = np.zeros((k + b, k + p))
    Z[:k, :k] = np.diag(sigma)
    Z[k:, :k] = F @ B
    Z[k:, k:] = F @ P
    G, s, Ht = np.linalg.svd(Z, full_matrices=False)
    kp = min(r, k + p)
    G, s, H = G[:, :kp], s[:kp], Ht[:kp].T.copy()
    G = G.copy()
    # sign convention (the page fixes none; singular vectors are sign-ambiguous): new basis
    # vector c points along old basis vector c, i.e. H[c, c] >= 0 for c < k. Reconstructions do
    # not depend on it; the stale-coordinate variant does.
    for c in range(min(k, kp)):
        if H[c, c] < 0:
            H[:, c] = -H[:, c]
            G[:, c] = -G[:, c]
    Ublk = np.zeros((n + b, k + b))
    Ublk[:n, :k] = U
    Ublk[n:, k:] = np.eye(b)
    U_new = Ublk @ G
    B_new = np.hstack([B, P]) @ H
    return U_new, s, B_new, H, P


def fold_from_coords(C: np.ndarray, sigma: np.ndarray, B: np.ndarray, F: np.ndarray, r: int):
    """One fold started from stored coordinates ``C = U diag(sigma)`` (e.g. a GPU state).

    ``U`` is recovered as ``C diag(1/sigma)`` on the columns with ``sigma > 0`` (zero columns
    otherwise), then :func:`fold` runs. Returns ``(C+, sigma+, B+, H_top)`` where ``C+ = U+
    diag(sigma+)`` and ``H_top = H[:k]`` maps old coordinates to new ones.
    """
    sigma = np.asarray(sigma, dtype=np.float64)
    k = sigma.size
    U = np.zeros_like(np.asarray(C, dtype=np.float64)[:, :k])
    nz = sigma > 0
    U[:, nz] = np.asarray(C, dtype=np.float64)[:, :k][:, nz] / sigma[nz]
    U_new, s, B_new, H, _ = fold(U, sigma, np.asarray(B, dtype=np.float64)[:, :k], F, r)
    return U_new * s, s, B_new, H[:k]


class OracleUnit:
    """One (sequence, layer, kv-head, path) of the cache: exact window plus low-rank history.

    iS-KV summary, section "Architecture Overview" (two components per K/V path) and section
    "Reconstruction and Storage".
    """

    def __init__(self, d: int, rank: int, block: int, window: int, rotate: bool = True,
                 fixed_basis: bool = False, coord_bf16: bool = False):
        self.d, self.rank, self.block, self.window, self.rotate = d, rank, block, window, rotate
        self.fixed_basis, self.coord_bf16 = fixed_basis, coord_bf16
        # folds that run the regular update before a fixed basis freezes (fill the rank budget)
        self.adapt_folds = -(-min(rank, d) // block)
        self.U = np.zeros((0, 0))
        self.sigma = np.zeros(0)
        self.B = np.zeros((d, 0))
        self.C_stale = np.zeros((0, 0))      # stored coordinates C (U Sigma, or as the mode keeps them)
        self._exact: list[np.ndarray] = []
        self.t = 0
        self.n = 0
        self.folds = 0
        self.comp_pos = np.zeros(0, dtype=np.int64)   # position of each compressed row
        self.prot_pos = np.zeros(0, dtype=np.int64)   # protected positions (exact for good)
        self.prot_rows = np.zeros((0, d))

    # -- state ---------------------------------------------------------------------------------
    @property
    def k(self) -> int:
        return self.sigma.size

    @property
    def exact(self) -> np.ndarray:
        return np.asarray(self._exact, dtype=np.float64).reshape(len(self._exact), self.d)

    def coords(self) -> np.ndarray:
        """Stored history coordinates ``U Sigma`` (``n x k``; unrotated in the stale mode)."""
        return self.C_stale

    def storage_scalars(self) -> int:
        """Persistent scalars of this path: ``k (n + d + 1)`` factors plus ``d e`` exact values.

        iS-KV summary, section "Reconstruction and Storage" (storage formula, per path).
        """
        return self.k * (self.n + self.d + 1) + self.d * (len(self._exact) + self.prot_pos.size)

    def storage_bytes(self, beta_e: int) -> int:
        """Persistent bytes of this path: the storage formula with bf16 (2 bytes) or fp32 (4 bytes)
        coordinates, fp32 basis and Sigma, and ``beta_e`` bytes per exact scalar."""
        beta_c = 2 if self.coord_bf16 else 4
        return (beta_c * self.k * self.n + 4 * self.k * (self.d + 1)
                + beta_e * self.d * (len(self._exact) + self.prot_pos.size))

    # -- updates -------------------------------------------------------------------------------
    def prefill(self, X: np.ndarray, protected) -> None:
        """Prefill of an empty unit ("Prefill Compression", step 3): rows ``X`` take positions
        ``0 .. T0-1``; the last ``window`` of them form the exact window, ``protected`` positions
        before it stay exact for good, and the remaining rows get one truncated SVD."""
        if self.t:
            raise ValueError("prefill needs an empty unit")
        X = np.asarray(X, dtype=np.float64)
        T0 = X.shape[0]
        end = max(0, T0 - self.window)
        prot = np.asarray(sorted(set(np.asarray(protected).tolist()) & set(range(end))),
                          dtype=np.int64)
        comp = np.asarray(sorted(set(range(end)) - set(prot.tolist())), dtype=np.int64)
        self.prot_pos, self.prot_rows = prot, X[prot]
        self.comp_pos = comp
        if comp.size:
            U, s, B = svd_r(X[comp], self.rank)
            self.U, self.sigma, self.B = U, s, B
            rnd = round_bf16 if self.coord_bf16 else (lambda x: x)
            self.C_stale = rnd(U * s)
            self.n = comp.size
            self.folds = 1                      # the initial factorisation counts as an update
        self._exact = [row.copy() for row in X[end:]]
        self.t = T0

    def append(self, rows: np.ndarray) -> int:
        """Append rows one by one; fold the oldest ``block`` exact rows whenever the window holds
        ``window + block`` rows. Returns the number of folds done."""
        done = 0
        for row in np.atleast_2d(np.asarray(rows, dtype=np.float64)):
            self._exact.append(row.copy())
            self.t += 1
            while len(self._exact) >= self.window + self.block:
                F = np.asarray(self._exact[: self.block])
                p0 = self.t - len(self._exact)          # position of the oldest window row
                del self._exact[: self.block]
                self._fold(F)
                self.comp_pos = np.concatenate([self.comp_pos, np.arange(p0, p0 + self.block)])
                done += 1
        return done

    def _fold(self, F: np.ndarray) -> None:
        k_old = self.k
        rnd = round_bf16 if self.coord_bf16 else (lambda x: x)
        if self.fixed_basis and self.folds >= self.adapt_folds:
            # frozen basis: the block's rows are stored as their coordinates in it
            self.C_stale = np.vstack([self.C_stale, rnd(F @ self.B)])
            self.n += F.shape[0]
            self.folds += 1
            return
        if self.coord_bf16:
            # the update starts from the stored (rounded) coordinates; its result is rounded
            C_new, s, B_new, _ = fold_from_coords(self.C_stale.reshape(self.n, k_old),
                                                  self.sigma, self.B, F, self.rank)
            if self.rotate:
                self.C_stale = rnd(C_new)
            else:
                kp = s.size
                C = np.zeros((self.n, kp))
                m = min(k_old, kp)
                C[:, :m] = self.C_stale[:, :m]
                self.C_stale = np.vstack([C, rnd(F @ B_new)])
            self.U = np.zeros((self.n + F.shape[0], s.size))      # not kept: C is the state
            self.sigma, self.B = s, B_new
            self.n += F.shape[0]
            self.folds += 1
            return
        U_new, s, B_new, H, _ = fold(self.U, self.sigma, self.B, F, self.rank)
        if self.rotate:
            # the regular update (also while a fixed basis is still adapting): C+ = U+ Sigma+
            self.C_stale = U_new * s
        else:
            kp = s.size
            C = np.zeros((self.n, kp))
            m = min(k_old, kp)
            C[:, :m] = self.C_stale[:, :m]
            self.C_stale = np.vstack([C, F @ B_new])
        self.U, self.sigma, self.B = U_new, s, B_new
        self.n += F.shape[0]
        self.folds += 1

    # -- reading -------------------------------------------------------------------------------
    def reconstruct(self) -> np.ndarray:
        """``X~`` in position order ("Reconstruction and Storage"): the compressed row ``j`` at
        position ``C_X[j]`` is ``(U Sigma B^T)[j]``, protected and window rows are exact."""
        out = np.zeros((self.t, self.d))
        if self.n:
            out[self.comp_pos] = self.coords() @ self.B.T
        out[self.prot_pos] = self.prot_rows
        e = len(self._exact)
        out[self.t - e:] = self.exact
        return out


# ----------------------------------------------------------------------------------------------
# Decode attention over the reconstructed cache
# ----------------------------------------------------------------------------------------------
def rope(X: np.ndarray, positions: np.ndarray, theta: float) -> np.ndarray:
    """Rotary embedding, half-split pairs ``(j, j + d/2)`` at angle ``pos * theta^(-2j/d)``."""
    X = np.asarray(X, dtype=np.float64)
    d = X.shape[-1]
    h = d // 2
    omega = theta ** (-2.0 * np.arange(h, dtype=np.float64) / d)
    ang = np.asarray(positions, dtype=np.float64)[:, None] * omega[None, :]
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = X[..., :h], X[..., h:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def attention(q: np.ndarray, K: np.ndarray, V: np.ndarray) -> np.ndarray:
    """Softmax attention of one query over rows of ``K``/``V``, scale ``1/sqrt(d)``, float64."""
    q = np.asarray(q, dtype=np.float64)
    s = (np.asarray(K, dtype=np.float64) @ q) / math.sqrt(q.size)
    s = s - s.max()
    p = np.exp(s)
    p /= p.sum()
    return p @ np.asarray(V, dtype=np.float64)


# ----------------------------------------------------------------------------------------------
# Prefill Compression (protection of outlier keys and their value neighbourhoods)
# ----------------------------------------------------------------------------------------------
def chunk_scores(K_rot: np.ndarray, chunk: int) -> np.ndarray:
    """Step 1 score of every chunk of ``chunk`` consecutive rows (the last one may be shorter):
    the smallest cosine between a rotated key of the chunk and the chunk's mean rotated key."""
    K_rot = np.asarray(K_rot, dtype=np.float64)
    out = []
    for c0 in range(0, K_rot.shape[0], chunk):
        blk = K_rot[c0:c0 + chunk]
        mean = blk.mean(axis=0)
        nm = np.linalg.norm(mean)
        nr = np.linalg.norm(blk, axis=1)
        cos = np.ones(blk.shape[0])
        ok = (nr > 0) & (nm > 0)
        cos[ok] = (blk[ok] @ mean) / (nr[ok] * nm)
        out.append(cos.min())
    return np.asarray(out)


def protected_positions(K: np.ndarray, positions: np.ndarray, chunk: int, m: int, suffix: int,
                        rope_theta: float | None) -> np.ndarray:
    """Step 1: protected key positions ``P_K`` (sorted) among the rows ``K`` at ``positions``
    (consecutive): the ``m`` lowest-scoring chunks plus the last ``suffix`` positions. Keys are
    rotated at their positions first when ``rope_theta`` is given."""
    positions = np.asarray(positions)
    if K.shape[0] == 0:
        return np.zeros(0, dtype=np.int64)
    K_rot = rope(K, positions, rope_theta) if rope_theta is not None else np.asarray(K, float)
    sc = chunk_scores(K_rot, chunk)
    order = np.argsort(sc, kind="stable")[:min(m, sc.size)]
    prot = set()
    for c in order:
        prot.update(positions[c * chunk:(c + 1) * chunk].tolist())
    if suffix > 0:
        prot.update(positions[-suffix:].tolist())
    return np.asarray(sorted(prot), dtype=np.int64)


def value_protected(P_K: np.ndarray, rho: int, lo: int, hi: int) -> np.ndarray:
    """Step 2: every position in ``[lo, hi)`` within ``rho`` tokens of a position of ``P_K``."""
    out = set()
    for p in np.asarray(P_K).tolist():
        out.update(range(max(lo, p - rho), min(hi, p + rho + 1)))
    return np.asarray(sorted(out), dtype=np.int64)


class OracleCache:
    """All units of a cache: ``[layer][sequence][kv-head]`` for the K and V paths."""

    def __init__(self, batch: int, n_layers: int, n_kv_heads: int, n_q_heads: int,
                 head_dim: int, rank_k: int, rank_v: int, block: int, window: int,
                 rope: bool = False, rope_theta: float = 5e5, rotate: bool = True,
                 fixed_basis: bool = False, coord_bf16: bool = False, joint: bool = False):
        self.batch, self.n_layers, self.n_kv, self.n_q = batch, n_layers, n_kv_heads, n_q_heads
        self.d, self.rope, self.theta, self.joint = head_dim, rope, rope_theta, joint
        # joint: one unit per (layer, sequence, path) over rows of length n_kv d, stored as the
        # single entry [layer][seq][0]
        d_unit = n_kv_heads * head_dim if joint else head_dim
        n_units = 1 if joint else n_kv_heads
        self.units = [[[[OracleUnit(d_unit, rank_k if w == 0 else rank_v, block, window, rotate,
                                    fixed_basis, coord_bf16)
                         for w in range(2)] for _ in range(n_units)] for _ in range(batch)]
                      for _ in range(n_layers)]

    def unit(self, layer: int, seq: int, head: int, which: int) -> OracleUnit:
        """The unit that holds kv-head ``head`` (the layer's joint unit when ``joint``)."""
        return self.units[layer][seq][0 if self.joint else head][which]

    def tokens(self, layer: int) -> int:
        return self.units[layer][0][0][0].t

    def _rows(self, X: np.ndarray, head: int) -> np.ndarray:
        """Kv-head ``head``'s columns of a reconstruction of its unit."""
        if not self.joint:
            return X
        return X[:, head * self.d:(head + 1) * self.d]

    def prefill(self, layer: int, K: np.ndarray, V: np.ndarray, chunk: int, m: int, suffix: int,
                rho: int) -> None:
        """Prefill with protection ("Prefill Compression"): ``K``, ``V``: ``[batch][n_kv][T0][d]``
        (pre-RoPE keys) of an empty layer. Per kv-head, ``P_K`` from the rotated keys of the rows
        outside the window, ``P_V`` within ``rho`` of ``P_K``; then each unit's prefill."""
        if self.joint:
            raise ValueError("prefill with protection is per kv-head: not in the joint mode")
        T0 = K.shape[2]
        end = max(0, T0 - self.units[layer][0][0][0].window)
        pos = np.arange(end)
        for s in range(self.batch):
            for h in range(self.n_kv):
                PK = protected_positions(K[s, h, :end], pos, chunk, m, suffix,
                                         self.theta if self.rope else None)
                PV = value_protected(PK, rho, 0, end)
                self.units[layer][s][h][0].prefill(K[s, h], PK)
                self.units[layer][s][h][1].prefill(V[s, h], PV)

    def append(self, layer: int, K: np.ndarray, V: np.ndarray) -> None:
        """``K``, ``V``: ``[batch][n_kv][m][d]`` rows (pre-RoPE keys)."""
        for s in range(self.batch):
            if self.joint:
                # position i's row of the joint unit: the kv-heads' rows side by side
                self.units[layer][s][0][0].append(np.concatenate(list(K[s]), axis=1))
                self.units[layer][s][0][1].append(np.concatenate(list(V[s]), axis=1))
                continue
            for h in range(self.n_kv):
                self.units[layer][s][h][0].append(K[s, h])
                self.units[layer][s][h][1].append(V[s, h])

    def keys_values(self, layer: int, seq: int, head: int):
        """Reconstructed keys (RoPE applied when enabled) and values of one kv-head."""
        K = self._rows(self.unit(layer, seq, head, 0).reconstruct(), head)
        V = self._rows(self.unit(layer, seq, head, 1).reconstruct(), head)
        if self.rope:
            K = rope(K, np.arange(K.shape[0]), self.theta)
        return K, V

    def decode(self, layer: int, q: np.ndarray) -> np.ndarray:
        """``q``: ``[batch][n_q][d]`` (already rotated) -> ``[batch][n_q][d]`` attention output."""
        if self.tokens(layer) == 0:
            raise ValueError("decode over an empty cache")
        G = self.n_q // self.n_kv
        out = np.zeros((self.batch, self.n_q, self.d))
        for s in range(self.batch):
            for h in range(self.n_kv):
                K, V = self.keys_values(layer, s, h)
                for g in range(h * G, (h + 1) * G):
                    out[s, g] = attention(q[s, g], K, V)
        return out

    def reconstruct(self, layer: int, which: int, apply_rope: bool = False) -> np.ndarray:
        """``[batch][n_kv][t][d]`` reconstructed rows of the K (0) or V (1) path."""
        out = []
        for s in range(self.batch):
            row = []
            for h in range(self.n_kv):
                X = self._rows(self.unit(layer, s, h, which).reconstruct(), h)
                if apply_rope and which == 0:
                    X = rope(X, np.arange(X.shape[0]), self.theta)
                row.append(X)
            out.append(row)
        return np.asarray(out)
