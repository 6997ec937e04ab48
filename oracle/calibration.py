"""Oracle calibration of the offline basis U and the coefficient map R (fp64, numpy).

TEST INFRASTRUCTURE: only the tests, the smoke check and the bench's CPU
baseline leg use this module; the product path never does.

Method: "SketchSSM: Write to the Full State, Read from a Compact Sketch"
(arXiv 2609.33051v1), Abstract -- queries are approximated in a low-rank,
state-weighted way, on basis vectors that are fixed offline; agihunt digest of
the same paper, bullet "Core idea".  The pages give no formula.  The reading
taken here, per head:

  G = mean over calibration states of S S^T          (dk x dk, state weighting)
  G <- G + ridge * (tr G / dk) * I                   (guard; G is full rank here)
  C = mean over calibration queries of q q^T         (dk x dk)
  R = (U^T G U)^-1 U^T G                             (G-weighted least squares:
                                                      c = R q minimises
                                                      ||S^T (q - U c)||^2 averaged
                                                      over the calibration states)
  U = G^-1/2 V_r, V_r the top-r eigenvectors of G^1/2 C G^1/2, eigenvalues in
      descending order, ties by index.  This U minimises the same averaged
      objective E_q E_S ||S^T (q - U R q)||^2 over all rank-r bases; any basis of
      the same span gives the same U R and the same sketch outputs.

Library primitives used as steps: numpy.linalg.eigh (symmetric eigensolver) and
numpy.linalg.solve.  Parity status: U R is pinned by its algebraic properties
and by brute-force minimisation on tiny heads (tests/test_oracle_calibrate.py);
the choice of objective itself is a reading, not fixed by the pages.
"""

from __future__ import annotations

import numpy as np


def gram_states(S_cal: np.ndarray) -> np.ndarray:
    """G = (1/Ns) sum_s S_s S_s^T for S_cal [Ns, dk, dv] (logical layout)."""
    S = np.asarray(S_cal, dtype=np.float64)
    return np.einsum("sic,sjc->ij", S, S) / S.shape[0]


def gram_queries(q_cal: np.ndarray) -> np.ndarray:
    """C = (1/Nq) sum_n q_n q_n^T for q_cal [Nq, dk]."""
    q = np.asarray(q_cal, dtype=np.float64)
    return q.T @ q / q.shape[0]


def _sym_power(G: np.ndarray, p: float) -> np.ndarray:
    lam, E = np.linalg.eigh(G)
    return (E * lam[None, :] ** p) @ E.T


def basis_from_grams(G: np.ndarray, C: np.ndarray, r: int, ridge: float = 1e-8):
    """U [dk, r] and R [r, dk] from the state Gram G and the query Gram C."""
    dk = G.shape[0]
    G = G + ridge * (np.trace(G) / dk) * np.eye(dk)
    Gh = _sym_power(G, 0.5)
    Ghi = _sym_power(G, -0.5)
    A = Gh @ C @ Gh
    A = 0.5 * (A + A.T)
    lam, V = np.linalg.eigh(A)
    order = np.argsort(-lam, kind="stable")[:r]
    U = Ghi @ V[:, order]
    R = np.linalg.solve(U.T @ G @ U, U.T @ G)
    return U, R


def calibrate(S_cal: np.ndarray, q_cal: np.ndarray, r: int, ridge: float = 1e-8):
    """Calibrate one head: S_cal [Ns, dk, dv] logical states, q_cal [Nq, dk]."""
    return basis_from_grams(gram_states(S_cal), gram_queries(q_cal), r, ridge)


def calibrate_heads(S_cal: np.ndarray, q_cal: np.ndarray, r: int, ridge: float = 1e-8):
    """All heads: S_cal [Ns, H, dk, dv] logical, q_cal [H, Nq, dk] -> U [H,dk,r], R [H,r,dk]."""
    S_cal = np.asarray(S_cal, dtype=np.float64)
    q_cal = np.asarray(q_cal, dtype=np.float64)
    H = S_cal.shape[1]
    Us, Rs = [], []
    for h in range(H):
        U, R = calibrate(S_cal[:, h], q_cal[h], r, ridge)
        Us.append(U)
        Rs.append(R)
    return np.stack(Us), np.stack(Rs)


# ---------------------------------------------------------------------------
# Query PCA, the unweighted alternative that the state weighting is measured
# against.  The abstract calls the method's approximation state-weighted; the
# plain alternative ignores the states and keeps the r principal directions of
# the calibration queries: U = the eigenvectors of C with the r largest
# eigenvalues (ties by index), R = U^T, the orthogonal projection onto their span.


def query_pca(q_cal: np.ndarray, r: int):
    """One head: U [dk, r] orthonormal, R = U^T [r, dk]."""
    lam, V = np.linalg.eigh(gram_queries(q_cal))
    order = np.argsort(-lam, kind="stable")[:r]
    U = V[:, order]
    return U, U.T.copy()


def query_pca_heads(q_cal: np.ndarray, r: int):
    """All heads: q_cal [H, Nq, dk] -> U [H, dk, r], R [H, r, dk]."""
    q_cal = np.asarray(q_cal, dtype=np.float64)
    pairs = [query_pca(q_cal[h], r) for h in range(q_cal.shape[0])]
    return np.stack([u for u, _ in pairs]), np.stack([rr for _, rr in pairs])


def objective(G: np.ndarray, C: np.ndarray, U: np.ndarray, R: np.ndarray) -> float:
    """Averaged squared read error tr(C (I - U R)^T G (I - U R)) of a basis/map pair."""
    E = np.eye(G.shape[0]) - U @ R
    return float(np.trace(C @ E.T @ G @ E))


# ---------------------------------------------------------------------------
# Heterogeneous per-head rank.  SketchSSM (arXiv 2609.33051v1) and the agihunt
# digest quote the traffic reduction at an *average* sketch rank of 8, so ranks
# may differ across heads.  The pages do not say how they are chosen; the reading
# taken here: spend a total rank budget of H * r_avg where it removes the most
# read error.  With the basis above, the averaged read error of head h at rank r
# is sum_{i > r} lam_{h,i}, the eigenvalues of G^1/2 C G^1/2 past the r largest
# (see residual_check in the tests), so the total error over heads is smallest
# when the budget takes the H * r_avg largest eigenvalues of all heads together,
# at most r_max per head.  Ties: larger value first, then lower head, then lower
# index.  Head h's basis is the first r_h columns of its rank-r_max basis (U^T G U
# is the identity, so its map R is the first r_h rows of the rank-r_max map).


def spectrum_from_grams(G: np.ndarray, C: np.ndarray, ridge: float = 1e-8) -> np.ndarray:
    """Eigenvalues of G^1/2 C G^1/2 (G with the ridge guard), in descending order."""
    dk = G.shape[0]
    G = G + ridge * (np.trace(G) / dk) * np.eye(dk)
    Gh = _sym_power(G, 0.5)
    A = Gh @ C @ Gh
    A = 0.5 * (A + A.T)
    return np.sort(np.linalg.eigvalsh(A))[::-1]


def allocate_ranks(spectra: np.ndarray, r_avg: int, r_max: int) -> np.ndarray:
    """Per-head ranks from per-head descending spectra [H, n] (n >= r_max): the H * r_avg
    largest values over all heads, at most r_max per head."""
    lam = np.asarray(spectra, dtype=np.float64)[:, :r_max]
    H = lam.shape[0]
    budget = H * r_avg
    # candidates (value, head, index), ordered by value descending, then head, then index
    order = sorted(((-lam[h, i], h, i) for h in range(H) for i in range(lam.shape[1])))
    ranks = np.zeros(H, dtype=np.int64)
    for _, h, _ in order[:budget]:
        ranks[h] += 1
    return ranks


def calibrate_heads_ranked(S_cal: np.ndarray, q_cal: np.ndarray, r_avg: int, r_max: int,
                           ridge: float = 1e-8):
    """All heads with an average rank: U [H,dk,r_max] and R [H,r_max,dk] whose columns / rows past
    head h's rank are zero, the ranks [H], and the spectra [H, dk]."""
    S_cal = np.asarray(S_cal, dtype=np.float64)
    q_cal = np.asarray(q_cal, dtype=np.float64)
    H = S_cal.shape[1]
    spectra = np.stack([spectrum_from_grams(gram_states(S_cal[:, h]), gram_queries(q_cal[h]), ridge)
                        for h in range(H)])
    ranks = allocate_ranks(spectra, r_avg, r_max)
    U, R = calibrate_heads(S_cal, q_cal, r_max, ridge)
    for h in range(H):
        U[h][:, ranks[h]:] = 0.0
        R[h][ranks[h]:, :] = 0.0
    return U, R, ranks, spectra
