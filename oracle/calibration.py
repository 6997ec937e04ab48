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


def objective(G: np.ndarray, C: np.ndarray, U: np.ndarray, R: np.ndarray) -> float:
    """Averaged squared read error tr(C (I - U R)^T G (I - U R)) of a basis/map pair."""
    E = np.eye(G.shape[0]) - U @ R
    return float(np.trace(C @ E.T @ G @ E))
