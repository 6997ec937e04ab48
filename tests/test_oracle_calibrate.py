"""Pins of the oracle's offline calibration (basis U, coefficient map R).

The pages fix only that queries are approximated on a low-rank basis fixed
offline, weighted by the state.  The pins check the algebra any such
least-squares map must satisfy, and check by brute force on tiny heads -- a
direct minimisation over the calibration data, not through the Gram formula --
that the oracle's basis minimises the averaged squared read error.
"""

import itertools

import numpy as np
import pytest
from scipy import optimize

from oracle import calibration as cal


def _data(rng, Ns, Nq, dk, dv, rank=None, noise=0.1):
    S = rng.standard_normal((Ns, dk, dv)) * rng.uniform(0.2, 2.0, (1, dk, 1))
    if rank is None:
        q = rng.standard_normal((Nq, dk)) * rng.uniform(0.3, 1.5, (1, dk))
    else:
        Q0 = np.linalg.qr(rng.standard_normal((dk, rank)))[0]
        q = rng.standard_normal((Nq, rank)) @ Q0.T + noise * rng.standard_normal((Nq, dk))
    return S, q


def _ridged_gram(S, ridge=1e-8):
    G = cal.gram_states(S)
    return G + ridge * np.trace(G) / G.shape[0] * np.eye(G.shape[0])


@pytest.mark.parametrize("r", [1, 3, 8])
def test_algebraic_properties(r):
    rng = np.random.default_rng(21)
    dk, dv = 16, 12
    S, q = _data(rng, 40, 300, dk, dv)
    U, R = cal.calibrate(S, q, r)
    G = _ridged_gram(S)
    Pi = U @ R
    np.testing.assert_allclose(R @ U, np.eye(r), atol=1e-10)
    np.testing.assert_allclose(Pi @ Pi, Pi, atol=1e-10)
    np.testing.assert_allclose(G @ Pi, (G @ Pi).T, atol=1e-9 * np.abs(G).max())
    np.testing.assert_allclose(U.T @ G @ (np.eye(dk) - Pi), 0.0, atol=1e-9 * np.abs(G).max())


def _data_objective(S, q, U):
    """Mean over states and queries of ||S^T q - S^T U c||^2 with c the per-query
    least-squares coefficients, solved on the stacked data (all states at once)."""
    A = np.concatenate([s.T @ U for s in S], axis=0)  # (Ns*dv, r)
    Y = np.concatenate([np.einsum("ic,ni->cn", s, q) for s in S], axis=0)  # (Ns*dv, Nq)
    c, *_ = np.linalg.lstsq(A, Y, rcond=None)
    res = Y - A @ c
    return float(np.sum(res ** 2) / (S.shape[0] * q.shape[0]))


def _sphere(n):
    i = np.arange(n) + 0.5
    phi = np.arccos(1 - i / n)  # upper hemisphere: u and -u span the same line
    th = np.pi * (1 + 5 ** 0.5) * i
    return np.stack([np.cos(th) * np.sin(phi), np.sin(th) * np.sin(phi), np.cos(phi)], 1)


def _proj(U, R):
    return U @ R


def test_brute_force_rank1_dk3():
    rng = np.random.default_rng(22)
    S, q = _data(rng, 6, 60, 3, 4)
    U, R = cal.calibrate(S, q, 1, ridge=0.0)
    grid = _sphere(4000)
    vals = np.array([_data_objective(S, q, u[:, None]) for u in grid])
    u0 = grid[np.argmin(vals)]
    f = lambda x: _data_objective(S, q, (x / np.linalg.norm(x))[:, None])  # noqa
    x = optimize.minimize(f, u0, method="Nelder-Mead",
                          options={"xatol": 1e-12, "fatol": 1e-15, "maxiter": 20000}).x
    best = x / np.linalg.norm(x)
    ours = U[:, 0] / np.linalg.norm(U[:, 0])
    assert _data_objective(S, q, U) <= f(best) * (1 + 1e-9)
    assert min(np.linalg.norm(best - ours), np.linalg.norm(best + ours)) < 1e-4


def test_brute_force_rank2_dk3():
    rng = np.random.default_rng(23)
    S, q = _data(rng, 5, 80, 3, 3)
    U, R = cal.calibrate(S, q, 2, ridge=0.0)

    def basis(n):
        n = n / np.linalg.norm(n)
        return np.linalg.svd(np.eye(3) - np.outer(n, n))[0][:, :2]

    grid = _sphere(4000)
    vals = np.array([_data_objective(S, q, basis(n)) for n in grid])
    f = lambda x: _data_objective(S, q, basis(x))  # noqa
    x = optimize.minimize(f, grid[np.argmin(vals)], method="Nelder-Mead",
                          options={"xatol": 1e-12, "fatol": 1e-15, "maxiter": 20000}).x
    Ub = basis(x)
    assert _data_objective(S, q, U) <= f(x) * (1 + 1e-9)
    # same span: the G-weighted projector of the brute-force basis equals the oracle's
    G = cal.gram_states(S)
    Rb = np.linalg.solve(Ub.T @ G @ Ub, Ub.T @ G)
    np.testing.assert_allclose(Ub @ Rb, U @ R, atol=1e-4)


def test_isotropic_state_weight_is_query_pca():
    """With G a multiple of I the basis spans the top principal directions of the queries."""
    rng = np.random.default_rng(24)
    dk, r = 12, 4
    O = np.linalg.qr(rng.standard_normal((dk, dk)))[0]
    S = np.stack([O * 1.7, -O * 1.7])  # S S^T = 1.7^2 I for both states
    q = rng.standard_normal((500, dk)) * np.linspace(3.0, 0.2, dk)[None, :]
    U, R = cal.calibrate(S, q, r, ridge=0.0)
    Vt = np.linalg.svd(q, full_matrices=False)[2]
    Ppca = Vt[:r].T @ Vt[:r]
    np.testing.assert_allclose(U @ R, Ppca, atol=1e-9)


def test_exact_low_rank_queries_are_reproduced():
    rng = np.random.default_rng(25)
    dk, dv, r = 16, 8, 5
    S, q = _data(rng, 30, 200, dk, dv, rank=r, noise=0.0)
    U, R = cal.calibrate(S, q, r)
    np.testing.assert_allclose(q @ (U @ R).T, q, atol=1e-9)


def test_complete_rank_is_identity():
    rng = np.random.default_rng(26)
    S, q = _data(rng, 20, 100, 8, 8)
    U, R = cal.calibrate(S, q, 8)
    np.testing.assert_allclose(U @ R, np.eye(8), atol=1e-9)


def test_beats_query_pca_and_random_bases():
    rng = np.random.default_rng(27)
    dk, dv, r = 16, 16, 4
    S, q = _data(rng, 50, 400, dk, dv, rank=8, noise=0.2)
    U, R = cal.calibrate(S, q, r, ridge=0.0)
    ours = _data_objective(S, q, U)
    Vt = np.linalg.svd(q, full_matrices=False)[2]
    assert ours <= _data_objective(S, q, Vt[:r].T) * (1 + 1e-12)
    for _ in range(20):
        assert ours <= _data_objective(S, q, rng.standard_normal((dk, r))) * (1 + 1e-12)


# ---- heterogeneous per-head rank (average rank budget) ----------------------

def _rand_grams(rng, dk, ns=40, nq=60):
    S = rng.standard_normal((ns, dk, 5))
    q = rng.standard_normal((nq, dk)) @ rng.standard_normal((dk, dk))
    return cal.gram_states(S), cal.gram_queries(q)


def test_residual_is_the_tail_of_the_spectrum():
    """Closed form: at rank r the averaged read error of the basis equals the sum of the
    eigenvalues of G^1/2 C G^1/2 past the r largest (pins spectrum_from_grams to objective)."""
    rng = np.random.default_rng(21)
    G, C = _rand_grams(rng, 7)
    lam = cal.spectrum_from_grams(G, C, ridge=0.0)
    assert np.all(np.diff(lam) <= 1e-12)
    for r in range(0, 8):
        if r == 0:
            err = np.trace(C @ G)
        else:
            U, R = cal.basis_from_grams(G, C, r, ridge=0.0)
            err = cal.objective(G, C, U, R)
        assert err == pytest.approx(lam[r:].sum(), rel=1e-9, abs=1e-9 * lam.sum())


def test_allocate_ranks_minimises_total_error_by_brute_force():
    rng = np.random.default_rng(22)
    for trial in range(20):
        H, n, r_max = 3, 5, 4
        r_avg = int(rng.integers(1, r_max + 1))
        spectra = -np.sort(-rng.exponential(size=(H, n)) * rng.uniform(0.2, 3.0, size=(H, 1)), axis=1)
        ranks = cal.allocate_ranks(spectra, r_avg, r_max)
        assert ranks.sum() == H * r_avg and ranks.max() <= r_max
        err = lambda rk: sum(spectra[h, rk[h]:].sum() for h in range(H))
        best = min(err(rk) for rk in itertools.product(range(r_max + 1), repeat=H) if sum(rk) == H * r_avg)
        assert err(ranks) == pytest.approx(best, rel=1e-12)


def test_allocate_ranks_equal_spectra_and_cap():
    lam = np.array([[5.0, 4.0, 3.0, 2.0, 1.0]] * 4)
    assert cal.allocate_ranks(lam, 3, 5).tolist() == [3, 3, 3, 3]
    dominant = np.array([[100.0, 90, 80, 70, 60], [1.0, 0.5, 0.2, 0.1, 0.05]])
    assert cal.allocate_ranks(dominant, 2, 3).tolist() == [3, 1]  # capped at r_max = 3
    assert cal.allocate_ranks(dominant, 2, 5).tolist() == [4, 0]


def test_ranked_basis_is_the_truncated_full_basis():
    rng = np.random.default_rng(23)
    H, dk = 4, 6
    S = rng.standard_normal((30, H, dk, 4)) * rng.uniform(0.3, 2.0, size=(1, H, 1, 1))
    q = rng.standard_normal((H, 50, dk))
    U, R, ranks, spectra = cal.calibrate_heads_ranked(S, q, 2, 4)
    U4, R4 = cal.calibrate_heads(S, q, 4)
    assert ranks.sum() == 2 * H
    for h in range(H):
        rh = ranks[h]
        assert np.all(U[h][:, rh:] == 0) and np.all(R[h][rh:] == 0)
        np.testing.assert_allclose(U[h][:, :rh], U4[h][:, :rh], rtol=0, atol=0)
        if rh:  # the same projector as a rank-r_h calibration of that head alone
            Ur, Rr = cal.calibrate(S[:, h], q[h], int(rh))
            np.testing.assert_allclose(U[h] @ R[h], Ur @ Rr, atol=1e-9)


# ---- query PCA (the unweighted basis the state weighting is compared with) ----

def test_query_pca_axis_aligned_closed_form():
    """Queries +-s_i e_i give C = diag(s_i^2) / dk exactly: the basis is the r axes with the
    largest s_i, in descending order, and R = U^T."""
    dk, r = 9, 4
    s = np.array([0.5, 3.0, 1.0, 7.0, 0.1, 2.0, 5.0, 0.7, 4.0])
    q = np.concatenate([np.diag(s), -np.diag(s)])
    U, R = cal.query_pca(q, r)
    top = [3, 6, 8, 1]  # s = 7, 5, 4, 3
    np.testing.assert_allclose(np.abs(U), np.eye(dk)[:, top], atol=1e-12)
    np.testing.assert_array_equal(R, U.T)


def test_query_pca_is_the_svd_projection():
    """Eckart-Young: the unweighted residual mean ||q - U R q||^2 of the PCA basis is the sum of
    the trailing squared singular values of the query matrix / Nq, and the projector is the
    span of the top right singular vectors (numpy's SVD, a different routine from eigh)."""
    rng = np.random.default_rng(31)
    dk, r, Nq = 14, 5, 300
    q = rng.standard_normal((Nq, dk)) * np.linspace(2.5, 0.3, dk)[None, :] @ np.linalg.qr(
        rng.standard_normal((dk, dk)))[0]
    U, R = cal.query_pca(q, r)
    np.testing.assert_allclose(R @ U, np.eye(r), atol=1e-12)
    sv, Vt = np.linalg.svd(q, full_matrices=False)[1:]
    np.testing.assert_allclose(U @ R, Vt[:r].T @ Vt[:r], atol=1e-10)
    resid = np.mean(np.sum((q - q @ (U @ R).T) ** 2, axis=1))
    np.testing.assert_allclose(resid, np.sum(sv[r:] ** 2) / Nq, rtol=1e-10)


def test_query_pca_equals_weighted_basis_under_isotropic_states():
    """The state-weighted calibration with S S^T the same multiple of I for every state has the
    same projector as the query-PCA basis."""
    rng = np.random.default_rng(32)
    dk, r = 10, 3
    O = np.linalg.qr(rng.standard_normal((dk, dk)))[0]
    S = np.stack([O * 0.8, O[:, ::-1] * 0.8])
    q = rng.standard_normal((400, dk)) * np.linspace(2.0, 0.5, dk)[None, :]
    Uw, Rw = cal.calibrate(S, q, r, ridge=0.0)
    Up, Rp = cal.query_pca_heads(q[None], r)
    np.testing.assert_allclose(Uw @ Rw, Up[0] @ Rp[0], atol=1e-9)
    # and the state weighting wins on a non-isotropic state population
    S2, q2 = _data(rng, 40, 300, dk, 6, rank=6, noise=0.3)
    U2, R2 = cal.calibrate(S2, q2, r, ridge=0.0)
    Up2, Rp2 = cal.query_pca(q2, r)
    G, C = cal.gram_states(S2), cal.gram_queries(q2)
    assert cal.objective(G, C, U2, R2) < cal.objective(G, C, Up2, Rp2)
