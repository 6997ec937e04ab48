"""Pins of the oracle's sketch read and of the decode schedules.

The SketchSSM pages fix what the sketch read must reduce to: with a complete
basis it is the exact read; a query that lies in the span of the basis is
reconstructed exactly from the stored basis outputs; the buffered tokens
contribute exactly; the approximation touches only the window-start state.
"""

import numpy as np
import pytest

KINDS = ["mamba2", "gdn", "kda"]


def _setup(rng, kind, T, N, dk, dv, unit_k=True):
    S0 = rng.standard_normal((N, dk, dv))
    K = rng.standard_normal((T, N, dk))
    if unit_k:
        K /= np.linalg.norm(K, axis=-1, keepdims=True)
    tok = {
        "k": K,
        "v": rng.standard_normal((T, N, dv)),
        "alpha": rng.uniform(0.5, 1.0, (T, N, dk) if kind == "kda" else (T, N)),
        "beta": None if kind == "mamba2" else rng.uniform(0.05, 1.0, (T, N)),
        "q": rng.standard_normal((T, N, dk)),
    }
    return S0, tok


def _left_inverse_pair(rng, N, dk, r):
    U = rng.standard_normal((N, dk, r))
    R = np.stack([np.linalg.solve(u.T @ u, u.T) for u in U])
    return U, R


@pytest.mark.parametrize("kind", KINDS)
def test_complete_basis_gives_exact_read(orc, kind):
    rng = np.random.default_rng(11)
    N, dk, dv, W, T = 3, 8, 6, 4, 14
    S0, tok = _setup(rng, kind, T, N, dk, dv)
    eye = np.broadcast_to(np.eye(dk), (N, dk, dk))
    Os, Ss, _ = orc.sketch_path(kind, S0, eye, eye, tok, W)
    Of, Sf = orc.fullread_path(kind, S0, tok)
    np.testing.assert_allclose(Os, Of, rtol=1e-12, atol=1e-12)
    assert np.array_equal(Ss, Sf)


@pytest.mark.parametrize("kind", KINDS)
def test_buffered_decomposition(orc, kind):
    """S_j^T q_j = S0^T q~ + o_buf at every step of a window, for any basis."""
    rng = np.random.default_rng(12)
    N, dk, dv, W = 4, 8, 5, 6
    S0, tok = _setup(rng, kind, W, N, dk, dv)
    U, R = _left_inverse_pair(rng, N, dk, 3)
    _, P = orc.update_window(kind, S0, U)
    for j in range(1, W + 1):
        sl = slice(0, j)
        _, qt, ob = orc.sketch_read(kind, P, R, tok["q"][j - 1], tok["k"][sl], tok["v"][sl],
                                    tok["alpha"][sl], None if tok["beta"] is None else tok["beta"][sl],
                                    return_parts=True)
        Sj, _ = orc.exact_steps(kind, S0, tok["k"][sl], tok["v"][sl], tok["alpha"][sl],
                                None if tok["beta"] is None else tok["beta"][sl])
        exact = np.einsum("nic,ni->nc", Sj, tok["q"][j - 1])
        np.testing.assert_allclose(np.einsum("nic,ni->nc", S0, qt) + ob, exact, rtol=1e-11, atol=1e-11)


@pytest.mark.parametrize("kind", KINDS)
def test_carried_query_dense_brute_force(orc, kind):
    """q~ = (M_j ... M_1)^T q with dense transition matrices, tiny heads."""
    rng = np.random.default_rng(13)
    N, dk, dv, j = 2, 4, 4, 3
    S0, tok = _setup(rng, kind, j, N, dk, dv, unit_k=False)
    U, R = _left_inverse_pair(rng, N, dk, 2)
    _, P = orc.update_window(kind, S0, U)
    _, qt, _ = orc.sketch_read(kind, P, R, tok["q"][j - 1], tok["k"], tok["v"], tok["alpha"],
                               tok["beta"], return_parts=True)
    for n in range(N):
        M = np.eye(dk)
        for t in range(j):
            k = tok["k"][t, n]
            a = tok["alpha"][t, n]
            b = 1.0 if kind == "mamba2" else tok["beta"][t, n]
            if kind == "mamba2":
                Mt = a * np.eye(dk)
            elif kind == "gdn":
                Mt = a * (np.eye(dk) - b * np.outer(k, k))
            else:
                Mt = (np.eye(dk) - b * np.outer(k, k)) @ np.diag(a)
            M = Mt @ M
        np.testing.assert_allclose(qt[n], M.T @ tok["q"][j - 1, n], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("kind", KINDS)
def test_error_is_projection_residual(orc, kind):
    """o_sketch - o_exact = -S0^T (I - U R) q~ (the only approximation)."""
    rng = np.random.default_rng(14)
    N, dk, dv, j = 3, 10, 7, 5
    S0, tok = _setup(rng, kind, j, N, dk, dv)
    U, R = _left_inverse_pair(rng, N, dk, 4)
    _, P = orc.update_window(kind, S0, U)
    o, qt, _ = orc.sketch_read(kind, P, R, tok["q"][j - 1], tok["k"], tok["v"], tok["alpha"],
                               tok["beta"], return_parts=True)
    Sj, _ = orc.exact_steps(kind, S0, tok["k"], tok["v"], tok["alpha"], tok["beta"])
    exact = np.einsum("nic,ni->nc", Sj, tok["q"][j - 1])
    resid = qt - np.einsum("nim,nmk,nk->ni", U, R, qt)
    np.testing.assert_allclose(o - exact, -np.einsum("nic,ni->nc", S0, resid), rtol=1e-10, atol=1e-11)


@pytest.mark.parametrize("kind", KINDS)
def test_window_of_one_is_rank_r_projection(orc, kind):
    """W = 1: each output is the full read of the projected carried query plus the token term."""
    rng = np.random.default_rng(15)
    N, dk, dv, T, r = 3, 8, 6, 5, 3
    S0, tok = _setup(rng, kind, T, N, dk, dv)
    U, R = _left_inverse_pair(rng, N, dk, r)
    Os, _, _ = orc.sketch_path(kind, S0, U, R, tok, 1)
    S = S0
    for t in range(T):
        sl = slice(t, t + 1)
        beta = None if tok["beta"] is None else tok["beta"][sl]
        _, P = orc.update_window(kind, S, U)
        _, qt, ob = orc.sketch_read(kind, P, R, tok["q"][t], tok["k"][sl], tok["v"][sl],
                                    tok["alpha"][sl], beta, return_parts=True)
        proj = np.einsum("nim,nmk,nk->ni", U, R, qt)
        np.testing.assert_allclose(Os[t], orc.read(S, proj) + ob, rtol=1e-11, atol=1e-11)
        S, _ = orc.exact_steps(kind, S, tok["k"][sl], tok["v"][sl], tok["alpha"][sl], beta)


@pytest.mark.parametrize("kind", KINDS)
def test_linear_in_query(orc, kind):
    rng = np.random.default_rng(16)
    N, dk, dv, j = 2, 8, 8, 4
    S0, tok = _setup(rng, kind, j, N, dk, dv)
    U, R = _left_inverse_pair(rng, N, dk, 3)
    _, P = orc.update_window(kind, S0, U)
    q1, q2 = rng.standard_normal((2, N, dk))
    f = lambda q: orc.sketch_read(kind, P, R, q, tok["k"], tok["v"], tok["alpha"], tok["beta"])  # noqa
    np.testing.assert_allclose(f(2.0 * q1 - 3.0 * q2), 2.0 * f(q1) - 3.0 * f(q2), rtol=1e-11, atol=1e-11)


def test_mamba2_query_in_basis_span_is_exact(orc):
    """Scalar decay keeps q~ on the query's line, so queries in span(U) read exactly."""
    rng = np.random.default_rng(17)
    N, dk, dv, W, T, r = 3, 16, 8, 4, 12, 5
    S0, tok = _setup(rng, "mamba2", T, N, dk, dv, unit_k=False)
    U, R = _left_inverse_pair(rng, N, dk, r)
    tok["q"] = np.einsum("nim,tnm->tni", U, rng.standard_normal((T, N, r)))
    Os, _, _ = orc.sketch_path("mamba2", S0, U, R, tok, W)
    Of, _ = orc.fullread_path("mamba2", S0, tok)
    np.testing.assert_allclose(Os, Of, rtol=1e-11, atol=1e-11)


def test_sketch_path_never_changes_state(orc):
    """The state after the sketch schedule is the exact state (error never written back)."""
    rng = np.random.default_rng(18)
    N, dk, dv, W, T = 2, 8, 8, 4, 12
    for kind in KINDS:
        S0, tok = _setup(rng, kind, T, N, dk, dv)
        U, R = _left_inverse_pair(rng, N, dk, 2)
        _, Ss, Ps = orc.sketch_path(kind, S0, U, R, tok, W)
        _, Sf = orc.fullread_path(kind, S0, tok)
        assert np.array_equal(Ss, Sf)
        np.testing.assert_allclose(Ps, np.einsum("nic,nim->ncm", Sf, U), rtol=1e-13, atol=1e-13)
