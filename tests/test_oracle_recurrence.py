"""Pins of the oracle's per-token recurrences, exact read and windowed update.

Each test checks the oracle against something other than itself: dense-matrix
products built from the update rules, closed forms, semantic properties of the
delta rule, special cases where one family reduces to another, and the fp64
bitwise identity between the windowed update and the per-step recurrence that
the SketchSSM pages imply (the state is updated exactly, once per window, and no
approximation error is written into it).
"""

import numpy as np
import pytest

KINDS = ["mamba2", "gdn", "kda"]


def _tokens(rng, kind, T, N, dk, dv, unit_k=False):
    K = rng.standard_normal((T, N, dk))
    if unit_k:
        K /= np.linalg.norm(K, axis=-1, keepdims=True)
    V = rng.standard_normal((T, N, dv))
    A = rng.uniform(0.3, 1.0, (T, N, dk) if kind == "kda" else (T, N))
    Bt = rng.uniform(0.05, 1.0, (T, N))
    Q = rng.standard_normal((T, N, dk))
    return K, V, A, Bt, Q


def _dense_M(kind, k, a, b):
    """Transition matrix M_t of S_t = M_t S_{t-1} + b k v^T as a dense dk x dk matrix."""
    dk = k.shape[0]
    I = np.eye(dk)
    if kind == "mamba2":
        return a * I
    P = I - b * np.outer(k, k)
    if kind == "gdn":
        return a * P
    return P @ np.diag(a)


@pytest.mark.parametrize("kind", KINDS)
def test_dense_brute_force(orc, kind):
    rng = np.random.default_rng(1)
    N, dk, dv, T = 3, 4, 5, 7
    S0 = rng.standard_normal((N, dk, dv))
    K, V, A, Bt, Q = _tokens(rng, kind, T, N, dk, dv)
    S, O = orc.exact_steps(kind, S0, K, V, A, Bt, Q)
    for n in range(N):
        Sd = S0[n].copy()
        for t in range(T):
            b = 1.0 if kind == "mamba2" else Bt[t, n]
            Sd = _dense_M(kind, K[t, n], A[t, n], b) @ Sd + b * np.outer(K[t, n], V[t, n])
            np.testing.assert_allclose(O[t, n], Sd.T @ Q[t, n], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(S[n], Sd, rtol=1e-12, atol=1e-12)


def test_mamba2_closed_form(orc):
    rng = np.random.default_rng(2)
    N, dk, dv, T = 4, 8, 6, 11
    S0 = rng.standard_normal((N, dk, dv))
    K, V, A, _, _ = _tokens(rng, "mamba2", T, N, dk, dv)
    S, _ = orc.exact_steps("mamba2", S0, K, V, A)
    gam = np.cumprod(A, axis=0)  # Gamma_t = a_1 ... a_t
    for n in range(N):
        ref = gam[-1, n] * S0[n]
        for t in range(T):
            ref = ref + (gam[-1, n] / gam[t, n]) * np.outer(K[t, n], V[t, n])
        np.testing.assert_allclose(S[n], ref, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("kind", ["gdn", "kda"])
def test_delta_rule_overwrites_key(orc, kind):
    """No decay, beta = 1, unit key: afterwards reading with the key returns exactly its value."""
    rng = np.random.default_rng(3)
    N, dk, dv, T = 5, 16, 8, 6
    S0 = rng.standard_normal((N, dk, dv))
    K, V, _, _, _ = _tokens(rng, kind, T, N, dk, dv, unit_k=True)
    A = np.ones((T, N, dk) if kind == "kda" else (T, N))
    Bt = np.ones((T, N))
    S = S0
    for t in range(T):
        S, O = orc.exact_steps(kind, S, K[t:t + 1], V[t:t + 1], A[t:t + 1], Bt[t:t + 1], K[t:t + 1])
        np.testing.assert_allclose(O[0], V[t], rtol=1e-12, atol=1e-12)


def test_delta_rule_idempotent_write(orc):
    rng = np.random.default_rng(4)
    N, dk, dv = 3, 8, 8
    S0 = rng.standard_normal((N, dk, dv))
    K, V, _, _, _ = _tokens(rng, "gdn", 1, N, dk, dv, unit_k=True)
    ones = np.ones((1, N))
    S1, _ = orc.exact_steps("gdn", S0, K, V, ones, ones)
    S2, _ = orc.exact_steps("gdn", S1, K, V, ones, ones)
    np.testing.assert_allclose(S2, S1, rtol=1e-12, atol=1e-12)


def test_kda_with_uniform_decay_is_gdn(orc):
    rng = np.random.default_rng(5)
    N, dk, dv, T = 4, 12, 10, 9
    S0 = rng.standard_normal((N, dk, dv))
    K, V, A, Bt, _ = _tokens(rng, "gdn", T, N, dk, dv)
    Sg, _ = orc.exact_steps("gdn", S0, K, V, A, Bt)
    Sk, _ = orc.exact_steps("kda", S0, K, V, np.repeat(A[..., None], dk, axis=-1), Bt)
    np.testing.assert_allclose(Sk, Sg, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("kind", ["gdn", "kda"])
def test_zero_beta_is_pure_decay(orc, kind):
    rng = np.random.default_rng(6)
    N, dk, dv = 3, 6, 7
    S0 = rng.standard_normal((N, dk, dv))
    K, V, A, _, _ = _tokens(rng, kind, 1, N, dk, dv)
    S, _ = orc.exact_steps(kind, S0, K, V, A, np.zeros((1, N)))
    ref = S0 * (A[0][:, :, None] if kind == "kda" else A[0][:, None, None])
    np.testing.assert_array_equal(S, ref)


def test_read_returns_rows(orc):
    rng = np.random.default_rng(7)
    S = rng.standard_normal((2, 5, 3))
    for i in range(5):
        q = np.zeros((2, 5))
        q[:, i] = 1.0
        np.testing.assert_array_equal(orc.read(S, q), S[:, i, :])


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("W", [1, 3, 4])
def test_window_update_bitwise_equals_per_step(orc, kind, W):
    """fp64: the state after each window equals, bit for bit, the per-step state."""
    rng = np.random.default_rng(8)
    N, dk, dv, T = 4, 8, 6, 3 * W + 2  # three full windows and a partial one
    S0 = rng.standard_normal((N, dk, dv))
    K, V, A, Bt, _ = _tokens(rng, kind, T, N, dk, dv)
    U = rng.standard_normal((N, dk, 3))
    S = S0
    for t0 in range(0, T, W):
        t1 = min(T, t0 + W)
        S, P = orc.update_window(kind, S, U, K[t0:t1], V[t0:t1], A[t0:t1], Bt[t0:t1])
        Sref, _ = orc.exact_steps(kind, S0, K[:t1], V[:t1], A[:t1], Bt[:t1])
        assert np.array_equal(S, Sref), (kind, W, t0)
        np.testing.assert_allclose(P, np.einsum("nic,nim->ncm", Sref, U), rtol=1e-13, atol=1e-13)


def test_bf16_rounding_matches_torch(orc):
    import torch

    rng = np.random.default_rng(9)
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-8, 8, 20000),
                        [0.0, -0.0, 1.0, 1.00390625, 1.005859375, 65504.0, 3.0e38]])
    ours = orc.round_bf16(x)
    ref = torch.from_numpy(x).float().to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(ours, ref)


def test_bf16_state_rounds_once_per_window(orc):
    rng = np.random.default_rng(10)
    N, dk, dv, W = 2, 8, 8, 4
    S0 = orc.round_bf16(rng.standard_normal((N, dk, dv)))
    K, V, A, Bt, _ = _tokens(rng, "gdn", W, N, dk, dv)
    U = rng.standard_normal((N, dk, 2))
    S, P = orc.update_window("gdn", S0, U, K, V, A, Bt, bf16_state=True)
    Sx, _ = orc.update_window("gdn", S0, U, K, V, A, Bt)
    np.testing.assert_array_equal(S, orc.round_bf16(Sx))
    np.testing.assert_allclose(P, np.einsum("nic,nim->ncm", S, U), rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("kind", KINDS)
def test_bf16_state_rounds_after_every_step(orc, kind):
    """The full-read path with a bf16 state stores the state after every token: the
    token's read sees the fp64 update of the stored (rounded) state, and the stored
    state is that update rounded to bf16.  Restated with dense transition matrices
    stepped in fp64 and torch's bf16 conversion after each step."""
    import torch

    def bf16(x):
        return torch.from_numpy(np.ascontiguousarray(x)).float().to(torch.bfloat16).double().numpy()

    rng = np.random.default_rng(11)
    N, dk, dv, T = 2, 6, 5, 9
    S0 = bf16(rng.standard_normal((N, dk, dv)))
    K, V, A, Bt, Q = _tokens(rng, kind, T, N, dk, dv)
    S, O = orc.exact_steps(kind, S0, K, V, A, Bt, Q, bf16_state=True)
    for n in range(N):
        Sd = S0[n].copy()
        for t in range(T):
            b = 1.0 if kind == "mamba2" else Bt[t, n]
            Sd = _dense_M(kind, K[t, n], A[t, n], b) @ Sd + b * np.outer(K[t, n], V[t, n])
            np.testing.assert_allclose(O[t, n], Sd.T @ Q[t, n], rtol=1e-12, atol=1e-12)
            Sd = bf16(Sd)
        np.testing.assert_array_equal(S[n], Sd)
    # the rounding is not the identity on these values: an unrounded run differs
    Sx, Ox = orc.exact_steps(kind, S0, K, V, A, Bt, Q)
    assert np.abs(Sx - S).max() > 1e-4 and np.abs(Ox - O).max() > 1e-4
