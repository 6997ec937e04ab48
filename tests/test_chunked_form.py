"""The chunked (WY) form that the tensor-core window update evaluates, checked in fp64 against the
oracle's token-by-token recurrence (CPU).

Per head, with tokens t = 0..n-1, decays a_t, strengths b_t, g_t = a_0 ... a_t and
gamma_{t,s} = a_{s+1} ... a_t (products only), the window's update is
    S_n = G S_0 + sum_s Gamma_{n-1,s} k_s w_s^T,     w = (I + A)^-1 y,
    y_t = b_t v_t - b_t S_0^T (g_t o k_t),           A[t][s] = b_t sum_i gamma_{t,s,i} k_t,i k_s,i (s < t),
with scalar decays for Gated DeltaNet (G = g_{n-1} I) and per-key-channel decays for KDA; the sketch
is P = S_n^T U = S_0^T (g_{n-1} o U) + sum_s w_s ((gamma_{n-1,s} o k_s) . U).  The algebra is
restated here from the recurrences; the oracle is the reference it must match, including zero
(reset) and tiny decays, where nothing may be divided.
"""

import numpy as np
import pytest


def _chunked(kind, S0, U, K, V, A, Bt):
    n, dk = K.shape
    a = A if kind == "kda" else np.repeat(A[:, None], dk, axis=1)  # [n, dk] per-channel decays
    g = np.cumprod(a, axis=0)                                         # g_t
    def gam(t, s):                                                    # gamma_{t,s} = a_{s+1} ... a_t
        return np.prod(a[s + 1:t + 1], axis=0)
    X = np.stack([S0.T @ (g[t] * K[t]) for t in range(n)])            # [n, dv]
    Y = Bt[:, None] * V - Bt[:, None] * X
    Am = np.zeros((n, n))
    for t in range(n):
        for s in range(t):
            Am[t, s] = Bt[t] * np.sum(gam(t, s) * K[t] * K[s])
    Wm = np.linalg.solve(np.eye(n) + Am, Y)                           # rows w_t
    Kt = np.stack([gam(n - 1, s) * K[s] for s in range(n)])           # gamma_{n-1,s} o k_s
    S = g[n - 1][:, None] * S0 + Kt.T @ Wm
    P = S0.T @ (g[n - 1][:, None] * U) + Wm.T @ (Kt @ U)
    return S, P


@pytest.mark.parametrize("kind", ["gdn", "kda"])
@pytest.mark.parametrize("case", ["plain", "reset", "tiny"])
def test_chunked_form_matches_recurrence(orc, kind, case):
    rng = np.random.default_rng({"plain": 41, "reset": 42, "tiny": 43}[case])
    dk, dv, r, n = 6, 5, 3, 7
    S0 = rng.standard_normal((dk, dv))
    U = rng.standard_normal((dk, r))
    K = rng.standard_normal((n, dk))
    K /= np.linalg.norm(K, axis=1, keepdims=True)
    V = rng.standard_normal((n, dv))
    A = rng.uniform(0.5, 1.0, (n, dk) if kind == "kda" else n)
    if case == "reset":
        A[3] = 0.0                     # a state reset in mid-window
    elif case == "tiny":
        A[1:] = A[1:] * 1e-30          # products far below the fp32 range (fp64 here)
    Bt = rng.uniform(0.1, 1.0, n)
    S, P = _chunked(kind, S0, U, K, V, A, Bt)
    Sref, Pref = orc.update_window(kind, S0[None], U[None], K[:, None], V[:, None], A[:, None], Bt[:, None])
    np.testing.assert_allclose(S, Sref[0], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(P, Pref[0], rtol=1e-11, atol=1e-12)
