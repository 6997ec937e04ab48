"""Plain fp64 CPU oracle of the SketchSSM windowed decode.

TEST INFRASTRUCTURE.  Only `tests/`, `__graft_entry__.smoke()` and the CPU
baseline leg of `bench.py` import this package.  The product path (the CUDA
library and its binding) never does, and this package never imports it.

Contents:
  sketchssm_oracle.c  per-token recurrences, exact read, windowed update with
                      sketch refresh, sketch read (C, fp64, OpenMP over heads)
  calibration.py      offline basis calibration (numpy fp64)
  this file           ctypes loader and the decode schedules (full-read path
                      and sketch path) in the order the SketchSSM pages give.

Logical layout here: a head's state is S [dk, dv]; many heads are [N, dk, dv];
tokens are time-major [T, N, ...].  The CUDA library stores S transposed
([.., dv, dk]); converting between the two is the caller's business.

Parity status: every function is pinned by the `-m "not gpu"` tests in
tests/test_oracle_*.py, except the choice of calibration objective (a reading).
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, Optional

import numpy as np

from . import calibration  # noqa: F401
from .calibration import calibrate, calibrate_heads, query_pca, query_pca_heads  # noqa: F401

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sketchssm_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

KIND = {"mamba2": 0, "gdn": 1, "kda": 2}

_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (-O2 -ffp-contract=off -fopenmp)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared",
               "-std=c99", "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i = ctypes.c_int
        lib.orc_exact_steps.argtypes = [i, i, i, i, i, P, P, P, P, P, P, P, i]
        lib.orc_read.argtypes = [i, i, i, P, P, P]
        lib.orc_update_window.argtypes = [i, i, i, i, i, i, P, P, P, P, P, P, P, i]
        lib.orc_sketch_read.argtypes = [i, i, i, i, i, i, P, P, P, P, P, P, P, P, P, P]
        lib.orc_round_bf16.argtypes = [ctypes.c_size_t, P]
        lib.orc_set_num_threads.argtypes = [i]
        for f in ("orc_exact_steps", "orc_read", "orc_update_window", "orc_sketch_read",
                  "orc_round_bf16", "orc_num_threads", "orc_set_num_threads"):
            getattr(lib, f).restype = ctypes.c_int
        _lib = lib
    return _lib


def num_threads() -> int:
    return int(_load().orc_num_threads())


def set_num_threads(n: int) -> None:
    """OpenMP threads of the following oracle calls (timing only; results do not depend on it)."""
    _check(_load().orc_set_num_threads(int(n)), "set_num_threads")


def f64(x) -> np.ndarray:
    """A C-contiguous float64 numpy copy of a numpy array or a (CPU/CUDA) torch tensor."""
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what}: invalid arguments (rc={rc})")


def round_bf16(x) -> np.ndarray:
    a = f64(x).copy()
    _check(_load().orc_round_bf16(a.size, _p(a)), "round_bf16")
    return a


def exact_steps(kind: str, S, K, V, A, Bt=None, Q=None, bf16_state: bool = False):
    """Per-step exact recurrence (the full-read path).

    S [N,dk,dv]; K [T,N,dk]; V [T,N,dv]; A [T,N] or [T,N,dk]; Bt [T,N]; Q [T,N,dk].
    Returns (S_T, O [T,N,dv] or None).
    """
    S = f64(S).copy()
    K, V, A, Bt, Q = f64(K), f64(V), f64(A), f64(Bt), f64(Q)
    N, dk, dv = S.shape
    T = K.shape[0]
    O = np.zeros((T, N, dv)) if Q is not None else None
    rc = _load().orc_exact_steps(KIND[kind], N, dk, dv, T, _p(S), _p(K), _p(V), _p(A), _p(Bt),
                                 _p(Q), _p(O), int(bf16_state))
    _check(rc, "exact_steps")
    return S, O


def read(S, Q):
    """o = S^T q per head: S [N,dk,dv], Q [N,dk] -> [N,dv]."""
    S, Q = f64(S), f64(Q)
    N, dk, dv = S.shape
    O = np.zeros((N, dv))
    _check(_load().orc_read(N, dk, dv, _p(S), _p(Q), _p(O)), "read")
    return O


def update_window(kind: str, S, U, K=None, V=None, A=None, Bt=None, bf16_state: bool = False):
    """Windowed update: tokens K[0..n-1] applied in order, then P = S^T U.

    S [N,dk,dv]; U [N,dk,r]; K [n,N,dk] (None or n = 0: sketch refresh only).
    Returns (S_new, P [N,dv,r]).
    """
    S = f64(S).copy()
    U = f64(U)
    N, dk, dv = S.shape
    r = U.shape[2]
    n = 0 if K is None else f64(K).shape[0]
    K, V, A, Bt = (f64(K), f64(V), f64(A), f64(Bt)) if n else (None, None, None, None)
    P = np.zeros((N, dv, r))
    rc = _load().orc_update_window(KIND[kind], N, dk, dv, r, n, _p(S), _p(K), _p(V), _p(A), _p(Bt),
                                   _p(U), _p(P), int(bf16_state))
    _check(rc, "update_window")
    return S, P


def sketch_read(kind: str, P, R, q, K, V, A, Bt=None, return_parts: bool = False):
    """Sketch read of step j = K.shape[0] (tokens 0..j-1 buffered, j-1 the current one).

    P [N,dv,r]; R [N,r,dk]; q [N,dk]; K [j,N,dk]; V [j,N,dv]; A [j,N(,dk)]; Bt [j,N].
    Returns o [N,dv] (and q~ [N,dk], o_buf [N,dv] with return_parts).
    """
    P, R, q = f64(P), f64(R), f64(q)
    N, dv, r = P.shape
    dk = R.shape[2]
    j = 0 if K is None else f64(K).shape[0]
    K, V, A, Bt = (f64(K), f64(V), f64(A), f64(Bt)) if j else (None, None, None, None)
    o = np.zeros((N, dv))
    qt = np.zeros((N, dk)) if return_parts else None
    ob = np.zeros((N, dv)) if return_parts else None
    rc = _load().orc_sketch_read(KIND[kind], N, dk, dv, r, j, _p(P), _p(R), _p(q), _p(K), _p(V),
                                 _p(A), _p(Bt), _p(o), _p(qt), _p(ob))
    _check(rc, "sketch_read")
    return (o, qt, ob) if return_parts else o


def _take(tok: Dict, a: int, b: int):
    return {key: (None if val is None else val[a:b]) for key, val in tok.items()}


def fullread_path(kind: str, S0, tok: Dict, bf16_state: bool = False):
    """The full-read baseline over tokens tok (k, v, alpha, beta, q; time-major, N heads):
    every step applies its token to S and reads S^T q.  Returns (O [T,N,dv], S_T)."""
    S, O = exact_steps(kind, S0, tok["k"], tok["v"], tok["alpha"], tok.get("beta"), tok["q"],
                       bf16_state)
    return O, S


def sketch_path(kind: str, S0, U, R, tok: Dict, W: int, bf16_state: bool = False):
    """The SketchSSM decode schedule over T tokens in windows of W.

    P <- S0^T U; then per window: steps j = 1..n read the sketch (P, R) plus the
    buffered tokens 1..j; after the window's last step the window update applies
    all n tokens exactly to S and refreshes P = S^T U.  U [N,dk,r], R [N,r,dk].
    Returns (O [T,N,dv], S_T, P_T).
    """
    S0 = f64(S0)
    if bf16_state:
        S0 = round_bf16(S0)
    S, P = update_window(kind, S0, U, bf16_state=bf16_state)
    T = tok["k"].shape[0]
    N, dk, dv = S.shape
    O = np.zeros((T, N, dv))
    for t0 in range(0, T, W):
        n = min(W, T - t0)
        win = _take(tok, t0, t0 + n)
        for j in range(1, n + 1):
            O[t0 + j - 1] = sketch_read(kind, P, R, win["q"][j - 1], win["k"][:j], win["v"][:j],
                                        win["alpha"][:j],
                                        None if win.get("beta") is None else win["beta"][:j])
        S, P = update_window(kind, S, U, win["k"], win["v"], win["alpha"], win.get("beta"),
                             bf16_state=bf16_state)
    return O, S, P


def per_head(x, H: int, heads=None):
    """Expand per-head-index arrays [H, ...] to flat heads [N, ...] (flat index n = b*H + h)."""
    x = f64(x)
    if heads is None:
        raise ValueError("heads (flat indices) required")
    idx = np.asarray(heads) % H
    return np.ascontiguousarray(x[idx])
