"""Python binding of the SketchSSM windowed-decode library (libsketchssm.so, sm_100a).

Argument marshalling only: every function below checks that it was handed
device tensors of the right dtype and size, then calls the C entry point of
the same name (include/sketchssm.h) with raw pointers and the current torch
CUDA stream.  All arithmetic runs in the library's CUDA kernels; there is no
CPU fallback, and calling any entry point without the built library raises.

Layouts (N = B*H heads, see include/sketchssm.h):
    S [B,H,dv,dk]  (state, transposed storage)   P [B,H,dv,r] fp32
    U [H,r,dk] fp32 (basis rows, U_rows[h,m,i] = U[i,m])      R [H,r,dk] fp32
    window buffer (head-major): k [B,H,W,dk], v [B,H,W,dv], alpha [B,H,W] (KDA [B,H,W,dk]), beta [B,H,W]
    one token (full-read step): q, k [B,H,dk], v [B,H,dv], alpha [B,H] (KDA [B,H,dk]), beta [B,H]
    q [B,H,dk], o [B,H,dv] fp32
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsketchssm.so")

KIND = {"mamba2": 0, "gdn": 1, "kda": 2}
DTYPE = {torch.float32: 0, torch.bfloat16: 1}
EXPORTS = (
    "sketchssm_status_string",
    "sketchssm_version",
    "sketchssm_update_window",
    "sketchssm_update_window_read",
    "sketchssm_update_window_tc",
    "sketchssm_decode_step",
    "sketchssm_decode_step_seq",
    "sketchssm_update_window_seqs",
    "sketchssm_fullread_decode",
    "sketchssm_replay_decode_step",
    "sketchssm_calibrate_workspace_bytes",
    "sketchssm_calibrate_basis",
    "sketchssm_calibrate_basis_noalloc",
    "sketchssm_calibrate_basis_ranked",
    "sketchssm_calibrate_query_pca",
    "sketchssm_update_window_ranked",
    "sketchssm_decode_step_ranked",
    "sketchssm_decode_step_wy",
    "sketchssm_device_error_count",
    "sketchssm_selftest_wait_giveup",
)


class sketchssm_dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("kind", "B", "H", "dk", "dv", "r", "W", "state_dtype", "qkv_dtype")]

    def __repr__(self):
        return "sketchssm_dims(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


class SketchSSMError(RuntimeError):
    def __init__(self, fn: str, status: int, text: str):
        super().__init__(f"{fn} failed: status {status} ({text})")
        self.status = status


_lib = None


def library() -> ctypes.CDLL:
    """The loaded CUDA library.  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m recurrent_state_read_b200.build` (nvcc, sm_100a)")
        lib = ctypes.CDLL(LIB_PATH)
        P = ctypes.c_void_p
        D = ctypes.POINTER(sketchssm_dims)
        i = ctypes.c_int
        lib.sketchssm_status_string.argtypes = [i]
        lib.sketchssm_status_string.restype = ctypes.c_char_p
        lib.sketchssm_version.argtypes = []
        lib.sketchssm_version.restype = i
        lib.sketchssm_update_window.argtypes = [D, P, P, P, P, P, P, P, i, P]
        lib.sketchssm_update_window_read.argtypes = [D, P, P, P, P, P, P, P, i, P, P, P]
        lib.sketchssm_update_window_tc.argtypes = [D, P, P, P, P, P, P, P, i, P]
        lib.sketchssm_decode_step.argtypes = [D, P, P, P, P, P, P, P, i, P, P]
        lib.sketchssm_decode_step_seq.argtypes = [D, P, P, P, P, P, P, P, P, i, P, P]
        lib.sketchssm_update_window_seqs.argtypes = [D, P, P, P, P, P, P, P, i, P, i, P, P, i, P]
        lib.sketchssm_fullread_decode.argtypes = [D, P, P, P, P, P, P, P, P]
        lib.sketchssm_replay_decode_step.argtypes = [D, P, P, P, P, P, P, i, P, P]
        lib.sketchssm_calibrate_workspace_bytes.argtypes = [D, i, i]
        lib.sketchssm_calibrate_workspace_bytes.restype = ctypes.c_size_t
        lib.sketchssm_calibrate_basis.argtypes = [D, P, i, P, i, ctypes.c_double, P, P, P,
                                                  ctypes.c_size_t, P]
        lib.sketchssm_calibrate_basis_noalloc.argtypes = [D, P, i, P, i, ctypes.c_double, P, P, P]
        lib.sketchssm_calibrate_basis_ranked.argtypes = [D, P, i, P, i, ctypes.c_double, i, P, P, P, P, P,
                                                         ctypes.c_size_t, P]
        lib.sketchssm_calibrate_query_pca.argtypes = [D, P, i, P, P, P, ctypes.c_size_t, P]
        lib.sketchssm_update_window_ranked.argtypes = [D, P, P, P, P, P, P, P, P, i, P]
        lib.sketchssm_decode_step_ranked.argtypes = [D, P, P, P, P, P, P, P, P, i, P, P]
        lib.sketchssm_decode_step_wy.argtypes = [D, P, P, P, P, P, P, P, i, P, P, P]
        lib.sketchssm_device_error_count.argtypes = [i]
        lib.sketchssm_selftest_wait_giveup.argtypes = [ctypes.c_uint, P]
        lib.sketchssm_selftest_wait_giveup.restype = i
        lib.sketchssm_device_error_count.restype = i
        for f in ("sketchssm_update_window", "sketchssm_update_window_read", "sketchssm_update_window_tc",
                  "sketchssm_decode_step",
                  "sketchssm_replay_decode_step", "sketchssm_decode_step_seq", "sketchssm_update_window_seqs",
                  "sketchssm_calibrate_basis_ranked", "sketchssm_update_window_ranked",
                  "sketchssm_decode_step_ranked", "sketchssm_decode_step_wy", "sketchssm_fullread_decode",
                  "sketchssm_calibrate_basis", "sketchssm_calibrate_basis_noalloc",
                  "sketchssm_calibrate_query_pca"):
            getattr(lib, f).restype = i
        _lib = lib
    return _lib


def dims(kind, B, H, dk, dv, r, W, state_dtype=torch.float32, qkv_dtype=torch.bfloat16) -> sketchssm_dims:
    k = KIND[kind] if isinstance(kind, str) else int(kind)
    return sketchssm_dims(k, B, H, dk, dv, r, W, DTYPE[state_dtype], DTYPE[qkv_dtype])


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: Optional[torch.Tensor], name: str, numel: int = None, dtype=None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name}: expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if numel is not None and t.numel() < numel:
        raise ValueError(f"{name}: needs at least {numel} elements, has {t.numel()}")
    return ctypes.c_void_p(t.data_ptr())


def _dt(code: int):
    return torch.float32 if code == 0 else torch.bfloat16


def _check(fn: str, rc: int):
    if rc != 0:
        raise SketchSSMError(fn, rc, library().sketchssm_status_string(rc).decode())


def _token_ptrs(d: sketchssm_dims, slots: int, k, v, alpha, beta):
    """Pointers of `slots` tokens per head: slots = W for a head-major window buffer
    [B,H,W,..], slots = 1 for the single token plane [B,H,..] of a full-read step."""
    NH = d.B * d.H
    qt = _dt(d.qkv_dtype)
    na = d.dk if d.kind == KIND["kda"] else 1
    return (_ptr(k, "k", slots * NH * d.dk, qt), _ptr(v, "v", slots * NH * d.dv, qt),
            _ptr(alpha, "alpha", slots * NH * na, torch.float32),
            _ptr(beta, "beta", slots * NH, torch.float32))


def sketchssm_update_window(d: sketchssm_dims, S, P, U, k, v, alpha, beta, n_tokens: int, stream=None):
    """Apply window-buffer tokens 0..n_tokens-1 to S exactly and refresh P = S^T U (one kernel).
    P = None (and U = None): no sketch refresh."""
    NH = d.B * d.H
    args = (_ptr(S, "S", NH * d.dv * d.dk, _dt(d.state_dtype)),
            None if P is None else _ptr(P, "P", NH * d.dv * d.r, torch.float32),
            None if U is None else _ptr(U, "U", d.H * d.dk * d.r, torch.float32))
    toks = _token_ptrs(d, d.W, k, v, alpha, beta) if n_tokens > 0 else (None,) * 4
    _check("sketchssm_update_window",
           library().sketchssm_update_window(ctypes.byref(d), *args, *toks, int(n_tokens),
                                             ctypes.c_void_p(_stream(stream))))


def sketchssm_update_window_tc(d: sketchssm_dims, S, P, U, k, v, alpha, beta, n_tokens: int, stream=None):
    """sketchssm_update_window for Gated DeltaNet with the rank-n state increment on the tensor cores
    (dk = dv = 128, fp32 state, bf16 q/k/v, 1 <= n_tokens <= 16, r <= 16)."""
    NH = d.B * d.H
    args = (_ptr(S, "S", NH * d.dv * d.dk, _dt(d.state_dtype)),
            None if P is None else _ptr(P, "P", NH * d.dv * d.r, torch.float32),
            None if U is None else _ptr(U, "U", d.H * d.dk * d.r, torch.float32))
    toks = _token_ptrs(d, d.W, k, v, alpha, beta)
    _check("sketchssm_update_window_tc",
           library().sketchssm_update_window_tc(ctypes.byref(d), *args, *toks, int(n_tokens),
                                                ctypes.c_void_p(_stream(stream))))


def sketchssm_update_window_read(d: sketchssm_dims, S, P, U, k, v, alpha, beta, n_tokens: int, q, o,
                                 stream=None):
    """sketchssm_update_window plus the exact read o = S^T q of the step whose token is the last
    one applied (q [B,H,dk] qkv dtype, o [B,H,dv] fp32), in the same kernel."""
    NH = d.B * d.H
    args = (_ptr(S, "S", NH * d.dv * d.dk, _dt(d.state_dtype)), _ptr(P, "P", NH * d.dv * d.r, torch.float32),
            _ptr(U, "U", d.H * d.dk * d.r, torch.float32))
    toks = _token_ptrs(d, d.W, k, v, alpha, beta) if n_tokens > 0 else (None,) * 4
    _check("sketchssm_update_window_read",
           library().sketchssm_update_window_read(ctypes.byref(d), *args, *toks, int(n_tokens),
                                                  _ptr(q, "q", NH * d.dk, _dt(d.qkv_dtype)),
                                                  _ptr(o, "o", NH * d.dv, torch.float32),
                                                  ctypes.c_void_p(_stream(stream))))


def sketchssm_decode_step(d: sketchssm_dims, P, R, q, k, v, alpha, beta, j: int, o, stream=None):
    """Decode step j of the window from the sketch P and window-buffer tokens 0..j-1 into o."""
    NH = d.B * d.H
    toks = _token_ptrs(d, d.W, k, v, alpha, beta)
    _check("sketchssm_decode_step", library().sketchssm_decode_step(
        ctypes.byref(d), _ptr(P, "P", NH * d.dv * d.r, torch.float32),
        _ptr(R, "R", d.H * d.r * d.dk, torch.float32), _ptr(q, "q", NH * d.dk, _dt(d.qkv_dtype)),
        *toks, int(j), _ptr(o, "o", NH * d.dv, torch.float32), ctypes.c_void_p(_stream(stream))))


def _i32(t, name, numel):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != torch.int32 or not t.is_contiguous():
        raise TypeError(f"{name}: expected a contiguous int32 CUDA tensor")
    if t.numel() < numel:
        raise ValueError(f"{name}: needs at least {numel} elements, has {t.numel()}")
    return ctypes.c_void_p(t.data_ptr())


def sketchssm_decode_step_seq(d: sketchssm_dims, P, R, q, k, v, alpha, beta, j_seq, o, sm_share: int = 0,
                              stream=None):
    """Decode step with a step index per sequence (j_seq: int32 [B] on the device, 1..W, or 0 for no
    step); sm_share > 0 caps the CTAs per SM so that a concurrent kernel fits."""
    NH = d.B * d.H
    toks = _token_ptrs(d, d.W, k, v, alpha, beta)
    _check("sketchssm_decode_step_seq", library().sketchssm_decode_step_seq(
        ctypes.byref(d), _ptr(P, "P", NH * d.dv * d.r, torch.float32),
        _ptr(R, "R", d.H * d.r * d.dk, torch.float32), _ptr(q, "q", NH * d.dk, _dt(d.qkv_dtype)),
        *toks, _i32(j_seq, "j_seq", d.B), int(sm_share), _ptr(o, "o", NH * d.dv, torch.float32),
        ctypes.c_void_p(_stream(stream))))


def sketchssm_update_window_seqs(d: sketchssm_dims, S, P, U, k, v, alpha, beta, n_tokens: int, seqs,
                                 q=None, o=None, sm_share: int = 0, stream=None):
    """The window update (and with q, o the exact read) for the sequences listed in seqs (int32 on the
    device) only."""
    NH = d.B * d.H
    n_seqs = int(seqs.numel())
    toks = _token_ptrs(d, d.W, k, v, alpha, beta) if n_tokens > 0 else (None,) * 4
    _check("sketchssm_update_window_seqs", library().sketchssm_update_window_seqs(
        ctypes.byref(d), _ptr(S, "S", NH * d.dv * d.dk, _dt(d.state_dtype)),
        None if P is None else _ptr(P, "P", NH * d.dv * d.r, torch.float32),
        None if U is None else _ptr(U, "U", d.H * d.dk * d.r, torch.float32), *toks, int(n_tokens),
        _i32(seqs, "seqs", n_seqs), n_seqs, None if q is None else _ptr(q, "q", NH * d.dk, _dt(d.qkv_dtype)),
        None if o is None else _ptr(o, "o", NH * d.dv, torch.float32), int(sm_share),
        ctypes.c_void_p(_stream(stream))))


def sketchssm_replay_decode_step(d: sketchssm_dims, S, q, k, v, alpha, beta, j: int, o, stream=None):
    """ReplaySSM-style decode step j: the exact read o = S^T q~ + o_buf of the window-start state S
    (read, not written) and window-buffer tokens 0..j-1."""
    NH = d.B * d.H
    toks = _token_ptrs(d, d.W, k, v, alpha, beta)
    _check("sketchssm_replay_decode_step", library().sketchssm_replay_decode_step(
        ctypes.byref(d), _ptr(S, "S", NH * d.dv * d.dk, _dt(d.state_dtype)),
        _ptr(q, "q", NH * d.dk, _dt(d.qkv_dtype)), *toks, int(j), _ptr(o, "o", NH * d.dv, torch.float32),
        ctypes.c_void_p(_stream(stream))))


def sketchssm_fullread_decode(d: sketchssm_dims, S, q, k, v, alpha, beta, o, stream=None):
    """Baseline decode step: read, update and write the full state; o = S^T q."""
    NH = d.B * d.H
    toks = _token_ptrs(d, 1, k, v, alpha, beta)
    _check("sketchssm_fullread_decode", library().sketchssm_fullread_decode(
        ctypes.byref(d), _ptr(S, "S", NH * d.dv * d.dk, _dt(d.state_dtype)),
        _ptr(q, "q", NH * d.dk, _dt(d.qkv_dtype)), *toks, _ptr(o, "o", NH * d.dv, torch.float32),
        ctypes.c_void_p(_stream(stream))))


def sketchssm_calibrate_workspace_bytes(d: sketchssm_dims, Nq: int, Ns: int) -> int:
    return int(library().sketchssm_calibrate_workspace_bytes(ctypes.byref(d), int(Nq), int(Ns)))


def sketchssm_calibrate_basis(d: sketchssm_dims, q_cal, S_cal, U, R, workspace=None, ridge: float = 1e-8,
                              stream=None):
    """Offline basis: q_cal [H,Nq,dk] fp32, S_cal [Ns,H,dv,dk] -> U [H,r,dk] (rows), R [H,r,dk].

    `workspace` is a uint8 CUDA tensor of at least sketchssm_calibrate_workspace_bytes bytes; when
    None, one is allocated here through torch (the library itself never allocates).
    """
    Nq = q_cal.shape[1]
    Ns = S_cal.shape[0]
    need = sketchssm_calibrate_workspace_bytes(d, Nq, Ns)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q_cal.device)
    _check("sketchssm_calibrate_basis", library().sketchssm_calibrate_basis(
        ctypes.byref(d), _ptr(q_cal, "q_cal", d.H * Nq * d.dk, torch.float32), int(Nq),
        _ptr(S_cal, "S_cal", Ns * d.H * d.dv * d.dk, _dt(d.state_dtype)), int(Ns), float(ridge),
        _ptr(U, "U", d.H * d.dk * d.r, torch.float32), _ptr(R, "R", d.H * d.r * d.dk, torch.float32),
        _ptr(workspace, "workspace"), ctypes.c_size_t(workspace.numel() * workspace.element_size()),
        ctypes.c_void_p(_stream(stream))))


def sketchssm_calibrate_query_pca(d: sketchssm_dims, q_cal, U, R, workspace=None, stream=None):
    """Query-PCA basis (no state weighting): q_cal [H,Nq,dk] fp32 -> U, R [H,r,dk] with U = R the
    top-r principal directions of each head's calibration queries.  Workspace as
    sketchssm_calibrate_basis with Ns = 1."""
    Nq = q_cal.shape[1]
    need = sketchssm_calibrate_workspace_bytes(d, Nq, 1)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q_cal.device)
    _check("sketchssm_calibrate_query_pca", library().sketchssm_calibrate_query_pca(
        ctypes.byref(d), _ptr(q_cal, "q_cal", d.H * Nq * d.dk, torch.float32), int(Nq),
        _ptr(U, "U", d.H * d.dk * d.r, torch.float32), _ptr(R, "R", d.H * d.r * d.dk, torch.float32),
        _ptr(workspace, "workspace"), ctypes.c_size_t(workspace.numel() * workspace.element_size()),
        ctypes.c_void_p(_stream(stream))))


def sketchssm_calibrate_basis_ranked(d: sketchssm_dims, q_cal, S_cal, r_avg: int, U, R, rank, lam,
                                     workspace=None, ridge: float = 1e-8, stream=None):
    """Offline basis with a rank per head under the average rank r_avg (d.r is the largest rank):
    U, R [H,r,dk] with rows past rank[h] zero, rank int32 [H], lam float64 [H,r] (each head's r
    largest eigenvalues, descending).  Workspace as sketchssm_calibrate_basis."""
    Nq = q_cal.shape[1]
    Ns = S_cal.shape[0]
    need = sketchssm_calibrate_workspace_bytes(d, Nq, Ns)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q_cal.device)
    _check("sketchssm_calibrate_basis_ranked", library().sketchssm_calibrate_basis_ranked(
        ctypes.byref(d), _ptr(q_cal, "q_cal", d.H * Nq * d.dk, torch.float32), int(Nq),
        _ptr(S_cal, "S_cal", Ns * d.H * d.dv * d.dk, _dt(d.state_dtype)), int(Ns), float(ridge), int(r_avg),
        _ptr(U, "U", d.H * d.dk * d.r, torch.float32), _ptr(R, "R", d.H * d.r * d.dk, torch.float32),
        _i32(rank, "rank", d.H), _ptr(lam, "lam", d.H * d.r, torch.float64),
        _ptr(workspace, "workspace"), ctypes.c_size_t(workspace.numel() * workspace.element_size()),
        ctypes.c_void_p(_stream(stream))))


def sketchssm_update_window_ranked(d: sketchssm_dims, S, P, U, rank, k, v, alpha, beta, n_tokens: int,
                                   stream=None):
    """sketchssm_update_window for a basis with a rank per head (rank int32 [H] on the device)."""
    NH = d.B * d.H
    toks = _token_ptrs(d, d.W, k, v, alpha, beta) if n_tokens > 0 else (None,) * 4
    _check("sketchssm_update_window_ranked", library().sketchssm_update_window_ranked(
        ctypes.byref(d), _ptr(S, "S", NH * d.dv * d.dk, _dt(d.state_dtype)),
        _ptr(P, "P", NH * d.dv * d.r, torch.float32), _ptr(U, "U", d.H * d.dk * d.r, torch.float32),
        _i32(rank, "rank", d.H), *toks, int(n_tokens), ctypes.c_void_p(_stream(stream))))


def sketchssm_decode_step_ranked(d: sketchssm_dims, P, R, rank, q, k, v, alpha, beta, j: int, o, stream=None):
    """sketchssm_decode_step for a basis with a rank per head (rank int32 [H] on the device)."""
    NH = d.B * d.H
    toks = _token_ptrs(d, d.W, k, v, alpha, beta)
    _check("sketchssm_decode_step_ranked", library().sketchssm_decode_step_ranked(
        ctypes.byref(d), _ptr(P, "P", NH * d.dv * d.r, torch.float32),
        _ptr(R, "R", d.H * d.r * d.dk, torch.float32), _i32(rank, "rank", d.H),
        _ptr(q, "q", NH * d.dk, _dt(d.qkv_dtype)), *toks, int(j), _ptr(o, "o", NH * d.dv, torch.float32),
        ctypes.c_void_p(_stream(stream))))


def sketchssm_selftest_wait_giveup(tries: int = 1000, stream=None):
    """Make the bounded-wait failure path run once (a wait that nothing satisfies): it is
    counted in sketchssm_device_error_count and the context stays usable."""
    _check("sketchssm_selftest_wait_giveup",
           library().sketchssm_selftest_wait_giveup(int(tries), ctypes.c_void_p(_stream(stream))))


def wy_gram_buffer(d: sketchssm_dims, device="cuda"):
    """The per-head Gram buffer of sketchssm_decode_step_wy: [B, H, W, W rounded up to 4] fp32."""
    return torch.empty(d.B, d.H, d.W, (d.W + 3) // 4 * 4, dtype=torch.float32, device=device)


def sketchssm_decode_step_wy(d: sketchssm_dims, P, R, q, k, v, alpha, beta, j: int, G, o, stream=None):
    """Decode step j with the WY form of the backward pass; G from wy_gram_buffer, steps in order."""
    NH = d.B * d.H
    toks = _token_ptrs(d, d.W, k, v, alpha, beta)
    _check("sketchssm_decode_step_wy", library().sketchssm_decode_step_wy(
        ctypes.byref(d), _ptr(P, "P", NH * d.dv * d.r, torch.float32),
        _ptr(R, "R", d.H * d.r * d.dk, torch.float32), _ptr(q, "q", NH * d.dk, _dt(d.qkv_dtype)),
        *toks, int(j), _ptr(G, "G", NH * d.W * ((d.W + 3) // 4 * 4), torch.float32),
        _ptr(o, "o", NH * d.dv, torch.float32), ctypes.c_void_p(_stream(stream))))


def sketchssm_calibrate_basis_noalloc(d: sketchssm_dims, q_cal, S_cal, U, R, ridge: float = 1e-8, stream=None):
    """sketchssm_calibrate_basis for callers that cannot allocate device memory: the library
    works in a fixed 3 MiB scratch array of its own (see include/sketchssm.h); neither the
    library nor this wrapper allocates.  Calls that overlap on the GPU race on that scratch."""
    Nq = q_cal.shape[1]
    Ns = S_cal.shape[0]
    _check("sketchssm_calibrate_basis_noalloc", library().sketchssm_calibrate_basis_noalloc(
        ctypes.byref(d), _ptr(q_cal, "q_cal", d.H * Nq * d.dk, torch.float32), int(Nq),
        _ptr(S_cal, "S_cal", Ns * d.H * d.dv * d.dk, _dt(d.state_dtype)), int(Ns), float(ridge),
        _ptr(U, "U", d.H * d.dk * d.r, torch.float32), _ptr(R, "R", d.H * d.r * d.dk, torch.float32),
        ctypes.c_void_p(_stream(stream))))


def sketchssm_device_error_count(reset: bool = False) -> int:
    """Bounded in-kernel waits that gave up on the current device (0 in normal operation)."""
    n = int(library().sketchssm_device_error_count(int(reset)))
    if n < 0:
        raise SketchSSMError("sketchssm_device_error_count", n, library().sketchssm_status_string(n).decode())
    return n
