"""GPU parity at the edges of the recurrences: zero, vanishing and growing decays,
b = 0 and k = 0 tokens, against the fp64 oracle.

The window update folds each head's decays into a running product g_t and
divides by it (update_window.cu).  These cases take that product to zero or out
of the fp32 range, where the kernel must switch that head to the plain per-token
recurrence without changing any result:
  * reset: a zero decay in mid-window (every key channel for KDA), all kinds;
  * tiny: a = 1e-3 on every token, W = 16 and W = 64 (g_t underflows by token 7);
  * channel: KDA with one key channel decaying at 1e-6 (that channel's product
    underflows, the others stay in range);
  * growth: a = 8 on the first 24 tokens of a 40-token window, then 1/8 (g_t
    reaches 2^72, above the range, while the state stays finite over two windows);
  * beta0: b = 0 on every token (GDN, KDA: no delta step, decay only);
  * k0: every third key is zero (nothing added, nothing removed).
Each case checks S and P after one window update, the fused exact read of the
window's last step, and two windows of the whole schedule (sketch path and
full-read path) against the oracle.  No value may be NaN and no bounded wait may
give up.  The largest layout (KDA, r = dk = 128, W = 64) runs the
one-CTA-per-head kernel; the others run the persistent kernel.
Tolerances as everywhere (tests/helpers.py): fp32 state 1e-5 max relative, outputs
1e-4 relative L2.
"""

import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from tests.helpers import (BF16_OUT_TOL, BF16_STATE_TOL, STATE_TOL, TIGHT_OUT, flat_tokens, rel_l2, state_err,
                           to_device, to_gpu_state, to_logical, to_window)

pytestmark = pytest.mark.gpu

KIND_CFG = {"mamba2": 1, "gdn": 2, "kda": 3}


def _edit(kind, case, tok):
    """Apply an edge case to time-major CPU tokens (a copy)."""
    tok = {k: (None if v is None else v.clone()) for k, v in tok.items()}
    W = tok["k"].shape[0]
    if case == "reset":
        tok["alpha"][W // 2] = 0.0
    elif case == "tiny":
        tok["alpha"][:] = 1e-3
    elif case == "channel":
        assert kind == "kda"
        tok["alpha"][..., 5] = 1e-6
    elif case == "growth":  # g_t climbs to 2^72 (past the fold's range), then back to 2^24
        tok["alpha"][:24] = 8.0
        tok["alpha"][24:] = 0.125
    elif case == "beta0":
        tok["beta"][:] = 0.0
    elif case == "k0":
        tok["k"][1::3] = 0
    else:
        raise ValueError(case)
    return tok


CASES = [
    # kind, case, dk, dv, r, W, state dtype, qkv dtype
    ("mamba2", "reset", 128, 64, 8, 16, torch.float32, torch.bfloat16),
    ("gdn", "reset", 128, 128, 8, 16, torch.float32, torch.bfloat16),
    ("kda", "reset", 128, 128, 8, 16, torch.float32, torch.bfloat16),
    ("mamba2", "tiny", 128, 64, 8, 16, torch.float32, torch.bfloat16),
    ("gdn", "tiny", 128, 128, 8, 16, torch.float32, torch.bfloat16),
    ("kda", "tiny", 128, 128, 8, 16, torch.float32, torch.bfloat16),
    ("mamba2", "tiny", 128, 64, 8, 64, torch.float32, torch.bfloat16),
    ("gdn", "tiny", 128, 128, 8, 64, torch.float32, torch.bfloat16),
    ("kda", "tiny", 128, 128, 8, 64, torch.float32, torch.bfloat16),
    ("kda", "channel", 128, 128, 8, 16, torch.float32, torch.bfloat16),
    ("kda", "channel", 64, 64, 4, 8, torch.float32, torch.float32),
    ("mamba2", "growth", 128, 64, 8, 40, torch.float32, torch.bfloat16),
    ("gdn", "growth", 128, 128, 8, 40, torch.float32, torch.bfloat16),
    ("kda", "growth", 128, 128, 8, 40, torch.float32, torch.bfloat16),
    ("gdn", "beta0", 128, 128, 8, 16, torch.float32, torch.bfloat16),
    ("kda", "beta0", 128, 128, 8, 16, torch.float32, torch.bfloat16),
    ("mamba2", "k0", 128, 64, 8, 16, torch.float32, torch.bfloat16),
    ("gdn", "k0", 128, 128, 8, 16, torch.float32, torch.bfloat16),
    ("kda", "k0", 128, 128, 8, 16, torch.float32, torch.bfloat16),
    ("gdn", "reset", 64, 64, 4, 8, torch.bfloat16, torch.float32),
    ("kda", "tiny", 128, 128, 8, 16, torch.bfloat16, torch.bfloat16),
    ("kda", "reset", 128, 128, 128, 64, torch.float32, torch.float32),  # one CTA per head
    ("kda", "tiny", 128, 128, 128, 64, torch.float32, torch.float32),   # one CTA per head
]


def _ids(c):
    return f"{c[0]}-{c[1]}-dk{c[2]}-dv{c[3]}-r{c[4]}-W{c[5]}-S{str(c[6])[6:]}-q{str(c[7])[6:]}"


def _setup(kind, case, dk, dv, r, W, sdt, qdt, B=3, H=5, seed=0):
    import recurrent_state_read_b200 as rs

    cfg = wl.workload(KIND_CFG[kind], B=B, H=H, dk=dk, dv=dv, r=r, W=W,
                      qkv_dtype="f32" if qdt == torch.float32 else "bf16",
                      state_dtype="f32" if sdt == torch.float32 else "bf16", q_rank=min(8, dk))
    d = rs.dims(kind, B, H, dk, dv, r, W, sdt, qdt)
    g = torch.Generator().manual_seed(2000 + seed)
    S0 = torch.randn(B * H, dk, dv, generator=g, dtype=torch.float64).numpy()
    S0 = oracle.round_bf16(S0) if sdt == torch.bfloat16 else S0.astype(np.float32).astype(np.float64)
    U = torch.randn(H, dk, r, generator=g) / dk ** 0.5
    R = torch.randn(H, r, dk, generator=g) / dk ** 0.5
    toks = [_edit(kind, case, wl.token_block(cfg, "decode", w * W, W, with_query=True)) for w in range(2)]
    return cfg, d, S0, U, R, toks


def _tol(sdt):
    return (STATE_TOL, TIGHT_OUT) if sdt == torch.float32 else (BF16_STATE_TOL, BF16_OUT_TOL)


@pytest.mark.parametrize("case", CASES, ids=[_ids(c) for c in CASES])
def test_update_window_edges(case):
    """One window update (S, P) and the fused exact read of its last step."""
    import recurrent_state_read_b200 as rs

    kind, what, dk, dv, r, W, sdt, qdt = case
    cfg, d, S0, U, R, toks = _setup(kind, what, dk, dv, r, W, sdt, qdt)
    B, H = d.B, d.H
    Uh = oracle.per_head(U, H, np.arange(B * H))
    tok = toks[0]
    ft = flat_tokens(tok)
    dev = to_device(tok)
    win = to_window(dev)
    Ug = U.transpose(1, 2).contiguous().cuda()
    s_tol, o_tol = _tol(sdt)
    rs.sketchssm_device_error_count(1)
    bf = sdt == torch.bfloat16
    Sref, Pref = oracle.update_window(kind, S0, Uh, ft["k"], ft["v"], ft["alpha"], ft["beta"], bf16_state=bf)
    _, Oref = oracle.exact_steps(kind, S0, ft["k"], ft["v"], ft["alpha"], ft["beta"], ft["q"])
    for read in (False, True):
        S = to_gpu_state(S0, B, H, sdt)
        P = torch.full((B, H, dv, r), float("nan"), device="cuda")
        o = torch.full((B, H, dv), float("nan"), device="cuda")
        if read:
            rs.sketchssm_update_window_read(d, S, P, Ug, win["k"], win["v"], win["alpha"], win["beta"], W,
                                            dev["q"][W - 1], o)
        else:
            rs.sketchssm_update_window(d, S, P, Ug, win["k"], win["v"], win["alpha"], win["beta"], W)
        torch.cuda.synchronize()
        assert torch.isfinite(S.float()).all() and torch.isfinite(P).all()
        es = state_err(to_logical(S), Sref)
        ep = state_err(P.reshape(B * H, dv, r).double().cpu().numpy(), Pref)
        assert es <= s_tol, (read, es)
        assert ep <= s_tol, (read, ep)
        if read:
            assert torch.isfinite(o).all()
            eo = rel_l2(o.reshape(B * H, dv).double().cpu().numpy(), Oref[W - 1])
            assert eo <= TIGHT_OUT, eo
    assert rs.sketchssm_device_error_count(1) == 0


@pytest.mark.parametrize("case", CASES, ids=[_ids(c) for c in CASES])
def test_schedules_edges(case):
    """Two windows of the sketch path and of the full-read path, every step's output and the final
    state, against the oracle's schedules on the same edited tokens."""
    import recurrent_state_read_b200 as rs
    from recurrent_state_read_b200.decode import WindowBuffer, fullread_window, sketch_window

    kind, what, dk, dv, r, W, sdt, qdt = case
    cfg, d, S0, U, R, toks = _setup(kind, what, dk, dv, r, W, sdt, qdt, seed=1)
    B, H = d.B, d.H
    N = B * H
    heads = np.arange(N)
    bf = sdt == torch.bfloat16
    s_tol, o_tol = _tol(sdt)
    ft = {k: (None if toks[0][k] is None else np.concatenate([flat_tokens(t)[k] for t in toks]))
          for k in toks[0]}
    Uh, Rh = oracle.per_head(U, H, heads), oracle.per_head(R, H, heads)
    Os_ref, Ss_ref, Ps_ref = oracle.sketch_path(kind, S0, Uh, Rh, ft, W, bf16_state=bf)
    Of_ref, Sf_ref = oracle.fullread_path(kind, S0, ft, bf16_state=bf)

    rs.sketchssm_device_error_count(1)
    S = to_gpu_state(S0, B, H, sdt)
    Sf = S.clone()
    P = torch.empty(B, H, dv, r, device="cuda")
    Ug, Rg = U.transpose(1, 2).contiguous().cuda(), R.cuda().contiguous()
    rs.sketchssm_update_window(d, S, P, Ug, None, None, None, None, 0)
    buf = WindowBuffer.empty(d)
    T = 2 * W
    o_s = torch.empty(T, B, H, dv, device="cuda")
    o_f = torch.empty_like(o_s)
    for w, tok in enumerate(toks):
        dtok = to_device(tok)
        buf.fill(dtok)
        sketch_window(d, S, P, Ug, Rg, buf, o_s[w * W:(w + 1) * W])
        fullread_window(d, Sf, dtok, o_f[w * W:(w + 1) * W])
    torch.cuda.synchronize()
    for t in (o_s, o_f, S, Sf, P):
        assert torch.isfinite(t.float()).all()
    e_os = rel_l2(o_s.reshape(T, N, dv).double().cpu().numpy(), Os_ref)
    e_of = rel_l2(o_f.reshape(T, N, dv).double().cpu().numpy(), Of_ref)
    e_ss, e_sf = state_err(to_logical(S), Ss_ref), state_err(to_logical(Sf), Sf_ref)
    e_p = state_err(P.reshape(N, dv, r).double().cpu().numpy(), Ps_ref)
    assert max(e_ss, e_sf, e_p) <= s_tol, (e_ss, e_sf, e_p)
    assert max(e_os, e_of) <= o_tol, (e_os, e_of)
    assert rs.sketchssm_device_error_count(1) == 0


TC_EDGES = ["reset", "tiny", "beta0", "k0"]


@pytest.mark.parametrize("what", TC_EDGES)
def test_update_window_tc_edges(what):
    """sketchssm_update_window_tc (Gated DeltaNet, state increment on the tensor cores) on the same
    edge cases: it multiplies decays and never divides by them, so a zero or vanishing decay needs
    no special path there; results against the oracle's window update."""
    import recurrent_state_read_b200 as rs

    cfg, d, S0, U, R, toks = _setup("gdn", what, 128, 128, 8, 16, torch.float32, torch.bfloat16)
    B, H = d.B, d.H
    Uh = oracle.per_head(U, H, np.arange(B * H))
    ft = flat_tokens(toks[0])
    win = to_window(to_device(toks[0]))
    rs.sketchssm_device_error_count(1)
    S = to_gpu_state(S0, B, H)
    P = torch.full((B, H, 128, 8), float("nan"), device="cuda")
    rs.sketchssm_update_window_tc(d, S, P, U.transpose(1, 2).contiguous().cuda(), win["k"], win["v"],
                                  win["alpha"], win["beta"], 16)
    torch.cuda.synchronize()
    Sref, Pref = oracle.update_window("gdn", S0, Uh, ft["k"], ft["v"], ft["alpha"], ft["beta"])
    assert torch.isfinite(S).all() and torch.isfinite(P).all()
    assert state_err(to_logical(S), Sref) <= STATE_TOL
    assert state_err(P.reshape(B * H, 128, 8).double().cpu().numpy(), Pref) <= STATE_TOL
    assert rs.sketchssm_device_error_count(1) == 0
