"""GPU parity of each kernel alone, through the C ABI, against the fp64 oracle.

Inputs: seeded tokens from the workload generator at reduced batch (B=3, H=5,
a ragged 15 heads), seeded Gaussian states, bases and coefficient maps; both
sides see the same values.  Each case isolates one kernel: the window update
is fed the same window-start state as the oracle, the decode step the same
sketch.  Sizes and edge cases: every kind, dk/dv in {64,128}, fp32/bf16 state
and q/k/v, r from 1 to 32 and r = dk, n_tokens = 0 (sketch refresh only),
partial and full windows, W = 1 and W = 64.
"""

import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from tests.helpers import (BF16_OUT_TOL, BF16_STATE_TOL, STATE_TOL, TIGHT_OUT, flat_tokens, rel_l2,
                           state_err, to_device, to_gpu_state, to_logical, to_window)

pytestmark = pytest.mark.gpu

KIND_CFG = {"mamba2": 1, "gdn": 2, "kda": 3}


def _setup(kind, dk, dv, r, W, sdt, qdt, B=3, H=5, seed=0):
    import recurrent_state_read_b200 as rs

    cfg = wl.workload(KIND_CFG[kind], B=B, H=H, dk=dk, dv=dv, r=r, W=W,
                      qkv_dtype="f32" if qdt == torch.float32 else "bf16",
                      state_dtype="f32" if sdt == torch.float32 else "bf16",
                      q_rank=min(8, dk))
    d = rs.dims(kind, B, H, dk, dv, r, W, sdt, qdt)
    g = torch.Generator().manual_seed(1000 + seed)
    S0 = torch.randn(B * H, dk, dv, generator=g, dtype=torch.float64).numpy()
    S0 = oracle.round_bf16(S0) if sdt == torch.bfloat16 else S0.astype(np.float32).astype(np.float64)
    U = torch.randn(H, dk, r, generator=g) / dk ** 0.5
    R = torch.randn(H, r, dk, generator=g) / dk ** 0.5
    tok = wl.token_block(cfg, "decode", 0, W, with_query=True)
    return cfg, d, S0, U, R, tok


CASES = [
    # kind, dk, dv, r, W, state dtype, qkv dtype
    ("mamba2", 128, 64, 8, 16, torch.float32, torch.bfloat16),
    ("gdn", 128, 128, 8, 16, torch.float32, torch.bfloat16),
    ("kda", 128, 128, 8, 16, torch.float32, torch.bfloat16),
    ("mamba2", 64, 64, 8, 8, torch.float32, torch.float32),
    ("gdn", 64, 128, 4, 5, torch.float32, torch.float32),
    ("kda", 128, 64, 16, 7, torch.float32, torch.bfloat16),
    ("gdn", 128, 128, 32, 32, torch.float32, torch.bfloat16),
    ("gdn", 128, 128, 13, 4, torch.float32, torch.bfloat16),
    ("mamba2", 128, 64, 1, 1, torch.float32, torch.bfloat16),
    ("kda", 64, 64, 64, 3, torch.float32, torch.float32),      # r == dk
    ("gdn", 128, 128, 8, 64, torch.float32, torch.bfloat16),   # longest window
    ("mamba2", 128, 64, 8, 16, torch.bfloat16, torch.bfloat16),
    ("gdn", 128, 128, 8, 16, torch.bfloat16, torch.bfloat16),
    ("kda", 128, 128, 8, 16, torch.bfloat16, torch.bfloat16),
    ("gdn", 64, 64, 4, 8, torch.bfloat16, torch.float32),
    ("kda", 128, 128, 128, 64, torch.float32, torch.float32),  # largest layout: one CTA per head
    ("gdn", 128, 128, 4, 24, torch.float32, torch.float32),    # fp32 tokens: the CUDA-core update
    ("gdn", 128, 128, 16, 13, torch.float32, torch.bfloat16),  # n = 13: the tensor-core update, r = 16
    ("gdn", 128, 128, 8, 32, torch.float32, torch.bfloat16),   # W = 32: n = 16 on the tensor cores
]


def _ids(c):
    return f"{c[0]}-dk{c[1]}-dv{c[2]}-r{c[3]}-W{c[4]}-S{str(c[5])[6:]}-q{str(c[6])[6:]}"


@pytest.mark.parametrize("case", CASES, ids=[_ids(c) for c in CASES])
def test_update_window(case):
    import recurrent_state_read_b200 as rs

    kind, dk, dv, r, W, sdt, qdt = case
    cfg, d, S0, U, R, tok = _setup(kind, dk, dv, r, W, sdt, qdt)
    B, H = d.B, d.H
    heads = np.arange(B * H)
    Uh = oracle.per_head(U, H, heads)
    ft = flat_tokens(tok)
    dev = to_window(to_device(tok))
    for n in sorted({0, 1, max(1, W // 2), W}):
        S = to_gpu_state(S0, B, H, sdt)
        P = torch.full((B, H, dv, r), float("nan"), device="cuda")
        rs.sketchssm_update_window(d, S, P, U.transpose(1, 2).contiguous().cuda(), dev["k"], dev["v"],
                                   dev["alpha"], dev["beta"], n)
        torch.cuda.synchronize()
        sl = slice(0, n)
        Sref, Pref = oracle.update_window(kind, S0, Uh, ft["k"][sl] if n else None, ft["v"][sl],
                                          ft["alpha"][sl], None if ft["beta"] is None else ft["beta"][sl],
                                          bf16_state=sdt == torch.bfloat16)
        tol = STATE_TOL if sdt == torch.float32 else BF16_STATE_TOL
        es = state_err(to_logical(S), Sref)
        ep = state_err(P.reshape(B * H, dv, r).double().cpu().numpy(), Pref)
        assert es <= tol, (n, es)
        assert ep <= tol, (n, ep)
        if n == 0:  # a sketch refresh leaves the state untouched, bit for bit
            assert torch.equal(S, to_gpu_state(S0, B, H, sdt))


@pytest.mark.parametrize("case", CASES, ids=[_ids(c) for c in CASES])
def test_update_window_read(case):
    """The window update with the last step's exact read fused in: S and P as the plain update,
    o = S_n^T q_n against the oracle's exact per-step read (before any storage rounding)."""
    import recurrent_state_read_b200 as rs

    kind, dk, dv, r, W, sdt, qdt = case
    cfg, d, S0, U, R, tok = _setup(kind, dk, dv, r, W, sdt, qdt, seed=5)
    B, H = d.B, d.H
    Uh = oracle.per_head(U, H, np.arange(B * H))
    ft = flat_tokens(tok)
    dev = to_device(tok)
    win = to_window(dev)
    beta = lambda sl: None if ft["beta"] is None else ft["beta"][sl]
    for n in sorted({1, max(1, W // 2), W}):
        S = to_gpu_state(S0, B, H, sdt)
        P = torch.full((B, H, dv, r), float("nan"), device="cuda")
        o = torch.full((B, H, dv), float("nan"), device="cuda")
        rs.sketchssm_update_window_read(d, S, P, U.transpose(1, 2).contiguous().cuda(), win["k"], win["v"],
                                        win["alpha"], win["beta"], n, dev["q"][n - 1], o)
        torch.cuda.synchronize()
        sl = slice(0, n)
        Sref, Pref = oracle.update_window(kind, S0, Uh, ft["k"][sl], ft["v"][sl], ft["alpha"][sl], beta(sl),
                                          bf16_state=sdt == torch.bfloat16)
        _, Oref = oracle.exact_steps(kind, S0, ft["k"][sl], ft["v"][sl], ft["alpha"][sl], beta(sl), ft["q"][sl])
        tol = STATE_TOL if sdt == torch.float32 else BF16_STATE_TOL
        assert state_err(to_logical(S), Sref) <= tol, n
        assert state_err(P.reshape(B * H, dv, r).double().cpu().numpy(), Pref) <= tol, n
        assert rel_l2(o.reshape(B * H, dv).cpu(), Oref[n - 1]) <= TIGHT_OUT, n


@pytest.mark.parametrize("case", CASES, ids=[_ids(c) for c in CASES])
def test_decode_step(case):
    import recurrent_state_read_b200 as rs

    kind, dk, dv, r, W, sdt, qdt = case
    cfg, d, S0, U, R, tok = _setup(kind, dk, dv, r, W, sdt, qdt, seed=1)
    B, H = d.B, d.H
    heads = np.arange(B * H)
    g = torch.Generator().manual_seed(7)
    P = torch.randn(B, H, dv, r, generator=g)
    ft = flat_tokens(tok)
    dev = to_device(tok)
    win = to_window(dev)
    Rh = oracle.per_head(R, H, heads)
    for j in sorted({1, max(1, W // 2), W}):
        o = torch.full((B, H, dv), float("nan"), device="cuda")
        rs.sketchssm_decode_step(d, P.cuda(), R.cuda(), dev["q"][j - 1], win["k"], win["v"], win["alpha"],
                                 win["beta"], j, o)
        torch.cuda.synchronize()
        sl = slice(0, j)
        ref = oracle.sketch_read(kind, P.reshape(B * H, dv, r), Rh, ft["q"][j - 1], ft["k"][sl], ft["v"][sl],
                                 ft["alpha"][sl], None if ft["beta"] is None else ft["beta"][sl])
        err = rel_l2(o.reshape(B * H, dv).cpu(), ref)
        assert err <= TIGHT_OUT, (j, err)


@pytest.mark.parametrize("case", CASES, ids=[_ids(c) for c in CASES])
def test_replay_decode_step(case):
    """ReplaySSM-style step j: the exact read of the window-start state through the buffered tokens
    equals the oracle's per-step exact read S_j^T q_j; the state is not written."""
    import recurrent_state_read_b200 as rs

    kind, dk, dv, r, W, sdt, qdt = case
    cfg, d, S0, U, R, tok = _setup(kind, dk, dv, r, W, sdt, qdt, seed=6)
    B, H = d.B, d.H
    ft = flat_tokens(tok)
    dev = to_device(tok)
    win = to_window(dev)
    S = to_gpu_state(S0, B, H, sdt)
    S_before = S.clone()
    _, Oref = oracle.exact_steps(kind, S0, ft["k"], ft["v"], ft["alpha"], ft["beta"], ft["q"])
    for j in sorted({1, max(1, W // 2), W}):
        o = torch.full((B, H, dv), float("nan"), device="cuda")
        rs.sketchssm_replay_decode_step(d, S, dev["q"][j - 1], win["k"], win["v"], win["alpha"], win["beta"], j, o)
        torch.cuda.synchronize()
        assert rel_l2(o.reshape(B * H, dv).cpu(), Oref[j - 1]) <= TIGHT_OUT, j
    assert torch.equal(S, S_before)


def test_update_window_without_sketch():
    """P = NULL: the state update alone (the ReplaySSM-style window end), same state as with a refresh."""
    import recurrent_state_read_b200 as rs

    kind, dk, dv, r, W = "gdn", 128, 128, 8, 16
    cfg, d, S0, U, R, tok = _setup(kind, dk, dv, r, W, torch.float32, torch.bfloat16, seed=7)
    B, H = d.B, d.H
    ft = flat_tokens(tok)
    win = to_window(to_device(tok))
    S = to_gpu_state(S0, B, H)
    rs.sketchssm_update_window(d, S, None, None, win["k"], win["v"], win["alpha"], win["beta"], W)
    torch.cuda.synchronize()
    Sref, _ = oracle.exact_steps(kind, S0, ft["k"], ft["v"], ft["alpha"], ft["beta"])
    assert state_err(to_logical(S), Sref) <= STATE_TOL


@pytest.mark.parametrize("case", CASES, ids=[_ids(c) for c in CASES])
def test_fullread_decode(case):
    import recurrent_state_read_b200 as rs

    kind, dk, dv, r, W, sdt, qdt = case
    cfg, d, S0, U, R, tok = _setup(kind, dk, dv, r, W, sdt, qdt, seed=2)
    B, H = d.B, d.H
    ft = flat_tokens(tok)
    dev = to_device(tok)
    S = to_gpu_state(S0, B, H, sdt)
    T = min(W, 6)
    outs = torch.full((T, B, H, dv), float("nan"), device="cuda")
    for t in range(T):
        rs.sketchssm_fullread_decode(d, S, dev["q"][t], dev["k"][t], dev["v"][t], dev["alpha"][t],
                                     None if dev["beta"] is None else dev["beta"][t], outs[t])
    torch.cuda.synchronize()
    sl = slice(0, T)
    Sref, Oref = oracle.exact_steps(kind, S0, ft["k"][sl], ft["v"][sl], ft["alpha"][sl],
                                    None if ft["beta"] is None else ft["beta"][sl], ft["q"][sl],
                                    bf16_state=sdt == torch.bfloat16)
    bf = sdt == torch.bfloat16
    assert state_err(to_logical(S), Sref) <= (BF16_STATE_TOL if bf else STATE_TOL)
    assert rel_l2(outs.reshape(T, B * H, dv).cpu(), Oref) <= (BF16_OUT_TOL if bf else TIGHT_OUT)


@pytest.mark.parametrize("kind", ["mamba2", "gdn", "kda"])
def test_update_window_many_heads_per_cta(kind):
    """2100 heads (B=7, H=300): the persistent window update runs several heads per CTA, across
    changes of h (new basis rows) inside one CTA; every head is checked."""
    import recurrent_state_read_b200 as rs

    dk = dv = 64
    r, W = 8, 8
    cfg, d, S0, U, R, tok = _setup(kind, dk, dv, r, W, torch.float32, torch.float32, B=7, H=300, seed=3)
    B, H = d.B, d.H
    Uh = oracle.per_head(U, H, np.arange(B * H))
    ft = flat_tokens(tok)
    dev = to_window(to_device(tok))
    for n in (0, 5, W):
        S = to_gpu_state(S0, B, H)
        P = torch.full((B, H, dv, r), float("nan"), device="cuda")
        rs.sketchssm_update_window(d, S, P, U.transpose(1, 2).contiguous().cuda(), dev["k"], dev["v"],
                                   dev["alpha"], dev["beta"], n)
        torch.cuda.synchronize()
        sl = slice(0, n)
        Sref, Pref = oracle.update_window(kind, S0, Uh, ft["k"][sl] if n else None, ft["v"][sl],
                                          ft["alpha"][sl], None if ft["beta"] is None else ft["beta"][sl])
        assert state_err(to_logical(S), Sref) <= STATE_TOL, n
        assert state_err(P.reshape(B * H, dv, r).double().cpu().numpy(), Pref) <= STATE_TOL, n


TC_PIPE = [("gdn", 16, 8), ("gdn", 16, 13), ("gdn", 8, 4), ("gdn", 16, 16), ("gdn", 4, 1),
           ("kda", 16, 8), ("kda", 16, 3), ("kda", 8, 4)]


@pytest.mark.parametrize("case", TC_PIPE, ids=[f"{c[0]}-W{c[1]}-r{c[2]}" for c in TC_PIPE])
def test_update_window_tc_pipeline(case):
    """sketchssm_update_window_tc, the delta-rule update on the tensor cores (dk = dv = 128, fp32
    state, bf16 keys), over 2100 heads (B=7, H=300): each persistent CTA runs ~15 heads through its
    state stages, reusing stages, token buffers and barrier phases, across changes of h; full and
    partial windows, ranks that need padding.  Every head is checked."""
    import recurrent_state_read_b200 as rs

    kind, W, r = case
    cfg, d, S0, U, R, tok = _setup(kind, 128, 128, r, W, torch.float32, torch.bfloat16, B=7, H=300, seed=11)
    B, H = d.B, d.H
    Uh = oracle.per_head(U, H, np.arange(B * H))
    ft = flat_tokens(tok)
    dev = to_window(to_device(tok))
    Ug = U.transpose(1, 2).contiguous().cuda()
    rs.sketchssm_device_error_count(1)
    for n in sorted({1, min(7, W), W // 2 + 1, W}):
        S = to_gpu_state(S0, B, H)
        P = torch.full((B, H, 128, r), float("nan"), device="cuda")
        rs.sketchssm_update_window_tc(d, S, P, Ug, dev["k"], dev["v"], dev["alpha"], dev["beta"], n)
        torch.cuda.synchronize()
        sl = slice(0, n)
        Sref, Pref = oracle.update_window(kind, S0, Uh, ft["k"][sl], ft["v"][sl], ft["alpha"][sl], ft["beta"][sl])
        es = state_err(to_logical(S), Sref)
        ep = state_err(P.reshape(B * H, 128, r).double().cpu().numpy(), Pref)
        assert es <= STATE_TOL and ep <= STATE_TOL, (n, es, ep)
    assert rs.sketchssm_device_error_count(1) == 0


@pytest.mark.parametrize("kind", ["mamba2", "gdn", "kda"])
def test_decode_step_many_heads_per_warp(kind):
    """6400 heads (B=16, H=400): the pipelined decode step runs several heads per warp, across
    changes of h (new coefficient rows) inside one warp's run; every head is checked."""
    import recurrent_state_read_b200 as rs

    dk = dv = 64
    r, W = 8, 8
    cfg, d, S0, U, R, tok = _setup(kind, dk, dv, r, W, torch.float32, torch.bfloat16, B=16, H=400, seed=4)
    B, H = d.B, d.H
    g = torch.Generator().manual_seed(9)
    P = torch.randn(B, H, dv, r, generator=g)
    ft = flat_tokens(tok)
    dev = to_device(tok)
    win = to_window(dev)
    Rh = oracle.per_head(R, H, np.arange(B * H))
    for j in (1, 5, W):
        o = torch.full((B, H, dv), float("nan"), device="cuda")
        rs.sketchssm_decode_step(d, P.cuda(), R.cuda(), dev["q"][j - 1], win["k"], win["v"], win["alpha"],
                                 win["beta"], j, o)
        torch.cuda.synchronize()
        sl = slice(0, j)
        ref = oracle.sketch_read(kind, P.reshape(B * H, dv, r), Rh, ft["q"][j - 1], ft["k"][sl], ft["v"][sl],
                                 ft["alpha"][sl], None if ft["beta"] is None else ft["beta"][sl])
        assert rel_l2(o.reshape(B * H, dv).cpu(), ref) <= TIGHT_OUT, j


def test_complete_basis_sketch_is_exact_read():
    """r = dk with U = R = I: decode-step outputs equal the full-read outputs (GPU both sides)."""
    import recurrent_state_read_b200 as rs

    kind, dk, dv, W = "gdn", 64, 64, 8
    cfg, d, S0, U, R, tok = _setup(kind, dk, dv, dk, W, torch.float32, torch.float32)
    B, H = d.B, d.H
    eye = torch.eye(dk).expand(H, dk, dk).contiguous().cuda()
    dev = to_device(tok)
    win = to_window(dev)
    S = to_gpu_state(S0, B, H)
    Sf = S.clone()
    P = torch.empty(B, H, dv, dk, device="cuda")
    rs.sketchssm_update_window(d, S, P, eye, None, None, None, None, 0)
    o_s = torch.empty(W, B, H, dv, device="cuda")
    o_f = torch.empty(W, B, H, dv, device="cuda")
    for j in range(1, W + 1):
        rs.sketchssm_decode_step(d, P, eye, dev["q"][j - 1], win["k"], win["v"], win["alpha"], win["beta"],
                                 j, o_s[j - 1])
        rs.sketchssm_fullread_decode(d, Sf, dev["q"][j - 1], dev["k"][j - 1], dev["v"][j - 1],
                                     dev["alpha"][j - 1], dev["beta"][j - 1], o_f[j - 1])
    torch.cuda.synchronize()
    assert rel_l2(o_s.cpu(), o_f.cpu()) <= TIGHT_OUT


def test_invalid_arguments_launch_nothing():
    import recurrent_state_read_b200 as rs

    d = rs.dims("gdn", 2, 2, 128, 128, 8, 16)
    S = torch.zeros(2, 2, 128, 128, device="cuda")
    P = torch.zeros(2, 2, 128, 8, device="cuda")
    U = torch.zeros(2, 128, 8, device="cuda")
    k = torch.zeros(17, 2, 2, 128, dtype=torch.bfloat16, device="cuda")  # room for 17 slots
    a = torch.zeros(17, 2, 2, device="cuda")
    with pytest.raises(rs.SketchSSMError) as e:
        rs.sketchssm_update_window(d, S, P, U, k, k, a, a, 17)  # W = 16
    assert e.value.status == -3
    with pytest.raises(rs.SketchSSMError) as e:
        rs.sketchssm_update_window(d, S, P, U, k, k, a, None, 4)  # GDN needs beta
    assert e.value.status == -1
    bad = rs.dims("gdn", 2, 2, 96, 128, 8, 16)
    with pytest.raises(rs.SketchSSMError) as e:
        rs.sketchssm_update_window(bad, S, P, U, k, k, a, a, 4)
    assert e.value.status == -2
    o = torch.zeros(2, 2, 128, device="cuda")
    with pytest.raises(rs.SketchSSMError) as e:
        rs.sketchssm_decode_step(d, P, U, k[0], k, k, a, a, 0, o)
    assert e.value.status == -3
    torch.cuda.synchronize()
    assert torch.count_nonzero(S) == 0 and torch.count_nonzero(P) == 0


def test_no_bounded_wait_gave_up():
    """Every bounded in-kernel wait in the runs above completed (none gave up)."""
    import recurrent_state_read_b200 as rs

    assert rs.sketchssm_device_error_count() == 0


@pytest.mark.parametrize("kind", ["mamba2", "gdn", "kda"])
def test_ranked_update_and_decode(kind):
    """Rank per head (basis rows past rank[h] zero): the ranked window update and decode step give
    the oracle's results for the zero-padded basis, i.e. each head's rank-r_h sketch read."""
    import recurrent_state_read_b200 as rs

    dk, dv, r, W = 128, 128 if kind != "mamba2" else 64, 16, 16
    cfg, d, S0, U, R, tok = _setup(kind, dk, dv, r, W, torch.float32, torch.bfloat16, B=3, H=7, seed=8)
    B, H = d.B, d.H
    ranks = torch.tensor([0, 3, 8, 9, 16, 5, 12], dtype=torch.int32)
    for h in range(H):
        U[h][:, ranks[h]:] = 0
        R[h][ranks[h]:] = 0
    heads = np.arange(B * H)
    Uh, Rh = oracle.per_head(U, H, heads), oracle.per_head(R, H, heads)
    ft = flat_tokens(tok)
    dev = to_device(tok)
    win = to_window(dev)
    S = to_gpu_state(S0, B, H)
    P = torch.full((B, H, dv, r), float("nan"), device="cuda")
    rk = ranks.cuda()
    Ur = U.transpose(1, 2).contiguous().cuda()
    rs.sketchssm_update_window_ranked(d, S, P, Ur, rk, win["k"], win["v"], win["alpha"], win["beta"], W)
    torch.cuda.synchronize()
    Sref, Pref = oracle.update_window(kind, S0, Uh, ft["k"], ft["v"], ft["alpha"], ft["beta"])
    assert state_err(to_logical(S), Sref) <= STATE_TOL
    assert state_err(P.reshape(B * H, dv, r).double().cpu().numpy(), Pref) <= STATE_TOL
    assert torch.isfinite(P).all()
    for j in (1, 9, W):
        o = torch.full((B, H, dv), float("nan"), device="cuda")
        rs.sketchssm_decode_step_ranked(d, P, R.cuda(), rk, dev["q"][j - 1], win["k"], win["v"], win["alpha"],
                                        win["beta"], j, o)
        torch.cuda.synchronize()
        sl = slice(0, j)
        ref = oracle.sketch_read(kind, Pref, Rh, ft["q"][j - 1], ft["k"][sl], ft["v"][sl], ft["alpha"][sl],
                                 None if ft["beta"] is None else ft["beta"][sl])
        assert rel_l2(o.reshape(B * H, dv).cpu(), ref) <= TIGHT_OUT, j
    assert rs.sketchssm_device_error_count(1) == 0


WY_CASES = [
    ("gdn", 128, 128, 8, 16, torch.bfloat16),
    ("kda", 128, 128, 8, 16, torch.bfloat16),
    ("gdn", 64, 64, 4, 5, torch.float32),       # odd window: padded Gram rows
    ("kda", 64, 128, 16, 7, torch.float32),
    ("gdn", 128, 64, 8, 32, torch.bfloat16),    # the longest window of the WY form
    ("kda", 128, 128, 32, 32, torch.bfloat16),
    ("mamba2", 128, 64, 8, 16, torch.bfloat16),  # no delta chain: the plain step
]


@pytest.mark.parametrize("case", WY_CASES, ids=[f"{c[0]}-dk{c[1]}-dv{c[2]}-r{c[3]}-W{c[4]}" for c in WY_CASES])
def test_decode_step_wy(case):
    """The WY form of the backward pass, steps 1..W in order on one Gram buffer (uninitialised:
    NaN), against the oracle's token-by-token sketch read; the buffer's rows against the Gram
    definition G_ut = sum_i k_t[i] k_u[i] a_{t+1}[i] ... a_u[i]."""
    import recurrent_state_read_b200 as rs

    kind, dk, dv, r, W, qdt = case
    cfg, d, S0, U, R, tok = _setup(kind, dk, dv, r, W, torch.float32, qdt, seed=9)
    B, H = d.B, d.H
    g = torch.Generator().manual_seed(10)
    P = torch.randn(B, H, dv, r, generator=g)
    ft = flat_tokens(tok)
    dev = to_device(tok)
    win = to_window(dev)
    Rh = oracle.per_head(R, H, np.arange(B * H))
    G = rs.wy_gram_buffer(d)
    G.fill_(float("nan"))
    Pd, Rd = P.cuda(), R.cuda()
    for j in range(1, W + 1):
        o = torch.full((B, H, dv), float("nan"), device="cuda")
        rs.sketchssm_decode_step_wy(d, Pd, Rd, dev["q"][j - 1], win["k"], win["v"], win["alpha"], win["beta"], j,
                                    G, o)
        torch.cuda.synchronize()
        sl = slice(0, j)
        ref = oracle.sketch_read(kind, P.reshape(B * H, dv, r), Rh, ft["q"][j - 1], ft["k"][sl], ft["v"][sl],
                                 ft["alpha"][sl], None if ft["beta"] is None else ft["beta"][sl])
        assert rel_l2(o.reshape(B * H, dv).cpu(), ref) <= TIGHT_OUT, j
    if kind == "mamba2":
        return
    Gg = G.reshape(B * H, W, -1).double().cpu().numpy()
    k, a = ft["k"], ft["alpha"]
    for n in range(B * H):
        for u in range(1, W):
            for t in range(u):
                dec = np.prod(a[t + 1:u + 1, n], axis=0) if kind == "kda" else np.prod(a[t + 1:u + 1, n])
                ref_g = np.sum(k[t, n] * k[u, n] * dec)
                assert abs(Gg[n, u, t] - ref_g) <= 1e-4 * max(1.0, abs(ref_g)), (n, u, t)


def test_bounded_wait_gives_up_and_the_context_survives():
    """Failure detection without a GPU fault: a bounded wait that nothing satisfies gives up, is
    counted, and the next real kernel runs normally."""
    import recurrent_state_read_b200 as rs

    torch.cuda.synchronize()
    rs.sketchssm_device_error_count(1)  # start from zero
    rs.sketchssm_selftest_wait_giveup(1000)
    assert rs.sketchssm_device_error_count(1) == 1
    assert rs.sketchssm_device_error_count(0) == 0  # reset took
    kind, dk, dv, r, W, sdt, qdt = CASES[1]
    cfg, d, S0, U, R, tok = _setup(kind, dk, dv, r, W, sdt, qdt, seed=12)
    dev = to_device(tok)
    win = to_window(dev)
    P = torch.randn(d.B, d.H, dv, r, device="cuda")
    o = torch.full((d.B, d.H, dv), float("nan"), device="cuda")
    rs.sketchssm_decode_step(d, P, R.cuda(), dev["q"][3], win["k"], win["v"], win["alpha"], win["beta"], 4, o)
    torch.cuda.synchronize()
    assert torch.isfinite(o).all()
    assert rs.sketchssm_device_error_count(1) == 0


def test_update_window_tc_not_applicable():
    """Sizes outside the tensor-core update's envelope are rejected before any launch."""
    import recurrent_state_read_b200 as rs

    cfg, d, S0, U, R, tok = _setup("kda", 128, 128, 16, 16, torch.float32, torch.bfloat16)  # KDA: r <= 8
    dev = to_window(to_device(tok))
    S = to_gpu_state(S0, d.B, d.H)
    P = torch.zeros(d.B, d.H, 128, 16, device="cuda")
    with pytest.raises(rs.SketchSSMError):
        rs.sketchssm_update_window_tc(d, S, P, U.transpose(1, 2).contiguous().cuda(), dev["k"], dev["v"],
                                      dev["alpha"], dev["beta"], 16)
    torch.cuda.synchronize()
    assert torch.equal(S, to_gpu_state(S0, d.B, d.H))  # nothing was launched
