"""GPU parity of the whole decode schedules on the five workloads.

Each test runs the sketch path (decode steps from the sketch + one fused
window update per window) and the full-read baseline through the C ABI and
compares them with the fp64 oracle:
  * the tiny Mamba-2 case over all heads and all 64 steps, with the basis
    calibrated by the oracle from the full calibration recipe;
  * Mamba-2 at serving batch, Gated DeltaNet, KDA (r = 4, 8, 16) and sweep
    points of the GDN shape at full batch and head count -- the launch
    configuration the bench times -- with the oracle run on a seeded sample of
    heads (heads are independent, so a sampled head's result does not depend on
    the others).  There the GPU builds its start state with its own prefill
    (window updates over the prefill tokens) and the oracle with its own, so the
    comparison covers the prefill as well; the basis comes from the oracle's
    calibration on a reduced calibration set.
The contract tolerances (state 1e-5 max relative, sketch outputs 2e-3 relative
L2) and the tighter fp32-derived ones are in tests/helpers.py.  The sketch's
approximation error against the exact read is printed, never gated.
"""

import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from tests.helpers import (BF16_OUT_TOL, BF16_STATE_TOL, OUT_TOL, STATE_TOL, TIGHT_OUT, flat_tokens,
                           rel_l2, state_err, to_device, to_gpu_state, to_logical)

pytestmark = pytest.mark.gpu


def _dims(cfg):
    import recurrent_state_read_b200 as rs

    return rs.dims(cfg.kind, cfg.B, cfg.H, cfg.dk, cfg.dv, cfg.r, cfg.W, cfg.torch_state_dtype,
                   cfg.torch_qkv_dtype)


def _oracle_calibration(cfg, n_seq, n_tokens, n_q, device):
    """U, R [H,...] fp64 from the oracle on n_seq calibration sequences of n_tokens tokens."""
    tok = wl.token_block(cfg, "cal", 0, n_tokens, device=device, B=n_seq)
    ft = flat_tokens(tok)
    S = np.zeros((n_seq * cfg.H, cfg.dk, cfg.dv))
    S, _ = oracle.exact_steps(cfg.kind, S, ft["k"], ft["v"], ft["alpha"], ft["beta"])
    S_cal = S.reshape(n_seq, cfg.H, cfg.dk, cfg.dv)
    q_cal = wl.calibration_queries(cfg, device="cpu", n=n_q).double().numpy()
    return oracle.calibrate_heads(S_cal, q_cal, cfg.r)


def _run_gpu(cfg, S0_gpu, U, R, source, n_steps):
    """Sketch path and full-read path on the GPU.  Returns outputs, final states, final sketch."""
    import recurrent_state_read_b200 as rs
    from recurrent_state_read_b200.decode import WindowBuffer, fullread_window, sketch_window

    d = _dims(cfg)
    S = S0_gpu.clone()
    Sf = S0_gpu.clone()
    P = torch.empty(cfg.B, cfg.H, cfg.dv, cfg.r, device="cuda")
    Ug, Rg = U.float().transpose(1, 2).contiguous().cuda(), R.float().cuda().contiguous()  # U as rows
    rs.sketchssm_update_window(d, S, P, Ug, None, None, None, None, 0)
    buf = WindowBuffer.empty(d)
    o_s = torch.empty(n_steps, cfg.B, cfg.H, cfg.dv, device="cuda")
    o_f = torch.empty_like(o_s)
    for t0 in range(0, n_steps, cfg.W):
        n = min(cfg.W, n_steps - t0)
        tok = {k: (None if v is None else v.contiguous()) for k, v in source(t0, n).items()}
        buf.fill(tok, n)
        sketch_window(d, S, P, Ug, Rg, buf, o_s[t0:t0 + n], n)
        fullread_window(d, Sf, tok, o_f[t0:t0 + n], n)
    torch.cuda.synchronize()
    return o_s, o_f, S, Sf, P


def _check(cfg, heads, O_s, O_f, S, Sf, P, ref_s, ref_f, label):
    Os_ref, Ss_ref, Ps_ref = ref_s
    Of_ref, Sf_ref = ref_f
    hs = torch.as_tensor(heads, device="cuda")
    T = O_s.shape[0]
    Os = O_s.reshape(T, -1, cfg.dv)[:, hs].double().cpu().numpy()
    Of = O_f.reshape(T, -1, cfg.dv)[:, hs].double().cpu().numpy()
    bf = cfg.state_dtype == "bf16"
    e_os, e_of = rel_l2(Os, Os_ref), rel_l2(Of, Of_ref)
    e_ss, e_sf = state_err(to_logical(S, heads), Ss_ref), state_err(to_logical(Sf, heads), Sf_ref)
    Pl = P.reshape(-1, cfg.dv, cfg.r)[hs].double().cpu().numpy()
    e_p = state_err(Pl, Ps_ref)
    approx = rel_l2(Os_ref, Of_ref)
    print(f"{label}: out sketch {e_os:.2e} full {e_of:.2e} | state sketch {e_ss:.2e} full {e_sf:.2e} "
          f"| P {e_p:.2e} | sketch-vs-exact approximation {approx:.3e}")
    if bf:
        assert max(e_ss, e_sf, e_p) <= BF16_STATE_TOL
        assert max(e_os, e_of) <= BF16_OUT_TOL
    else:
        assert max(e_ss, e_sf) <= STATE_TOL and e_p <= STATE_TOL
        assert e_os <= OUT_TOL and e_of <= OUT_TOL
        assert max(e_os, e_of) <= TIGHT_OUT


def test_config0_all_heads():
    cfg = wl.CONFIGS[0]
    N = cfg.n_heads
    heads = np.arange(N)
    # start state: the oracle's 128-token prefill, rounded to the fp32 state both sides read
    pre = flat_tokens(wl.token_block(cfg, "prefill", 0, cfg.prefill))
    S0, _ = oracle.exact_steps(cfg.kind, np.zeros((N, cfg.dk, cfg.dv)), pre["k"], pre["v"], pre["alpha"])
    S0 = S0.astype(np.float32).astype(np.float64)
    U, R = _oracle_calibration(cfg, cfg.n_cal_seq, cfg.prefill, cfg.n_cal_q, "cpu")
    U, R = torch.from_numpy(U).float(), torch.from_numpy(R).float()
    dec = wl.token_block(cfg, "decode", 0, cfg.steps, with_query=True)
    ft = flat_tokens(dec)
    Uh, Rh = oracle.per_head(U, cfg.H, heads), oracle.per_head(R, cfg.H, heads)
    ref_s = oracle.sketch_path(cfg.kind, S0, Uh, Rh, ft, cfg.W)
    ref_f = oracle.fullread_path(cfg.kind, S0, ft)
    devtok = to_device(dec)
    src = lambda t0, n: {k: (None if v is None else v[t0:t0 + n]) for k, v in devtok.items()}  # noqa
    out = _run_gpu(cfg, to_gpu_state(S0, cfg.B, cfg.H), U, R, src, cfg.steps)
    _check(cfg, heads, *out, ref_s, ref_f, "config0")


def _sampled(cfg, n_windows=2, n_heads=48, cal=(8, 64, 512), label=""):
    import recurrent_state_read_b200 as rs
    from recurrent_state_read_b200.decode import prefill

    heads = wl.sample_heads(cfg, n_heads).numpy()
    d = _dims(cfg)
    # GPU prefill over all heads; the oracle prefills the sampled heads from the same tokens
    S0 = torch.zeros(cfg.B, cfg.H, cfg.dv, cfg.dk, dtype=cfg.torch_state_dtype, device="cuda")
    P = torch.empty(cfg.B, cfg.H, cfg.dv, cfg.r, device="cuda")
    Uz = torch.zeros(cfg.H, cfg.r, cfg.dk, device="cuda")
    sampled_pre = []

    def pre_source(t0, n):
        tok = wl.token_block(cfg, "prefill", t0, n, device="cuda")
        sampled_pre.append(flat_tokens(tok, heads))
        return tok

    prefill(d, S0, P, Uz, pre_source, cfg.prefill)
    ft_pre = {k: (None if sampled_pre[0][k] is None else np.concatenate([s[k] for s in sampled_pre]))
              for k in sampled_pre[0]}
    bf = cfg.state_dtype == "bf16"
    S0_ref = np.zeros((len(heads), cfg.dk, cfg.dv))
    for w0 in range(0, cfg.prefill, cfg.W):  # the oracle's window updates, rounding as the GPU stores
        sl = slice(w0, w0 + cfg.W)
        S0_ref, _ = oracle.update_window(cfg.kind, S0_ref, np.zeros((len(heads), cfg.dk, 1)), ft_pre["k"][sl],
                                         ft_pre["v"][sl], ft_pre["alpha"][sl],
                                         None if ft_pre["beta"] is None else ft_pre["beta"][sl], bf16_state=bf)
    torch.cuda.synchronize()
    e0 = state_err(to_logical(S0, heads), S0_ref)
    assert e0 <= (BF16_STATE_TOL if bf else STATE_TOL), e0
    # basis from the oracle's calibration on a reduced calibration set
    U, R = _oracle_calibration(cfg, *cal, device="cuda")
    U, R = torch.from_numpy(U).float(), torch.from_numpy(R).float()
    n_steps = n_windows * cfg.W
    sampled_dec = []

    def dec_source(t0, n):
        tok = wl.token_block(cfg, "decode", t0, n, device="cuda", with_query=True)
        sampled_dec.append(flat_tokens(tok, heads))
        return tok

    out = _run_gpu(cfg, S0, U, R, dec_source, n_steps)
    ft = {k: (None if sampled_dec[0][k] is None else np.concatenate([s[k] for s in sampled_dec]))
          for k in sampled_dec[0]}
    # the oracle continues from its own start state (fp32 / bf16 as stored)
    S0r = oracle.round_bf16(S0_ref) if bf else S0_ref.astype(np.float32).astype(np.float64)
    Uh, Rh = oracle.per_head(U, cfg.H, heads), oracle.per_head(R, cfg.H, heads)
    ref_s = oracle.sketch_path(cfg.kind, S0r, Uh, Rh, ft, cfg.W, bf16_state=bf)
    ref_f = oracle.fullread_path(cfg.kind, S0r, ft, bf16_state=bf)
    _check(cfg, heads, *out, ref_s, ref_f, label or cfg.describe())


def test_config1_mamba2_serving():
    _sampled(wl.CONFIGS[1])


def test_config2_gdn():
    _sampled(wl.CONFIGS[2])


@pytest.mark.parametrize("r", [4, 8, 16])
def test_config3_kda(r):
    _sampled(wl.workload(3, r=r))


# every (r, W) of the GDN sweep at B = 64 in both state dtypes, the B = 1024 corners, and one B = 256 point
SWEEP = ([dict(B=64, r=r, W=W, state_dtype=dt) for dt in ("f32", "bf16") for r in (4, 8, 16, 32) for W in (4, 8, 16, 32)]
         + [dict(B=1024, r=r, W=W, state_dtype=dt) for dt in ("f32", "bf16") for r in (4, 32) for W in (4, 32)]
         + [dict(B=256, r=16, W=8, state_dtype="bf16")])


@pytest.mark.parametrize("pt", SWEEP, ids=[f"B{p['B']}-r{p['r']}-W{p['W']}-{p['state_dtype']}" for p in SWEEP])
def test_config4_sweep_points(pt):
    _sampled(wl.workload(4, **pt), n_windows=1, n_heads=32)


@pytest.mark.parametrize("cfg_id", [1, 2, 3])
def test_full_length_schedule(cfg_id):
    """All 256 decode steps (16 windows) of the Mamba-2, GDN and KDA workloads at full batch, on
    sampled heads: error growth across every window of the run stays within the contract."""
    cfg = wl.CONFIGS[cfg_id]
    _sampled(cfg, n_windows=cfg.steps // cfg.W, n_heads=24, label=f"{cfg.describe()} (all {cfg.steps} steps)")
