"""GPU offline calibration (sketchssm_calibrate_basis) against the oracle's.

The two sides take different routes (the GPU: Cholesky of G, Jacobi on
L^T C L, U = L^-T V_r; the oracle: symmetric square roots from numpy's eigh and
a generic solve), so their U need not agree column by column; what any valid
answer must share is the G-weighted projector U R, the identity R U = I and the
calibration objective.  The calibration states are the oracle's prefill states
of seeded calibration sequences; the queries come from the workload generator.
"""

import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from oracle import calibration as cal
from tests.helpers import flat_tokens, to_gpu_state

pytestmark = pytest.mark.gpu


def _cal_inputs(cfg, n_seq, n_tokens, n_q):
    tok = flat_tokens(wl.token_block(cfg, "cal", 0, n_tokens, B=n_seq))
    S = np.zeros((n_seq * cfg.H, cfg.dk, cfg.dv))
    S, _ = oracle.exact_steps(cfg.kind, S, tok["k"], tok["v"], tok["alpha"], tok["beta"])
    S = S.astype(np.float32).astype(np.float64)
    q = wl.calibration_queries(cfg, n=n_q)
    return S.reshape(n_seq, cfg.H, cfg.dk, cfg.dv), q


@pytest.mark.parametrize("cid,n_seq,n_tokens,n_q,r", [
    (0, 64, 128, 1024, 8),     # the tiny Mamba-2 case with its full calibration recipe
    (2, 16, 64, 1024, 8),      # GDN shape, reduced calibration set
    (3, 16, 64, 1024, 16),     # KDA shape
    (1, 8, 64, 1024, 4),       # Mamba-2 dk=128, dv=64
    (2, 8, 32, 512, 128),      # complete basis: U R = I
])
def test_calibrate_matches_oracle(cid, n_seq, n_tokens, n_q, r):
    import recurrent_state_read_b200 as rs

    cfg = wl.workload(cid, H=min(wl.CONFIGS[cid].H, 6), r=r)
    S_cal, q_cal = _cal_inputs(cfg, n_seq, n_tokens, n_q)
    U_ref, R_ref = oracle.calibrate_heads(S_cal, q_cal.double().numpy(), r)
    d = rs.dims(cfg.kind, n_seq, cfg.H, cfg.dk, cfg.dv, r, cfg.W, torch.float32, cfg.torch_qkv_dtype)
    S_gpu = to_gpu_state(S_cal.reshape(n_seq * cfg.H, cfg.dk, cfg.dv), n_seq, cfg.H)
    U = torch.full((cfg.H, r, cfg.dk), float("nan"), device="cuda")  # basis rows
    R = torch.full((cfg.H, r, cfg.dk), float("nan"), device="cuda")
    rs.sketchssm_calibrate_basis(d, q_cal.cuda().contiguous(), S_gpu, U, R)
    torch.cuda.synchronize()
    U, R = U.transpose(1, 2).double().cpu().numpy(), R.double().cpu().numpy()
    for h in range(cfg.H):
        Pi, Pi_ref = U[h] @ R[h], U_ref[h] @ R_ref[h]
        scale = max(1.0, np.abs(Pi_ref).max())
        assert np.abs(Pi - Pi_ref).max() <= 1e-5 * scale, (h, np.abs(Pi - Pi_ref).max())
        np.testing.assert_allclose(R[h] @ U[h], np.eye(r), atol=1e-5)
        G = cal.gram_states(S_cal[:, h])
        C = cal.gram_queries(q_cal[h].double().numpy())
        j_gpu, j_ref = cal.objective(G, C, U[h], R[h]), cal.objective(G, C, U_ref[h], R_ref[h])
        assert j_gpu <= j_ref * (1 + 1e-4) + 1e-12 * np.trace(G @ C), (h, j_gpu, j_ref)


@pytest.mark.parametrize("cid,r", [(1, 8), (2, 8), (3, 16), (0, 4)])
def test_query_pca_matches_oracle(cid, r):
    """sketchssm_calibrate_query_pca: the projector U R onto the top-r query directions, R U = I
    and R = U^T, against the oracle's eigh-based query PCA on the same queries."""
    import recurrent_state_read_b200 as rs

    cfg = wl.workload(cid, H=min(wl.CONFIGS[cid].H, 5), r=r)
    q_cal = wl.calibration_queries(cfg, n=1024)
    U_ref, R_ref = oracle.query_pca_heads(q_cal.double().numpy(), r)
    d = rs.dims(cfg.kind, 1, cfg.H, cfg.dk, cfg.dv, r, cfg.W, torch.float32, cfg.torch_qkv_dtype)
    U = torch.full((cfg.H, r, cfg.dk), float("nan"), device="cuda")
    R = torch.full((cfg.H, r, cfg.dk), float("nan"), device="cuda")
    rs.sketchssm_calibrate_query_pca(d, q_cal.cuda().contiguous(), U, R)
    torch.cuda.synchronize()
    U, R = U.transpose(1, 2).double().cpu().numpy(), R.double().cpu().numpy()
    for h in range(cfg.H):
        Pi, Pi_ref = U[h] @ R[h], U_ref[h] @ R_ref[h]
        assert np.abs(Pi - Pi_ref).max() <= 1e-5, (h, np.abs(Pi - Pi_ref).max())
        np.testing.assert_allclose(R[h] @ U[h], np.eye(r), atol=1e-5)
        np.testing.assert_allclose(R[h], U[h].T, atol=1e-6)


def test_calibrate_bf16_states():
    import recurrent_state_read_b200 as rs

    cfg = wl.workload(2, H=3, r=8)
    S_cal, q_cal = _cal_inputs(cfg, 16, 64, 512)
    S_cal = oracle.round_bf16(S_cal)
    U_ref, R_ref = oracle.calibrate_heads(S_cal, q_cal.double().numpy(), 8)
    d = rs.dims("gdn", 16, cfg.H, 128, 128, 8, 16, torch.bfloat16, torch.bfloat16)
    S_gpu = to_gpu_state(S_cal.reshape(-1, 128, 128), 16, cfg.H, torch.bfloat16)
    U = torch.empty(cfg.H, 8, 128, device="cuda")  # basis rows
    R = torch.empty(cfg.H, 8, 128, device="cuda")
    rs.sketchssm_calibrate_basis(d, q_cal.cuda().contiguous(), S_gpu, U, R)
    torch.cuda.synchronize()
    for h in range(cfg.H):
        Pi = U[h].T.double().cpu().numpy() @ R[h].double().cpu().numpy()
        Pi_ref = U_ref[h] @ R_ref[h]
        assert np.abs(Pi - Pi_ref).max() <= 1e-5 * max(1.0, np.abs(Pi_ref).max())


@pytest.mark.parametrize("cid,r_max,r_avg", [(2, 16, 8), (1, 16, 8), (0, 8, 4)])
def test_calibrate_ranked_matches_oracle(cid, r_max, r_avg):
    """Ranked calibration: the GPU's eigenvalues against the oracle's spectra; the ranks, an integer
    decision, bit for bit against the oracle's allocation applied to the GPU's eigenvalues; rows
    past each rank zero; each head's projector against a rank-r_h oracle calibration."""
    import recurrent_state_read_b200 as rs

    cfg = wl.workload(cid, H=min(wl.CONFIGS[cid].H, 8), r=r_max, q_rank=12)
    S_cal, q_cal = _cal_inputs(cfg, 16, 64, 1024)
    # heads of different scales, so that the budget is spread unevenly
    S_cal = S_cal * np.linspace(0.5, 2.0, cfg.H)[None, :, None, None]
    q_np = q_cal.double().numpy() * np.linspace(0.5, 1.5, cfg.H)[:, None, None]
    q_cal = torch.from_numpy(q_np).float()
    d = rs.dims(cfg.kind, 16, cfg.H, cfg.dk, cfg.dv, r_max, cfg.W, torch.float32, cfg.torch_qkv_dtype)
    S_gpu = to_gpu_state(S_cal.reshape(16 * cfg.H, cfg.dk, cfg.dv), 16, cfg.H)
    U = torch.full((cfg.H, r_max, cfg.dk), float("nan"), device="cuda")
    R = torch.full((cfg.H, r_max, cfg.dk), float("nan"), device="cuda")
    rank = torch.full((cfg.H,), -1, dtype=torch.int32, device="cuda")
    lam = torch.full((cfg.H, r_max), float("nan"), dtype=torch.float64, device="cuda")
    rs.sketchssm_calibrate_basis_ranked(d, q_cal.cuda().contiguous(), S_gpu, r_avg, U, R, rank, lam)
    torch.cuda.synchronize()
    lam_g, rank_g = lam.cpu().numpy(), rank.cpu().numpy()
    q_f = q_cal.double().numpy()
    for h in range(cfg.H):
        spec = cal.spectrum_from_grams(cal.gram_states(S_cal[:, h]), cal.gram_queries(q_f[h]))[:r_max]
        np.testing.assert_allclose(lam_g[h], spec, rtol=1e-6, atol=1e-9 * spec[0])
    assert rank_g.tolist() == cal.allocate_ranks(lam_g, r_avg, r_max).tolist()
    assert rank_g.sum() == cfg.H * r_avg and len(set(rank_g.tolist())) > 1
    Ug, Rg = U.transpose(1, 2).double().cpu().numpy(), R.double().cpu().numpy()
    for h in range(cfg.H):
        rh = int(rank_g[h])
        assert np.all(Ug[h][:, rh:] == 0) and np.all(Rg[h][rh:] == 0)
        if rh:
            U_ref, R_ref = cal.calibrate(S_cal[:, h], q_f[h], rh)
            Pi, Pi_ref = Ug[h] @ Rg[h], U_ref @ R_ref
            assert np.abs(Pi - Pi_ref).max() <= 1e-5 * max(1.0, np.abs(Pi_ref).max()), h
