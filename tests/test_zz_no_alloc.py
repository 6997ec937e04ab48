"""The allocation-free calibration entry point against the ordinary one.

sketchssm_calibrate_basis_noalloc serves callers that cannot allocate device
memory when they calibrate (an engine whose memory all belongs to its own
pool, a plug-in under a fixed budget, code that cannot take cudaFree's device
synchronisation); it works in a fixed scratch array inside the library.  This
test calls it through the C ABI twice in a row -- so the second call starts
from the scratch contents the first call left -- and checks each result
against sketchssm_calibrate_basis on the same inputs, with head counts that
need several passes over the scratch.  It lives in a file of its own that
pytest collects last.
"""

import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kind,H,dk,dv,r", [("gdn", 12, 128, 128, 8), ("mamba2", 40, 64, 64, 4)])
def test_noalloc_matches_workspace_entry_point(kind, H, dk, dv, r):
    import recurrent_state_read_b200 as rs

    Ns, Nq = 8, 256
    g = torch.Generator(device="cuda").manual_seed(5)
    S_cal = torch.randn(Ns, H, dv, dk, generator=g, device="cuda")
    d = rs.dims(kind, Ns, H, dk, dv, r, 16, torch.float32, torch.bfloat16)
    U_ref = torch.empty(H, r, dk, device="cuda")  # basis rows
    R_ref = torch.empty(H, r, dk, device="cuda")
    for call in range(2):
        q_cal = torch.randn(H, Nq, dk, generator=g, device="cuda")
        rs.sketchssm_calibrate_basis(d, q_cal, S_cal, U_ref, R_ref)
        U = torch.full((H, r, dk), float("nan"), device="cuda")
        R = torch.full((H, r, dk), float("nan"), device="cuda")
        rs.sketchssm_calibrate_basis_noalloc(d, q_cal, S_cal, U, R)
        torch.cuda.synchronize()
        assert torch.isfinite(U).all() and torch.isfinite(R).all(), call
        Pi = torch.einsum("hri,hrk->hik", U.double(), R.double())
        Pi_ref = torch.einsum("hri,hrk->hik", U_ref.double(), R_ref.double())
        scale = max(1.0, float(Pi_ref.abs().max()))
        assert float((Pi - Pi_ref).abs().max()) <= 1e-5 * scale, call
        assert torch.allclose(U, U_ref, rtol=1e-5, atol=1e-6 * float(U_ref.abs().max())), call
        assert torch.allclose(R, R_ref, rtol=1e-5, atol=1e-6 * float(R_ref.abs().max())), call
