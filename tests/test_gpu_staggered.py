"""GPU parity of the staggered serving schedule against the fp64 oracle.

Sequences reach the ends of their windows at different steps: sequence b runs
its windows with a phase of b mod W steps.  At each global step, the sequences
inside a window take a sketch step (sketchssm_decode_step_seq, one step index
per sequence) while the sequences whose window ends are updated and read
exactly in the same call (sketchssm_update_window_seqs with the query).

Reference: a sequence with phase p behaves as if its first window had started p
steps earlier with p identity tokens (k = 0, v = 0, decay 1), which change
neither the state nor any read.  Padding every head's token stream that way
aligns all windows, so the oracle's aligned sketch schedule gives the sketch
steps and its per-step exact recurrence gives the window-end steps.
"""

import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from tests.helpers import TIGHT_OUT, flat_tokens, rel_l2, state_err, to_gpu_state, to_logical

pytestmark = pytest.mark.gpu


def _padded(ft, phase, H, T, W):
    """[T, N, ...] token arrays -> [T + W, N, ...] with head n's token t at t + phase[n // H] and
    identity tokens elsewhere."""
    out = {}
    N = next(v for v in ft.values() if v is not None).shape[1]
    for key, x in ft.items():
        if x is None:
            out[key] = None
            continue
        fill = 1.0 if key == "alpha" else 0.0
        y = np.full((T + W,) + x.shape[1:], fill)
        for n in range(N):
            p = phase[n // H]
            y[p:p + T, n] = x[:, n]
        out[key] = y
    return out


@pytest.mark.parametrize("kind", ["mamba2", "gdn", "kda"])
def test_staggered_schedule(kind):
    import recurrent_state_read_b200 as rs
    from recurrent_state_read_b200.decode import WindowBuffer, stagger_plan, staggered_step

    cfg_id = {"mamba2": 1, "gdn": 2, "kda": 3}[kind]
    B, H, dk, dv, r, W, T = 8, 3, 64, 64, 8, 4, 11
    cfg = wl.workload(cfg_id, B=B, H=H, dk=dk, dv=dv, r=r, W=W, qkv_dtype="f32", q_rank=8)
    d = rs.dims(kind, B, H, dk, dv, r, W, torch.float32, torch.float32)
    N = B * H
    g = torch.Generator().manual_seed(11)
    S0 = torch.randn(N, dk, dv, generator=g, dtype=torch.float64).numpy().astype(np.float32).astype(np.float64)
    U = torch.randn(H, dk, r, generator=g) / dk ** 0.5
    R = torch.randn(H, r, dk, generator=g) / dk ** 0.5
    tok = wl.token_block(cfg, "decode", 0, T, with_query=True)  # [T, B, H, ...], global steps
    ft = flat_tokens(tok)
    phase = [b % W for b in range(B)]

    # GPU: window buffers start with the identity prefix of each sequence's first window
    dev = torch.device("cuda")
    S = to_gpu_state(S0, B, H)
    P = torch.empty(B, H, dv, r, device=dev)
    Ur = U.transpose(1, 2).contiguous().to(dev)
    Rd = R.to(dev)
    rs.sketchssm_update_window(d, S, P, Ur, None, None, None, None, 0)
    buf = WindowBuffer.empty(d, device=dev, with_query=False)
    buf.k.zero_()
    buf.v.zero_()
    buf.alpha.fill_(1.0)
    if buf.beta is not None:
        buf.beta.zero_()
    plan = stagger_plan(B, W, dev)
    out = torch.full((T, B, H, dv), float("nan"), device=dev)
    tk = {k: (None if v is None else v.to(dev)) for k, v in tok.items()}
    for s in range(T):
        for b in range(B):  # each sequence writes its token into its own next slot
            slot = (s + phase[b]) % W
            buf.k[b, :, slot] = tk["k"][s, b]
            buf.v[b, :, slot] = tk["v"][s, b]
            buf.alpha[b, :, slot] = tk["alpha"][s, b]
            if buf.beta is not None:
                buf.beta[b, :, slot] = tk["beta"][s, b]
        staggered_step(d, S, P, Ur, Rd, buf, tk["q"][s].contiguous(), plan[s % W], out[s])
    torch.cuda.synchronize()
    assert rs.sketchssm_device_error_count(1) == 0

    # oracle on the padded, aligned streams
    pt = _padded(ft, phase, H, T, W)
    heads = np.arange(N)
    Os, _, _ = oracle.sketch_path(kind, S0, oracle.per_head(U, H, heads), oracle.per_head(R, H, heads), pt, W)
    _, Oe = oracle.exact_steps(kind, S0, pt["k"], pt["v"], pt["alpha"], pt["beta"], pt["q"])
    got = out.reshape(T, N, dv).double().cpu().numpy()
    for s in range(T):
        for b in range(B):
            tp = s + phase[b]
            ref = Oe if tp % W == W - 1 else Os
            sl = slice(b * H, (b + 1) * H)
            assert rel_l2(got[s, sl], ref[tp, sl]) <= TIGHT_OUT, (s, b)
    # the state after each sequence's last completed window
    for b in range(B):
        done = (T + phase[b]) // W * W  # padded steps applied so far
        Sref, _ = oracle.exact_steps(kind, S0[b * H:(b + 1) * H], pt["k"][:done, b * H:(b + 1) * H],
                                     pt["v"][:done, b * H:(b + 1) * H], pt["alpha"][:done, b * H:(b + 1) * H],
                                     None if pt["beta"] is None else pt["beta"][:done, b * H:(b + 1) * H])
        assert state_err(to_logical(S)[b * H:(b + 1) * H], Sref) <= 1e-5, b
