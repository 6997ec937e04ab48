"""The SketchSSM decode schedule on the GPU, composed from the C entry points.

Timeline (SketchSSM abstract and the agihunt digest's "Mechanism details"):
within a window of W steps the state is fixed; step j reads the sketch and the
buffered tokens 1..j; after the window's last step one kernel applies the W
buffered tokens to the state and refreshes the sketch.  The full-read baseline
updates and reads the whole state at every step; the ReplaySSM-style baseline
(the buffering the SketchSSM abstract starts from) reads the full window-start
state at every step and writes it once per window.  This module is host-side
control flow only: every arithmetic step runs in libsketchssm.so.
"""

from __future__ import annotations

import dataclasses
from typing import Optional

import torch

from . import (sketchssm_decode_step, sketchssm_decode_step_seq, sketchssm_dims, sketchssm_fullread_decode,
               sketchssm_replay_decode_step, sketchssm_update_window, sketchssm_update_window_read,
               sketchssm_update_window_seqs)


@dataclasses.dataclass
class WindowBuffer:
    """Device window buffer, head-major: k [B,H,W,dk], v [B,H,W,dv], alpha [B,H,W] (KDA
    [B,H,W,dk]), beta [B,H,W] (None for Mamba-2); q [W,B,H,dk] holds the queries of the
    window's steps (one [B,H,dk] plane per step)."""
    k: torch.Tensor
    v: torch.Tensor
    alpha: torch.Tensor
    beta: Optional[torch.Tensor]
    q: Optional[torch.Tensor] = None

    @staticmethod
    def empty(d: sketchssm_dims, device="cuda", with_query=True) -> "WindowBuffer":
        qt = torch.float32 if d.qkv_dtype == 0 else torch.bfloat16
        W, B, H = d.W, d.B, d.H
        a_shape = (B, H, W, d.dk) if d.kind == 2 else (B, H, W)
        return WindowBuffer(
            k=torch.empty(B, H, W, d.dk, dtype=qt, device=device),
            v=torch.empty(B, H, W, d.dv, dtype=qt, device=device),
            alpha=torch.empty(a_shape, dtype=torch.float32, device=device),
            beta=None if d.kind == 0 else torch.empty(B, H, W, dtype=torch.float32, device=device),
            q=torch.empty(W, B, H, d.dk, dtype=qt, device=device) if with_query else None,
        )

    def fill(self, tok: dict, n: Optional[int] = None):
        """Copy time-major tokens (dict of [n,B,H,...] tensors) into slots 0..n-1."""
        n = tok["k"].shape[0] if n is None else n
        for name in ("k", "v", "alpha", "beta"):
            dst = getattr(self, name)
            if dst is not None and tok.get(name) is not None:
                src = tok[name][:n]
                dst[:, :, :n].copy_(src.movedim(0, 2), non_blocking=True)
        if self.q is not None and tok.get("q") is not None:
            self.q[:n].copy_(tok["q"][:n], non_blocking=True)


def sketch_window(d: sketchssm_dims, S, P, U, R, buf: WindowBuffer, out, n: Optional[int] = None,
                  stream=None, exact_last: bool = False):
    """One window of the sketch path: n decode steps (outputs into out[0..n-1], each [B,H,dv]
    fp32) read the sketch; then one window update applies the n tokens and refreshes P.
    exact_last: step n is not read from the sketch but exactly, inside the window update
    (sketchssm_update_window_read), which holds the updated state anyway."""
    n = d.W if n is None else n
    for j in range(1, (n - 1 if exact_last else n) + 1):
        sketchssm_decode_step(d, P, R, buf.q[j - 1], buf.k, buf.v, buf.alpha, buf.beta, j, out[j - 1],
                              stream)
    if exact_last and n > 0:
        sketchssm_update_window_read(d, S, P, U, buf.k, buf.v, buf.alpha, buf.beta, n, buf.q[n - 1],
                                     out[n - 1], stream)
    else:
        sketchssm_update_window(d, S, P, U, buf.k, buf.v, buf.alpha, buf.beta, n, stream)


def stagger_plan(B: int, W: int, device="cuda"):
    """Staggered windows: sequence b runs its windows with a phase of b mod W steps, so that at every
    step about B/W sequences end a window.  For each step s of a W-step cycle: (j_seq, seqs), where
    j_seq [B] int32 is each sequence's sketch step (0 for the sequences whose window ends at s) and
    seqs int32 lists those sequences (their last step is read exactly by the window update)."""
    b = torch.arange(B)
    plan = []
    for s in range(W):
        j = (s + b) % W + 1
        ends = j == W
        plan.append((torch.where(ends, torch.zeros_like(j), j).to(torch.int32).to(device),
                     b[ends].to(torch.int32).to(device)))
    return plan


def staggered_step(d: sketchssm_dims, S, P, U, R, buf: WindowBuffer, q, plan_s, out, sm_share=(0, 0),
                   streams=(None, None)):
    """One decode step of the staggered schedule: the sequences inside a window read the sketch
    (q [B,H,dk] holds every sequence's query of this step; out [B,H,dv]), while the sequences whose
    window ends are updated and read exactly.  The two launches touch disjoint sequences, so they
    may run concurrently on two streams (streams = (decode, update)); sm_share caps each one's CTAs
    per SM so that both fit on the GPU together."""
    j_seq, seqs = plan_s
    sketchssm_decode_step_seq(d, P, R, q, buf.k, buf.v, buf.alpha, buf.beta, j_seq, out, sm_share[0],
                              streams[0])
    if seqs.numel() > 0:
        sketchssm_update_window_seqs(d, S, P, U, buf.k, buf.v, buf.alpha, buf.beta, d.W, seqs, q, out,
                                     sm_share[1], streams[1])


def replay_window(d: sketchssm_dims, S, buf: WindowBuffer, out, n: Optional[int] = None, stream=None):
    """One window of the ReplaySSM-style path: n decode steps each read the full window-start
    state exactly (no write); one window update then applies the n tokens (no sketch)."""
    n = d.W if n is None else n
    for j in range(1, n + 1):
        sketchssm_replay_decode_step(d, S, buf.q[j - 1], buf.k, buf.v, buf.alpha, buf.beta, j, out[j - 1],
                                     stream)
    sketchssm_update_window(d, S, None, None, buf.k, buf.v, buf.alpha, buf.beta, n, stream)


def fullread_window(d: sketchssm_dims, S, tok: dict, out, n: Optional[int] = None, stream=None):
    """n steps of the full-read baseline over time-major tokens (dict of contiguous
    [n,B,H,...] device tensors k, v, alpha, beta, q): one token plane per step."""
    n = tok["k"].shape[0] if n is None else n
    beta = tok.get("beta")
    for t in range(n):
        sketchssm_fullread_decode(d, S, tok["q"][t], tok["k"][t], tok["v"][t], tok["alpha"][t],
                                  None if beta is None else beta[t], out[t], stream)


def prefill(d: sketchssm_dims, S, P, U, token_source, n_tokens: int, stream=None):
    """Advance S through n_tokens tokens with window updates of up to W tokens each.

    token_source(t0, n) returns a dict of time-major device tensors [n,B,H,...] for tokens
    t0..t0+n-1.  P is refreshed as a by-product (the last refresh is the sketch of the final state).
    """
    buf = WindowBuffer.empty(d, device=S.device, with_query=False)
    for t0 in range(0, n_tokens, d.W):
        n = min(d.W, n_tokens - t0)
        buf.fill(token_source(t0, n), n)
        sketchssm_update_window(d, S, P, U, buf.k, buf.v, buf.alpha, buf.beta, n, stream)
    if n_tokens == 0:
        sketchssm_update_window(d, S, P, U, None, None, None, None, 0, stream)
