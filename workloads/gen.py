"""Seeded generators for the decode workloads of the SketchSSM pages.

Source of the workloads: the SketchSSM abstract (arXiv 2609.33051v1, readsearch
listing, "Abstract") names Mamba-2-, GDN- and KDA-based models served at large
decode batch; the shapes and distributions below are the five workload
definitions this library is measured on (a tiny Mamba-2 correctness case,
Mamba-2 at serving batch, Gated DeltaNet, KDA, and a GDN sweep).

Every random draw is keyed by (seed, workload id, stream, token index), so any
window of tokens can be regenerated on its own, on any torch device, without
generating the tokens before it.  The same device gives the same values; CPU
and CUDA generators give different (equally distributed) values, so a parity
check always generates once and hands the same tensors to both sides.

Readings taken where the workload text is silent (each one is listed in the
design notes with its reason):
  * the query generator basis Q0 is shared by all heads;
  * k and v of the Mamba-2 serving workload follow the tiny case
    (k ~ N(0,1)/sqrt(dk), v ~ N(0,1));
  * for GDN and KDA the query is drawn from the rank-8 generator and then
    L2-normalised, like k; v ~ N(0,1);
  * calibration: 1024 queries where the workload gives no count for Mamba-2,
    4096 for KDA; calibration states are the final prefill states of 64
    seeded calibration sequences with the workload's prefill length;
  * Mamba-2 has no beta (the update is S <- a S + k v^T); beta is None there.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import numpy as np
import torch

KINDS = {"mamba2": 0, "gdn": 1, "kda": 2}

# stream ids: independent random streams of one workload
_STREAM = {"prefill": 1, "decode": 2, "query": 3, "cal": 4, "calq": 5, "q0": 6, "heads": 7}


@dataclasses.dataclass(frozen=True)
class Workload:
    id: int
    kind: str
    B: int
    H: int
    dk: int
    dv: int
    r: int
    W: int
    steps: int
    prefill: int
    qkv_dtype: str  # "f32" | "bf16"
    state_dtype: str  # "f32" | "bf16"
    q_rank: int  # rank of the query generator Q0
    n_cal_q: int  # calibration queries per head
    n_cal_seq: int  # calibration sequences (states per head)
    decay_mu: float  # decay pre-activation x ~ N(mu, sigma)
    decay_sigma: float
    normalise_qk: bool
    seed: int = 0

    @property
    def kind_id(self) -> int:
        return KINDS[self.kind]

    @property
    def torch_qkv_dtype(self) -> torch.dtype:
        return torch.float32 if self.qkv_dtype == "f32" else torch.bfloat16

    @property
    def torch_state_dtype(self) -> torch.dtype:
        return torch.float32 if self.state_dtype == "f32" else torch.bfloat16

    @property
    def n_heads(self) -> int:
        return self.B * self.H

    def describe(self) -> str:
        return (f"{self.kind} B={self.B} H={self.H} dk={self.dk} dv={self.dv} r={self.r} "
                f"W={self.W} steps={self.steps} qkv={self.qkv_dtype} state={self.state_dtype}")


CONFIGS: Dict[int, Workload] = {
    # tiny Mamba-2 correctness case: everything fp32
    0: Workload(0, "mamba2", B=4, H=8, dk=64, dv=64, r=8, W=8, steps=64, prefill=128,
                qkv_dtype="f32", state_dtype="f32", q_rank=8, n_cal_q=1024, n_cal_seq=64,
                decay_mu=0.0, decay_sigma=1.0, normalise_qk=False),
    # Mamba-2 at serving batch
    1: Workload(1, "mamba2", B=256, H=128, dk=128, dv=64, r=8, W=16, steps=256, prefill=512,
                qkv_dtype="bf16", state_dtype="f32", q_rank=12, n_cal_q=1024, n_cal_seq=64,
                decay_mu=-2.0, decay_sigma=1.0, normalise_qk=False),
    # Gated DeltaNet
    2: Workload(2, "gdn", B=256, H=32, dk=128, dv=128, r=8, W=16, steps=256, prefill=512,
                qkv_dtype="bf16", state_dtype="f32", q_rank=8, n_cal_q=4096, n_cal_seq=64,
                decay_mu=-3.0, decay_sigma=1.0, normalise_qk=True),
    # KDA (channel-wise decay); r in {4, 8, 16}
    3: Workload(3, "kda", B=512, H=32, dk=128, dv=128, r=8, W=16, steps=256, prefill=512,
                qkv_dtype="bf16", state_dtype="f32", q_rank=8, n_cal_q=4096, n_cal_seq=64,
                decay_mu=-3.0, decay_sigma=1.5, normalise_qk=True),
    # GDN sweep base (B in {64,256,1024}, r in {4,8,16,32}, W in {4,8,16,32}, state f32/bf16)
    4: Workload(4, "gdn", B=256, H=32, dk=128, dv=128, r=8, W=16, steps=256, prefill=512,
                qkv_dtype="bf16", state_dtype="f32", q_rank=8, n_cal_q=4096, n_cal_seq=64,
                decay_mu=-3.0, decay_sigma=1.0, normalise_qk=True),
}


def workload(cfg_id: int, **override) -> Workload:
    """The workload `cfg_id`, with fields (B, r, W, state_dtype, steps, ...) overridden."""
    return dataclasses.replace(CONFIGS[cfg_id], **override)


def _seed(cfg: Workload, stream: str, index: int) -> int:
    ss = np.random.SeedSequence([cfg.seed, cfg.id, _STREAM[stream], index])
    return int(ss.generate_state(1, np.uint64)[0] & ((1 << 63) - 1))


def _gen(cfg: Workload, stream: str, index: int, device) -> torch.Generator:
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(_seed(cfg, stream, index))
    return g


def _softplus64(x: torch.Tensor) -> torch.Tensor:
    x = x.double()
    return torch.where(x > 30.0, x, torch.log1p(torch.exp(torch.clamp(x, max=30.0))))


def _decay(x: torch.Tensor) -> torch.Tensor:
    """exp(-softplus(x)), evaluated in fp64 and stored fp32."""
    return torch.exp(-_softplus64(x)).float()


def _sigmoid(x: torch.Tensor) -> torch.Tensor:
    return torch.sigmoid(x.double()).float()


def _l2n(x: torch.Tensor) -> torch.Tensor:
    x = x.double()
    return (x / torch.linalg.vector_norm(x, dim=-1, keepdim=True)).float()


def query_basis(cfg: Workload, device="cpu") -> torch.Tensor:
    """Q0: a seeded dk x q_rank matrix with orthonormal columns (QR of a Gaussian), fp32."""
    g = _gen(cfg, "q0", 0, "cpu")
    a = torch.randn(cfg.dk, cfg.q_rank, generator=g, dtype=torch.float64)
    q, rr = torch.linalg.qr(a)
    q = q * torch.sign(torch.diagonal(rr))[None, :]
    return q.float().to(device)


def _queries(cfg: Workload, g: torch.Generator, shape, Q0: torch.Tensor) -> torch.Tensor:
    """q = Q0 z + 0.1 eps, z ~ N(0, I_rank), eps ~ N(0, I_dk); L2-normalised for GDN/KDA."""
    dev = Q0.device
    z = torch.randn(*shape, cfg.q_rank, generator=g, device=dev)
    eps = torch.randn(*shape, cfg.dk, generator=g, device=dev)
    q = (z.double() @ Q0.double().T + 0.1 * eps.double()).float()
    if cfg.normalise_qk:
        q = _l2n(q)
    return q


def _token(cfg: Workload, stream: str, t: int, B: int, device, Q0: Optional[torch.Tensor],
           with_query: bool) -> Dict[str, torch.Tensor]:
    g = _gen(cfg, stream, t, device)
    dev = torch.device(device)
    H, dk, dv = cfg.H, cfg.dk, cfg.dv
    k = torch.randn(B, H, dk, generator=g, device=dev)
    v = torch.randn(B, H, dv, generator=g, device=dev)
    if cfg.kind == "kda":
        xa = torch.randn(B, H, dk, generator=g, device=dev) * cfg.decay_sigma + cfg.decay_mu
    else:
        xa = torch.randn(B, H, generator=g, device=dev) * cfg.decay_sigma + cfg.decay_mu
    xb = torch.randn(B, H, generator=g, device=dev)
    if cfg.normalise_qk:
        k = _l2n(k)
    else:
        k = k / math.sqrt(dk)
    out = {
        "k": k.to(cfg.torch_qkv_dtype),
        "v": v.to(cfg.torch_qkv_dtype),
        "alpha": _decay(xa),
        "beta": None if cfg.kind == "mamba2" else _sigmoid(xb),
    }
    if with_query:
        # decode queries have a stream of their own, so that k/v/decay draws do not
        # depend on whether queries are requested
        gq = _gen(cfg, "query", t, device)
        out["q"] = _queries(cfg, gq, (B, H), Q0.to(dev)).to(cfg.torch_qkv_dtype)
    return out


def token_block(cfg: Workload, stream: str, t0: int, n: int, device="cpu", B: Optional[int] = None,
                with_query: bool = False) -> Dict[str, torch.Tensor]:
    """Tokens t0 .. t0+n-1 of `stream` ("prefill", "decode" or "cal"), stacked time-major.

    Returns k [n,B,H,dk], v [n,B,H,dv] (qkv dtype), alpha [n,B,H] fp32 (KDA: [n,B,H,dk]),
    beta [n,B,H] fp32 (None for Mamba-2) and, with `with_query`, q [n,B,H,dk].
    `B` defaults to the workload's batch (the "cal" stream uses n_cal_seq).
    """
    if B is None:
        B = cfg.n_cal_seq if stream == "cal" else cfg.B
    if with_query and stream != "decode":
        raise ValueError("queries exist only on the decode stream")
    Q0 = query_basis(cfg, device) if with_query else None
    toks = [_token(cfg, stream, t, B, device, Q0, with_query) for t in range(t0, t0 + n)]
    out = {}
    for key in toks[0]:
        if toks[0][key] is None:
            out[key] = None
        else:
            out[key] = torch.stack([tk[key] for tk in toks], 0)
    return out


def calibration_queries(cfg: Workload, device="cpu", n: Optional[int] = None) -> torch.Tensor:
    """Calibration queries [H, n, dk] fp32 (values rounded to the workload's qkv dtype)."""
    n = cfg.n_cal_q if n is None else n
    g = _gen(cfg, "calq", 0, device)
    q = _queries(cfg, g, (n, cfg.H), query_basis(cfg, device))
    q = q.to(cfg.torch_qkv_dtype).float()
    return q.permute(1, 0, 2).contiguous()


def sample_heads(cfg: Workload, n: int) -> torch.Tensor:
    """A seeded sample of n distinct flat head indices b*H + h (sorted), for sampled parity checks."""
    g = _gen(cfg, "heads", 0, "cpu")
    n = min(n, cfg.n_heads)
    idx = torch.randperm(cfg.n_heads, generator=g)[:n]
    return torch.sort(idx).values
