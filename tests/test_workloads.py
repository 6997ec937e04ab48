"""The seeded input generator: shapes, determinism and distributions.

The expected moments come from numerical integration of the stated
distributions (scipy.integrate.quad), independent of the generator's code.
"""

import math

import numpy as np
import pytest
import torch
from scipy import integrate

import workloads as wl


def test_configs_match_workload_table():
    c = wl.CONFIGS
    assert (c[0].kind, c[0].B, c[0].H, c[0].dk, c[0].dv, c[0].r, c[0].W, c[0].steps) == \
        ("mamba2", 4, 8, 64, 64, 8, 8, 64)
    assert (c[1].kind, c[1].B, c[1].H, c[1].dk, c[1].dv, c[1].r, c[1].W, c[1].steps) == \
        ("mamba2", 256, 128, 128, 64, 8, 16, 256)
    assert (c[2].kind, c[2].B, c[2].H, c[2].dk, c[2].dv, c[2].r, c[2].W) == ("gdn", 256, 32, 128, 128, 8, 16)
    assert (c[3].kind, c[3].B, c[3].H, c[3].dk, c[3].dv, c[3].W) == ("kda", 512, 32, 128, 128, 16)
    assert c[1].qkv_dtype == "bf16" and c[0].qkv_dtype == "f32"
    assert c[0].prefill == 128 and c[1].prefill == 512
    assert c[0].n_cal_q == 1024 and c[2].n_cal_q == 4096


def test_shapes_and_dtypes():
    cfg = wl.workload(3, B=2, H=3)
    tok = wl.token_block(cfg, "decode", 5, 4, with_query=True)
    assert tok["k"].shape == (4, 2, 3, 128) and tok["k"].dtype == torch.bfloat16
    assert tok["alpha"].shape == (4, 2, 3, 128) and tok["alpha"].dtype == torch.float32
    assert tok["beta"].shape == (4, 2, 3)
    assert tok["q"].shape == (4, 2, 3, 128)
    m = wl.token_block(wl.workload(0), "prefill", 0, 2)
    assert m["beta"] is None and m["alpha"].shape == (2, 4, 8) and m["k"].dtype == torch.float32


def test_windows_regenerate_independently():
    cfg = wl.workload(2, B=3, H=2)
    a = wl.token_block(cfg, "decode", 0, 8, with_query=True)
    b = wl.token_block(cfg, "decode", 4, 4, with_query=True)
    for key in ("k", "v", "alpha", "beta", "q"):
        assert torch.equal(a[key][4:], b[key])
    c = wl.token_block(cfg, "decode", 4, 4)
    assert torch.equal(c["k"], b["k"])  # requesting queries does not shift other draws


def test_query_basis_orthonormal():
    for cid in (0, 1, 2):
        Q0 = wl.query_basis(wl.CONFIGS[cid]).double()
        np.testing.assert_allclose((Q0.T @ Q0).numpy(), np.eye(Q0.shape[1]), atol=1e-6)


def _normal_expect(f, mu, sigma):
    pdf = lambda x: math.exp(-0.5 * ((x - mu) / sigma) ** 2) / (sigma * math.sqrt(2 * math.pi))  # noqa
    return integrate.quad(lambda x: f(x) * pdf(x), mu - 12 * sigma, mu + 12 * sigma, limit=200)[0]


@pytest.mark.parametrize("cid", [1, 2, 3])
def test_decay_and_beta_distributions(cid):
    cfg = wl.workload(cid, B=64, H=32)
    tok = wl.token_block(cfg, "prefill", 0, 4)
    a = tok["alpha"].double().flatten().numpy()
    dec = lambda x: math.exp(-math.log1p(math.exp(x)))  # noqa: exp(-softplus(x))
    mean = _normal_expect(dec, cfg.decay_mu, cfg.decay_sigma)
    var = _normal_expect(lambda x: dec(x) ** 2, cfg.decay_mu, cfg.decay_sigma) - mean ** 2
    assert abs(a.mean() - mean) < 6 * math.sqrt(var / a.size)
    assert (a > 0).all() and (a < 1).all()
    if tok["beta"] is not None:
        b = tok["beta"].double().flatten().numpy()
        sig = lambda x: 1 / (1 + math.exp(-x))  # noqa
        mb = _normal_expect(sig, 0.0, 1.0)
        vb = _normal_expect(lambda x: sig(x) ** 2, 0.0, 1.0) - mb ** 2
        assert abs(b.mean() - mb) < 6 * math.sqrt(vb / b.size)


def test_key_and_query_scaling():
    m = wl.token_block(wl.workload(0), "prefill", 0, 64)
    k = m["k"].double()
    assert abs(float((k * k).sum(-1).mean()) - 1.0) < 0.05  # N(0,1)/sqrt(dk): E||k||^2 = 1
    g = wl.token_block(wl.workload(2, B=4, H=4), "decode", 0, 3, with_query=True)
    for key in ("k", "q"):
        nrm = torch.linalg.vector_norm(g[key].double(), dim=-1)
        assert torch.allclose(nrm, torch.ones_like(nrm), atol=1e-2)  # unit norm up to bf16 rounding


def test_queries_are_low_rank_plus_noise():
    cfg = wl.workload(0)
    q = wl.calibration_queries(cfg).double()  # [H, Nq, dk]
    Q0 = wl.query_basis(cfg).double()
    resid = q - q @ Q0 @ Q0.T
    # noise 0.1 per channel outside the rank-8 span: E||resid||^2 = 0.01 (dk - 8)
    assert abs(float((resid ** 2).sum(-1).mean()) - 0.01 * (cfg.dk - 8)) < 0.01 * (cfg.dk - 8) * 0.05
    assert abs(float(((q @ Q0) ** 2).sum(-1).mean()) - (8 + 0.08)) < 0.3


def test_sample_heads():
    cfg = wl.CONFIGS[2]
    h = wl.sample_heads(cfg, 100)
    assert len(set(h.tolist())) == 100 and int(h.max()) < cfg.n_heads
    assert torch.equal(h, wl.sample_heads(cfg, 100))
