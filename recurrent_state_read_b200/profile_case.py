"""A small, self-contained case of one kernel, for Nsight Compute captures.

    python -m recurrent_state_read_b200.profile_case --kernel update --config 1 --B 64 --launches 3

Builds seeded inputs directly on the device (a random state, a random basis,
one window of generated tokens) without prefill or calibration, then launches
the chosen kernel `--launches` times after one warm-up launch, so a capture
with `-k regex:<kernel> -s 1 -c <launches>` sees only the launches of interest.
Prints the per-launch CUDA-event time of the last launches (not a bench number).
"""

from __future__ import annotations

import argparse
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def main():
    import torch

    import recurrent_state_read_b200 as rs
    import workloads as wl
    from recurrent_state_read_b200.decode import WindowBuffer

    ap = argparse.ArgumentParser()
    ap.add_argument("--kernel", choices=["update", "decode", "fullread"], default="update")
    ap.add_argument("--config", type=int, default=1)
    ap.add_argument("--B", type=int)
    ap.add_argument("--r", type=int)
    ap.add_argument("--W", type=int)
    ap.add_argument("--state-dtype", choices=["f32", "bf16"])
    ap.add_argument("--j", type=int, help="decode step index (default W)")
    ap.add_argument("--launches", type=int, default=3)
    a = ap.parse_args()
    over = {k: getattr(a, k) for k in ("B", "r", "W") if getattr(a, k) is not None}
    if a.state_dtype:
        over["state_dtype"] = a.state_dtype
    cfg = wl.workload(a.config, **over)
    d = rs.dims(cfg.kind, cfg.B, cfg.H, cfg.dk, cfg.dv, cfg.r, cfg.W, cfg.torch_state_dtype, cfg.torch_qkv_dtype)
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev).manual_seed(0)
    S = (0.1 * torch.randn(cfg.B, cfg.H, cfg.dv, cfg.dk, generator=g, device=dev)).to(cfg.torch_state_dtype)
    P = torch.randn(cfg.B, cfg.H, cfg.dv, cfg.r, generator=g, device=dev)
    U = torch.randn(cfg.H, cfg.r, cfg.dk, generator=g, device=dev) / cfg.dk ** 0.5  # basis rows
    R = torch.randn(cfg.H, cfg.r, cfg.dk, generator=g, device=dev) / cfg.dk ** 0.5
    tok = wl.token_block(cfg, "decode", 0, cfg.W, device=dev, with_query=True)  # time-major
    buf = WindowBuffer.empty(d, device=dev)
    buf.fill(tok)
    o = torch.empty(cfg.B, cfg.H, cfg.dv, device=dev)
    j = cfg.W if a.j is None else a.j

    def launch():
        if a.kernel == "update":
            rs.sketchssm_update_window(d, S, P, U, buf.k, buf.v, buf.alpha, buf.beta, cfg.W)
        elif a.kernel == "decode":
            rs.sketchssm_decode_step(d, P, R, buf.q[j - 1], buf.k, buf.v, buf.alpha, buf.beta, j, o)
        else:
            rs.sketchssm_fullread_decode(d, S, tok["q"][0], tok["k"][0], tok["v"][0], tok["alpha"][0],
                                         None if tok["beta"] is None else tok["beta"][0], o)

    launch()
    torch.cuda.synchronize()
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(a.launches + 1)]
    evs[0].record()
    for i in range(a.launches):
        launch()
        evs[i + 1].record()
    torch.cuda.synchronize()
    ms = [evs[i].elapsed_time(evs[i + 1]) for i in range(a.launches)]
    print(f"{a.kernel} {cfg.describe()}: per-launch ms {['%.4f' % x for x in ms]}")


if __name__ == "__main__":
    main()
