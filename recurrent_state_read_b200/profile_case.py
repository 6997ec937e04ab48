"""A small, self-contained case of one kernel, for Nsight Compute captures.

    python -m recurrent_state_read_b200.profile_case --kernel update --config 1 --B 64 --launches 3
    python -m recurrent_state_read_b200.profile_case --traffic --config 2
    python -m recurrent_state_read_b200.profile_case --summarize-traffic launches.csv --config 2

Builds seeded inputs directly on the device (a random state, a random basis,
one window of generated tokens) without prefill or calibration, then launches
the chosen kernel `--launches` times after one warm-up launch, so a capture
with `-k regex:<kernel> -s 1 -c <launches>` sees only the launches of interest.
Prints the per-launch CUDA-event time of the last launches (not a bench number).

--traffic runs, at the workload's full size, one warm-up sketch window (W decode
steps + the window update), one measured sketch window, one warm-up full-read
window (W full-read steps) and one measured full-read window, in that order, so
that a capture of DRAM bytes per launch (`ncu --cache-control none`) sees each
measured window with the cache contents its predecessor left.
--summarize-traffic reads the CSV of such a capture and prints the DRAM bytes of
each measured window per token-step and their ratio (the speed target's
"measured reduction in state traffic").
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
    ap.add_argument("--traffic", action="store_true")
    ap.add_argument("--summarize-traffic", metavar="CSV")
    a = ap.parse_args()
    over = {k: getattr(a, k) for k in ("B", "r", "W") if getattr(a, k) is not None}
    if a.state_dtype:
        over["state_dtype"] = a.state_dtype
    cfg = wl.workload(a.config, **over)
    if a.summarize_traffic:
        summarize_traffic(a.summarize_traffic, cfg)
        return
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

    if a.traffic:
        from recurrent_state_read_b200.decode import fullread_window, sketch_window

        out = torch.empty(cfg.W, cfg.B, cfg.H, cfg.dv, device=dev)
        tok2 = wl.token_block(cfg, "decode", cfg.W, cfg.W, device=dev, with_query=True)
        buf2 = WindowBuffer.empty(d, device=dev)
        buf2.fill(tok2)
        rs.sketchssm_update_window(d, S, P, U, None, None, None, None, 0)  # (not in the capture filter's count)
        for b in (buf, buf2):  # warm-up window, measured window
            sketch_window(d, S, P, U, R, b, out)
        for t in (tok, tok2):
            fullread_window(d, S, {k: (None if v is None else v.contiguous()) for k, v in t.items()}, out)
        torch.cuda.synchronize()
        print(f"traffic {cfg.describe()}: launches in order: refresh 1, sketch windows 2 x {cfg.W + 1}, "
              f"full-read windows 2 x {cfg.W}")
        return
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


def summarize_traffic(path, cfg):
    """DRAM bytes per token-step of the measured sketch window and full-read window, from the ncu CSV
    (--metrics dram__bytes_read.sum,dram__bytes_write.sum) of a --traffic run."""
    import csv

    launches = {}
    with open(path) as f:
        rows = [r for r in csv.reader(line for line in f if not line.startswith("=="))]
    head = rows[0]
    ci = {k: head.index(k) for k in ("ID", "Kernel Name", "Metric Name", "Metric Value")}
    for r in rows[1:]:
        if len(r) < len(head):
            continue
        lid = int(r[ci["ID"]])
        e = launches.setdefault(lid, {"name": r[ci["Kernel Name"]], "bytes": 0.0})
        if r[ci["Metric Name"]] in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
            v = float(r[ci["Metric Value"]].replace(",", ""))
            unit = r[head.index("Metric Unit")] if "Metric Unit" in head else "byte"
            scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "KB": 1e3, "MB": 1e6, "GB": 1e9}.get(unit, 1)
            e["bytes"] += v * scale
    seq = [launches[k] for k in sorted(launches)]
    W = cfg.W
    if len(seq) != 1 + 2 * (W + 1) + 2 * W:
        raise SystemExit(f"expected {1 + 2 * (W + 1) + 2 * W} launches of the library's kernels, found {len(seq)}")
    sk = seq[1 + (W + 1):1 + 2 * (W + 1)]
    fr = seq[1 + 2 * (W + 1) + W:]
    ts = cfg.B * W
    sk_b = sum(e["bytes"] for e in sk) / ts
    fr_b = sum(e["bytes"] for e in fr) / ts
    print(f"sketch window: {len(sk)} launches, {sum(e['bytes'] for e in sk) / 1e6:.1f} MB, "
          f"{sk_b:.0f} B per token-step")
    print(f"full-read window: {len(fr)} launches, {sum(e['bytes'] for e in fr) / 1e6:.1f} MB, "
          f"{fr_b:.0f} B per token-step")
    print(f"sketch_dram_bytes_per_token_step: {sk_b:.0f}")
    print(f"fullread_dram_bytes_per_token_step: {fr_b:.0f}")
    print(f"measured_bytes_ratio: {fr_b / sk_b:.3f}")
    for e in sk:
        print(f"  {e['name'][:60]:60s} {e['bytes'] / 1e6:9.2f} MB")


if __name__ == "__main__":
    main()
