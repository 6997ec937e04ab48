"""Decode benchmark of the SketchSSM windowed decode on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 1] [--B .. --r .. --W .. --state-dtype ..]
    python bench.py --impl reference ...     # the fp64 CPU oracle on the host cores

One step is one window of the decode loop for the whole batch: W decode steps
that read only the sketch, then the fused window update (exact state update +
sketch refresh), i.e. B*W token-steps (a token-step is one new token of one
sequence through one linear-attention layer of H heads).  The full-read
baseline runs the same windows with one full-state read+write per token.
Inputs are seeded synthetic tensors shaped like the workload (default: Mamba-2
at serving batch, B=256 H=128 dk=128 dv=64 r=8 W=16, bf16 q/k/v, fp32 state);
the start state comes from a 512-token prefill run by the library's own window
update, and the basis from the library's calibration on 64 prefilled
calibration sequences.  Each step's working set (state, window buffer) is
larger than L2, and NWIN distinct windows are cycled, so no step reuses another
step's inputs from cache.  Timing: CUDA events on the launching stream, each
window captured as a CUDA graph (both paths alike), warm-up first; for N>1 each
rank runs an independent replica and the max time over ranks is taken.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode token-steps/s at B=256; achieved HBM GB/s vs peak; sketch vs full-read"
UNIT = "token-steps/s"
NWIN = 4  # distinct windows cycled through the timed steps
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", type=int, default=1)
    ap.add_argument("--B", type=int)
    ap.add_argument("--r", type=int)
    ap.add_argument("--W", type=int)
    ap.add_argument("--state-dtype", choices=["f32", "bf16"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=16.0)
    ap.add_argument("--rank-avg", type=int, default=0,
                    help="also time the sketch path with a rank per head: this average, the config's r the largest")
    ap.add_argument("--stagger-share", default="2,2",
                    help="CTAs per SM for the decode and update kernels of the staggered schedule")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the other workloads (GDN, KDA r = 4, 8, 16) of the single-GPU line")
    ap.add_argument("--workload-steps", type=int, default=30)
    ap.add_argument("--no-sweep", action="store_true", help="skip the GDN sweep of the single-GPU line")
    ap.add_argument("--sweep-steps", type=int, default=10)
    return ap.parse_args()


def workload_of(args):
    import workloads as wl

    over = {}
    for k in ("B", "r", "W"):
        if getattr(args, k) is not None:
            over[k] = getattr(args, k)
    if args.state_dtype:
        over["state_dtype"] = args.state_dtype
    return wl.workload(args.config, **over)


def config_json(cfg):
    names = {0: "Mamba-2 tiny correctness case", 1: "Mamba-2 decode at serving batch", 2: "Gated DeltaNet decode",
             3: "KDA decode", 4: "GDN sweep point"}
    return {
        "workload": f"{names[cfg.id]}: {cfg.kind} B={cfg.B} H={cfg.H} dk={cfg.dk} dv={cfg.dv} r={cfg.r} "
                    f"W={cfg.W}, q/k/v {cfg.qkv_dtype}, state {cfg.state_dtype}",
        "kind": cfg.kind, "B": cfg.B, "H": cfg.H, "dk": cfg.dk, "dv": cfg.dv, "r": cfg.r, "W": cfg.W,
        "qkv_dtype": cfg.qkv_dtype, "state_dtype": cfg.state_dtype, "prefill": cfg.prefill,
        "step": f"one window: {cfg.W} sketch decode steps + 1 fused window update = B*W token-steps",
        "l2": "inputs larger than L2 (state and window buffer per step), "
              f"{NWIN} distinct windows cycled; no flush",
    }


# ---------------------------------------------------------------- bytes model
def bytes_model(cfg):
    """Algorithmic HBM bytes of each kernel launch (every buffered-token re-read counted)."""
    NH = cfg.B * cfg.H
    s = 4 if cfg.state_dtype == "f32" else 2
    qb = 4 if cfg.qkv_dtype == "f32" else 2
    S = NH * cfg.dk * cfg.dv * s
    P = NH * cfg.dv * cfg.r * 4
    a = 4 * cfg.dk if cfg.kind == "kda" else 4
    b = 0 if cfg.kind == "mamba2" else 4
    tau = NH * (cfg.dk * qb + cfg.dv * qb + a + b)  # one buffered token, all heads
    q = NH * cfg.dk * qb
    o = NH * cfg.dv * 4
    UR = cfg.H * cfg.dk * cfg.r * 4
    upd = 2 * S + P + cfg.W * tau + UR
    dec = [P + UR + q + j * tau + o for j in range(1, cfg.W + 1)]
    full = 2 * S + q + tau + o
    replay = [S + q + j * tau + o for j in range(1, cfg.W + 1)]  # reads S, writes nothing
    replay_upd = 2 * S + cfg.W * tau                              # the window update without a sketch
    return {"S": S, "P": P, "tau": tau, "update": upd, "decode": dec, "decode_avg": sum(dec) / len(dec),
            "fullread": full, "sketch_step": upd + sum(dec), "full_step": cfg.W * full,
            "replay_avg": sum(replay) / len(replay), "replay_step": replay_upd + sum(replay)}


def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured (MEASURED_PEAKS.json hbm_gbs: 1 Gi bf16 copy)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback (earlier copy measurement on this pool)"


# The source files of each kernel (and the device headers they include) whose bytes key a committed ncu
# summary to the code it measured.  internal.h (host-side declarations and launch helpers) is left out.
KERNEL_SOURCES = {
    "decode_step": ("decode_step.cu", "decode_common.cuh", "common.cuh", "state_tile.cuh"),
    "update_window": ("update_window.cu", "common.cuh", "state_tile.cuh"),
    "update_window_tc": ("update_window_tc.cu", "common.cuh"),
    # every kernel of a sketch window and of a full-read window (with the tensor-core update: window_tc)
    "window": ("decode_step.cu", "decode_common.cuh", "update_window.cu", "fullread.cu", "common.cuh",
               "state_tile.cuh"),
    "window_tc": ("decode_step.cu", "decode_common.cuh", "update_window_tc.cu", "fullread.cu", "common.cuh",
                  "state_tile.cuh"),
}


def csrc_hash(kernel=None):
    """sha256 (16 hex digits) of a kernel's source files, or of every file under csrc/."""
    h = hashlib.sha256()
    d = os.path.join(ROOT, "recurrent_state_read_b200", "csrc")
    names = KERNEL_SOURCES[kernel] if kernel else sorted(os.listdir(d))
    for fn in names:
        with open(os.path.join(d, fn), "rb") as f:
            h.update(fn.encode() + f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel_tag, cfg):
    """DRAM bytes per launch from a committed ncu summary of the same kernel source, else None."""
    p = os.path.join(ROOT, "profiles", f"{kernel_tag}.txt")
    if not os.path.exists(p):
        return None
    kv = {}
    with open(p) as f:
        for line in f:
            if ":" in line and not line.startswith(" "):
                k, v = line.split(":", 1)
                kv[k.strip()] = v.strip()
    kernel = ("decode_step" if kernel_tag.startswith("decode_step")
              else "update_window_tc" if tc_update(cfg) else "update_window")
    if (kv.get("csrc_sha256") or "").split()[:1] != [csrc_hash(kernel)] or kv.get("workload_key") != workload_key(cfg):
        return None
    try:
        return float(kv["dram_bytes_per_launch_full_size"])
    except (KeyError, ValueError):
        return None


def workload_key(cfg):
    return f"{cfg.kind}-B{cfg.B}-H{cfg.H}-dk{cfg.dk}-dv{cfg.dv}-r{cfg.r}-W{cfg.W}-{cfg.qkv_dtype}-{cfg.state_dtype}"


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples every 200 ms while the bench runs; summarised over the timed regions."""
    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid=None):
        self.uuid = (uuid or "").lower().replace("gpu-", "")
        self.marks = []
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        self.t_start = time.time()

    def mark(self, on: bool):
        self.marks.append((time.time(), on))

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for line in out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            if self.uuid and self.uuid not in parts[0].lower():
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        pmax = max(r[2] for r in rows)
        loaded = [r for r in rows if r[2] > 0.35 * pmax] or rows
        reasons = sorted({n for r in loaded for n, v in zip(names, r[3]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max(r[1] for r in rows),
                "samples": len(rows), "samples_under_load": len(loaded), "power_w_max": pmax,
                "reasons": reasons}


# ---------------------------------------------------------------- CPU oracle
class OracleSample:
    """A bounded sample of the workload for the fp64 CPU oracle: `chunk` heads (whole sequences'
    worth of heads where they fit) with one window of seeded decode tokens.  One step runs the
    oracle's sketch path on it: sketch refresh, W sketch reads, window update."""

    def __init__(self, cfg, seed=0):
        import numpy as np

        import oracle
        import workloads as wl

        oracle.build()
        self.cfg = cfg
        H = cfg.H
        self.chunk = max(1, min(cfg.n_heads, 256 if cfg.dk * cfg.dv > 4096 else 1024))
        nb = max(1, -(-self.chunk // H))
        tok = wl.token_block(cfg, "decode", 0, cfg.W, device="cpu", B=nb, with_query=True)
        avail = nb * H
        self.chunk = min(self.chunk, avail)
        self.ft = {k: (None if v is None else
                       v.reshape(cfg.W, avail, *v.shape[3:])[:, :self.chunk].double().numpy())
                   for k, v in tok.items()}
        rng = np.random.default_rng(seed)
        self.U = rng.standard_normal((self.chunk, cfg.dk, cfg.r)) / np.sqrt(cfg.dk)
        self.R = rng.standard_normal((self.chunk, cfg.r, cfg.dk)) / np.sqrt(cfg.dk)
        self.S0 = rng.standard_normal((self.chunk, cfg.dk, cfg.dv))
        self.threads = oracle.num_threads()

    def step(self):
        import oracle

        oracle.sketch_path(self.cfg.kind, self.S0, self.U, self.R, self.ft, self.cfg.W,
                           bf16_state=self.cfg.state_dtype == "bf16")
        return (self.chunk / self.cfg.H) * self.cfg.W  # token-steps done

    def step_full(self):
        """The oracle's full-read path on the same sample: every token updates and reads the state."""
        import oracle

        oracle.fullread_path(self.cfg.kind, self.S0, self.ft, bf16_state=self.cfg.state_dtype == "bf16")
        return (self.chunk / self.cfg.H) * self.cfg.W

    def describe(self, n_steps, seconds):
        return (f"{n_steps} x (oracle sketch path, fp64: sketch refresh, {self.cfg.W} sketch reads, window "
                f"update) on {self.chunk} heads ({self.chunk / self.cfg.H:.2f} sequences x {self.cfg.H} heads) "
                f"of the workload, {seconds:.1f} s")


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform

    return platform.processor() or "unknown"


def _rate(fn, seconds: float):
    done, n = 0.0, 0
    t0 = time.perf_counter()
    while True:
        done += fn()
        n += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            return done / el, n, el


def cpu_oracle_rate(cfg, seconds: float):
    """The fp64 oracle on the host: its sketch path on all OpenMP threads (the reported value), its
    full-read path on the same sample, and the sketch path on one thread.  About half of `seconds`
    goes to the first, a quarter to each of the others."""
    import oracle

    smp = OracleSample(cfg)
    rate, n, el = _rate(smp.step, 0.5 * seconds)
    full, nf, elf = _rate(smp.step_full, 0.25 * seconds)
    oracle.set_num_threads(1)
    try:
        one, n1, el1 = _rate(smp.step, 0.25 * seconds)
    finally:
        oracle.set_num_threads(smp.threads)
    desc = (smp.describe(n, el) + f"; full-read path: {nf} x the same sample's {cfg.W} exact steps, {elf:.1f} s; "
            f"one thread: {n1} sketch-path steps, {el1:.1f} s")
    return {"value": rate, "unit": UNIT, "cores": smp.threads, "kind": "oracle", "sample": desc,
            "fullread_value": full, "single_thread_value": one, "cpu_model": cpu_model()}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    cfg = workload_of(args)
    smp = OracleSample(cfg)
    for _ in range(args.warmup):
        smp.step()
    done = 0.0
    t0 = time.perf_counter()
    for _ in range(args.steps):
        done += smp.step()
    elapsed = time.perf_counter() - t0
    value = done / elapsed
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "impl": "reference", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * elapsed / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_json(cfg),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": smp.threads, "kind": "oracle",
                         "sample": smp.describe(args.steps, elapsed)},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- multi-rank plumbing
def reduce_max(x: float, device=None) -> float:
    """Max of x over all ranks (identity without an initialised process group).

    With NCCL the value travels in a CUDA tensor on `device`; with gloo on the CPU."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, t_max: float) -> float:
    """Replicas: every rank processes the same units; the job's rate is all units over the slowest rank."""
    return world * units_per_rank / t_max


# ---------------------------------------------------------------- GPU arm: shared pieces
def dims_of(cfg, B=None, r=None):
    import recurrent_state_read_b200 as rs

    return rs.dims(cfg.kind, cfg.B if B is None else B, cfg.H, cfg.dk, cfg.dv, cfg.r if r is None else r, cfg.W,
                   cfg.torch_state_dtype, cfg.torch_qkv_dtype)


def prefill_state(cfg, dev, B=None):
    """The start state: cfg.prefill tokens through the library's window update, from S = 0."""
    import torch

    import workloads as wl
    from recurrent_state_read_b200.decode import prefill

    B = cfg.B if B is None else B
    d = dims_of(cfg, B=B)
    S0 = torch.zeros(B, cfg.H, cfg.dv, cfg.dk, dtype=cfg.torch_state_dtype, device=dev)
    P = torch.empty(B, cfg.H, cfg.dv, cfg.r, device=dev)
    U0 = torch.zeros(cfg.H, cfg.r, cfg.dk, device=dev)
    prefill(d, S0, P, U0, lambda t0, n: wl.token_block(cfg, "prefill", t0, n, device=dev, B=B), cfg.prefill)
    return S0


def calibration_states(cfg, dev):
    """Final prefill states of the cfg.n_cal_seq calibration sequences (the "cal" token stream)."""
    import torch

    import workloads as wl
    from recurrent_state_read_b200.decode import prefill

    dc = dims_of(cfg, B=cfg.n_cal_seq)
    S_cal = torch.zeros(cfg.n_cal_seq, cfg.H, cfg.dv, cfg.dk, dtype=cfg.torch_state_dtype, device=dev)
    P = torch.empty(cfg.n_cal_seq, cfg.H, cfg.dv, cfg.r, device=dev)
    U0 = torch.zeros(cfg.H, cfg.r, cfg.dk, device=dev)
    prefill(dc, S_cal, P, U0, lambda t0, n: wl.token_block(cfg, "cal", t0, n, device=dev), cfg.prefill)
    return S_cal


def calibrate(cfg, S_cal, q_cal, dev, r=None):
    """Basis rows U and coefficient map R [H, r, dk] from the library's offline calibration."""
    import torch

    import recurrent_state_read_b200 as rs

    r = cfg.r if r is None else r
    dc = dims_of(cfg, B=cfg.n_cal_seq, r=r)
    U = torch.empty(cfg.H, r, cfg.dk, device=dev)
    R = torch.empty(cfg.H, r, cfg.dk, device=dev)
    rs.sketchssm_calibrate_basis(dc, q_cal, S_cal, U, R)
    return U, R


def decode_windows(cfg, dev, B=None):
    """NWIN distinct windows of decode tokens: window buffers and the time-major token planes."""
    import workloads as wl
    from recurrent_state_read_b200.decode import WindowBuffer

    B = cfg.B if B is None else B
    d = dims_of(cfg, B=B)
    bufs, toks = [], []
    for i in range(NWIN):
        tok = wl.token_block(cfg, "decode", i * cfg.W, cfg.W, device=dev, B=B, with_query=True)
        tok = {k: (None if v is None else v.contiguous()) for k, v in tok.items()}
        b = WindowBuffer.empty(d, device=dev)
        b.fill(tok)
        bufs.append(b)
        toks.append(tok)
    return bufs, toks


def capture_graph(fn, stream):
    """fn's launches as a CUDA graph (one eager call first, outside capture, warms the launch path)."""
    import torch

    g = torch.cuda.CUDAGraph()
    fn()
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=stream):
        fn()
    return g


def timed_windows(parts, steps, warmup, stream, clocks, barrier):
    """Replay, per step i, the graphs parts[0][i % NWIN], parts[1][i % NWIN], ... in order, with CUDA
    events on the launching stream around each.  Returns (seconds over all steps, [seconds per part])."""
    import torch

    for i in range(warmup):
        for p in parts:
            p[i % NWIN].replay()
    barrier()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(parts) + 1)] for _ in range(steps)]
    clocks.mark(True)
    for i in range(steps):
        evs[i][0].record(stream)
        for k, p in enumerate(parts):
            p[i % NWIN].replay()
            evs[i][k + 1].record(stream)
    barrier()
    clocks.mark(False)
    total = evs[0][0].elapsed_time(evs[-1][-1]) / 1e3
    per = [sum(e[k].elapsed_time(e[k + 1]) for e in evs) / 1e3 for k in range(len(parts))]
    return total, per


def kernel_entry(bytes_, seconds, launches, peak):
    ms = 1e3 * seconds / launches
    gbps = bytes_ / ms / 1e6
    return {"us_per_launch": 1e3 * ms, "algorithmic_bytes": bytes_, "GBps": gbps, "frac_of_peak": gbps / peak,
            "nominal_8TBps_frac": gbps / 8000.0}


def measured_gate(cfg, speedup):
    """The speed target on measured DRAM bytes: the sketch path must beat the full-read path by at
    least 0.8 x (full-read DRAM bytes / sketch DRAM bytes per token-step), both from one committed
    ncu capture of each path's whole window (all kernels) whose kernel sources match these."""
    p = os.path.join(ROOT, "profiles", f"traffic_gate_{cfg.kind}.txt")
    if not os.path.exists(p):
        return None
    kv = {}
    with open(p) as f:
        for line in f:
            if ":" in line and not line.startswith(" "):
                k, v = line.split(":", 1)
                kv[k.strip()] = v.strip()
    srcs = "window_tc" if tc_update(cfg) else "window"
    if (kv.get("csrc_sha256") or "").split()[:1] != [csrc_hash(srcs)] or kv.get("workload_key") != workload_key(cfg):
        return None
    try:
        full = float(kv["fullread_dram_bytes_per_token_step"])
        sk = float(kv["sketch_dram_bytes_per_token_step"])
    except (KeyError, ValueError):
        return None
    ratio = full / sk
    return {"fullread_dram_bytes_per_token_step": full, "sketch_dram_bytes_per_token_step": sk,
            "measured_bytes_ratio": ratio, "bar": 0.8 * ratio, "speedup": speedup, "met": speedup >= 0.8 * ratio,
            "source": os.path.relpath(p, ROOT)}


def approx_error(d, S, P, U, R, buf, tok, dev):
    """Relative L2 error of the sketch path's outputs against the exact read on one window."""
    import torch

    from recurrent_state_read_b200.decode import fullread_window, sketch_window

    W = d.W
    out = torch.empty(W, d.B, d.H, d.dv, device=dev)
    out_f = torch.empty_like(out)
    S_a, Sf_a, P_a = S.clone(), S.clone(), P.clone()
    sketch_window(d, S_a, P_a, U, R, buf, out)
    fullread_window(d, Sf_a, tok, out_f)
    torch.cuda.synchronize()
    return float(torch.linalg.vector_norm((out - out_f).double()) / torch.linalg.vector_norm(out_f.double()))


def basis_ablation(cfg, d, S, P, U, R, q_cal, bufs, toks, stream, clocks, barrier, steps, warmup, weighted):
    """The sketch path with the query-PCA basis (sketchssm_calibrate_query_pca: top-r query directions,
    no state weighting) beside the state-weighted basis: approximation error on the first window and
    the sketch window's throughput with each.  `weighted` holds the state-weighted basis's figures."""
    import torch

    import recurrent_state_read_b200 as rs

    dc = dims_of(cfg, B=1)
    Up, Rp = torch.empty_like(U), torch.empty_like(R)
    rs.sketchssm_calibrate_query_pca(dc, q_cal, Up, Rp)
    Sp, Pp = S.clone(), torch.empty_like(P)
    rs.sketchssm_update_window(d, Sp, Pp, Up, None, None, None, None, 0)
    approx = approx_error(d, Sp, Pp, Up, Rp, bufs[0], toks[0], S.device)
    W = cfg.W
    out = torch.empty(W, cfg.B, cfg.H, cfg.dv, device=S.device)
    g_dec = [capture_graph(lambda b=b: [rs.sketchssm_decode_step(d, Pp, Rp, b.q[j - 1], b.k, b.v, b.alpha, b.beta,
                                                                 j, out[j - 1]) for j in range(1, W + 1)], stream)
             for b in bufs]
    g_upd = [capture_graph(lambda b=b: rs.sketchssm_update_window(d, Sp, Pp, Up, b.k, b.v, b.alpha, b.beta, W),
                           stream) for b in bufs]
    t_s, _ = timed_windows([g_dec, g_upd], steps, warmup, stream, clocks, barrier)
    del g_dec, g_upd, Sp, Pp
    return {"rank": cfg.r, "state_weighted": weighted,
            "query_pca": {"approx_rel_l2_first_window": approx, "value": steps * cfg.B * W / t_s, "unit": UNIT,
                          "steps": steps},
            "note": "query PCA: U = R^T = the top-r eigenvectors of the calibration queries' second moment "
                    "(sketchssm_calibrate_query_pca); same kernels and traffic, only the basis differs"}


def tc_update(cfg):
    """Whether sketchssm_update_window runs this workload's windows on the tensor cores (Gated DeltaNet,
    dk = dv = 128, fp32 state, bf16 q/k/v, r <= 16, 12 <= W <= 16 tokens per window)."""
    return (cfg.kind == "gdn" and cfg.dk == 128 and cfg.dv == 128 and cfg.state_dtype == "f32"
            and cfg.qkv_dtype == "bf16" and cfg.r <= 16 and 12 <= cfg.W <= 16)


def measure_workload(cfg, dev, stream, clocks, barrier, steps, warmup, peak):
    """One workload's sketch path (decode steps + window update), full-read path and ReplaySSM-style
    path, each over the same NWIN windows, with per-kernel rooflines, the traffic ratios and the
    sketch's approximation error on the first window."""
    import torch

    import recurrent_state_read_b200 as rs
    import workloads as wl
    from recurrent_state_read_b200.decode import fullread_window

    d = dims_of(cfg)
    bm = bytes_model(cfg)
    S0 = prefill_state(cfg, dev)
    S_cal = calibration_states(cfg, dev)
    q_cal = wl.calibration_queries(cfg, device=dev)
    U, R = calibrate(cfg, S_cal, q_cal, dev)
    del S_cal
    bufs, toks = decode_windows(cfg, dev)
    W = cfg.W
    S = S0.clone()
    P = torch.empty(cfg.B, cfg.H, cfg.dv, cfg.r, device=dev)
    rs.sketchssm_update_window(d, S, P, U, None, None, None, None, 0)
    approx = approx_error(d, S, P, U, R, bufs[0], toks[0], dev)
    out = torch.empty(W, cfg.B, cfg.H, cfg.dv, device=dev)
    Sf, Sr = S0.clone(), S0.clone()
    g_dec = [capture_graph(lambda b=b: [rs.sketchssm_decode_step(d, P, R, b.q[j - 1], b.k, b.v, b.alpha, b.beta, j,
                                                                 out[j - 1]) for j in range(1, W + 1)], stream)
             for b in bufs]
    g_upd = [capture_graph(lambda b=b: rs.sketchssm_update_window(d, S, P, U, b.k, b.v, b.alpha, b.beta, W), stream)
             for b in bufs]
    g_full = [capture_graph(lambda t=t: fullread_window(d, Sf, t, out), stream) for t in toks]
    g_rdec = [capture_graph(lambda b=b: [rs.sketchssm_replay_decode_step(d, Sr, b.q[j - 1], b.k, b.v, b.alpha,
                                                                         b.beta, j, out[j - 1])
                                         for j in range(1, W + 1)], stream) for b in bufs]
    g_rupd = [capture_graph(lambda b=b: rs.sketchssm_update_window(d, Sr, None, None, b.k, b.v, b.alpha, b.beta, W),
                            stream) for b in bufs]
    t_s, (t_dec, t_upd) = timed_windows([g_dec, g_upd], steps, warmup, stream, clocks, barrier)
    t_f, _ = timed_windows([g_full], steps, warmup, stream, clocks, barrier)
    t_r, _ = timed_windows([g_rdec, g_rupd], steps, warmup, stream, clocks, barrier)
    del g_dec, g_upd, g_full, g_rdec, g_rupd
    tok_steps = steps * cfg.B * W
    kernels = {"update_window": kernel_entry(bm["update"], t_upd, steps, peak),
               "decode_step": kernel_entry(bm["decode_avg"], t_dec, steps * W, peak),
               "fullread_decode": kernel_entry(bm["fullread"], t_f, steps * W, peak)}
    if tc_update(cfg):
        kernels["update_window"]["path"] = ("tensor cores: chunked form, S_0^T [K; U] and the rank-n increment "
                                            "on tcgen05 (kind::tf32, split operands)")
    elif cfg.kind == "kda" and cfg.r <= 8 and cfg.state_dtype == "f32" and cfg.qkv_dtype == "bf16" and W <= 16:
        # the tensor-core form of the KDA update, an explicit alternative (not the default), same windows
        St, Pt = S.clone(), P.clone()
        g_tc = [capture_graph(lambda b=b: rs.sketchssm_update_window_tc(d, St, Pt, U, b.k, b.v, b.alpha, b.beta, W),
                              stream) for b in bufs]
        t_tc, _ = timed_windows([g_tc], steps, warmup, stream, clocks, barrier)
        del g_tc, St, Pt
        kernels["update_window_tc"] = kernel_entry(bm["update"], t_tc, steps, peak)
        kernels["update_window_tc"]["note"] = ("sketchssm_update_window_tc for KDA: chunked form on tcgen05 with "
                                               "split decayed keys (not the default: slower than update_window)")
    dominant = "update_window" if t_upd >= t_dec else "decode_step"
    value, value_f = tok_steps / t_s, tok_steps / t_f
    speedup = value / value_f
    exact_last = None
    if cfg.kind != "mamba2":  # W-1 sketch steps + the update with the fused exact read of step W
        from recurrent_state_read_b200.decode import sketch_window
        Sx, Px = S.clone(), P.clone()
        outx = torch.empty(W, cfg.B, cfg.H, cfg.dv, device=dev)
        g_x = [capture_graph(lambda b=b: sketch_window(d, Sx, Px, U, R, b, outx, exact_last=True), stream) for b in bufs]
        t_x, _ = timed_windows([g_x], max(3, steps // 3), warmup, stream, clocks, barrier)
        del g_x
        # its approximation error on the first window, from the window-start state of the sketch path
        Sa, Pa, Sf1 = S.clone(), P.clone(), S.clone()
        rs.sketchssm_update_window(d, Sa, Pa, U, None, None, None, None, 0)
        out_f1 = torch.empty_like(outx)
        sketch_window(d, Sa, Pa, U, R, bufs[0], outx, exact_last=True)
        fullread_window(d, Sf1, toks[0], out_f1)
        torch.cuda.synchronize()
        approx_x = float(torch.linalg.vector_norm((outx - out_f1).double()) / torch.linalg.vector_norm(out_f1.double()))
        exact_last = {"value": max(3, steps // 3) * cfg.B * W / t_x, "unit": UNIT,
                      "ms_per_step": 1e3 * t_x / max(3, steps // 3),
                      "schedule": f"{W - 1} sketch decode steps + 1 window update that also reads step {W} exactly",
                      "approx_rel_l2_first_window": approx_x}
        del Sx, Px, Sa, Pa, Sf1, outx, out_f1
    ablation = None
    if cfg.r == 8:
        ablation = basis_ablation(cfg, d, S, P, U, R, q_cal, bufs, toks, stream, clocks, barrier,
                                  max(3, steps // 3), warmup,
                                  {"approx_rel_l2_first_window": approx, "value": value, "unit": UNIT})
    state_ratio = (2 * W * bm["S"]) / (2 * bm["S"] + (W + 1) * bm["P"])
    return {
        "workload": config_json(cfg)["workload"], "value": value, "unit": UNIT, "steps": steps, "warmup": warmup,
        "ms_per_step": 1e3 * t_s / steps, "kernels": kernels,
        "roofline": {"bound": "hbm", "kernel": dominant, "achieved": kernels[dominant]["GBps"], "peak": peak,
                     "unit": "GB/s", "frac": kernels[dominant]["frac_of_peak"],
                     "nominal_8TBps_frac": kernels[dominant]["nominal_8TBps_frac"]},
        "sketch_window_GBps": bm["sketch_step"] / (t_s / steps) / 1e9,
        "fullread": {"value": value_f, "unit": UNIT, "ms_per_step": 1e3 * t_f / steps},
        "replay": {"value": tok_steps / t_r, "unit": UNIT, "ms_per_step": 1e3 * t_r / steps},
        "sketch_vs_fullread": {
            "speedup": speedup,
            "algorithmic_bytes_per_token_step": {"sketch": bm["sketch_step"] / (cfg.B * W),
                                                 "fullread": bm["full_step"] / (cfg.B * W)},
            "algorithmic_bytes_ratio": bm["full_step"] / bm["sketch_step"],
            "state_bytes_ratio": state_ratio,
            "gate_on_state_bytes": {"bar": 0.8 * state_ratio, "met": speedup >= 0.8 * state_ratio},
            "gate_on_measured_bytes": measured_gate(cfg, speedup),
            "approx_rel_l2_first_window": approx},
        **({"exact_last_step": exact_last} if exact_last else {}),
        **({"basis_ablation": ablation} if ablation else {}),
    }


SWEEP_B = (64, 256, 1024)
SWEEP_R = (4, 8, 16, 32)
SWEEP_W = (4, 8, 16, 32)
SWEEP_DT = ("f32", "bf16")


def run_sweep(dev, stream, clocks, barrier, steps, warmup, peak):
    """The GDN sweep on the sketch path: B x r x W x state dtype (96 points), and the full-read path
    per (B, state dtype).  Per (W, dtype) the calibration states are prefilled once and calibrated
    at each r; per (B, W, dtype) the start state is prefilled once and timed at each r."""
    import torch

    import recurrent_state_read_b200 as rs
    import workloads as wl
    from recurrent_state_read_b200.decode import fullread_window

    points, fulls = [], []
    for sdt in SWEEP_DT:
        for W in SWEEP_W:
            base = wl.workload(4, W=W, state_dtype=sdt)
            S_cal = calibration_states(base, dev)
            q_cal = wl.calibration_queries(base, device=dev)
            bases = {r: calibrate(base, S_cal, q_cal, dev, r=r) for r in SWEEP_R}
            del S_cal
            for B in SWEEP_B:
                cfgB = wl.workload(4, B=B, W=W, state_dtype=sdt)
                S0 = prefill_state(cfgB, dev)
                bufs, toks = decode_windows(cfgB, dev)
                out = torch.empty(W, B, cfgB.H, cfgB.dv, device=dev)
                for r in SWEEP_R:
                    cfg = wl.workload(4, B=B, W=W, r=r, state_dtype=sdt)
                    d = dims_of(cfg)
                    bm = bytes_model(cfg)
                    U, R = bases[r]
                    S = S0.clone()
                    P = torch.empty(B, cfg.H, cfg.dv, r, device=dev)
                    rs.sketchssm_update_window(d, S, P, U, None, None, None, None, 0)
                    g_dec = [capture_graph(lambda b=b: [rs.sketchssm_decode_step(d, P, R, b.q[j - 1], b.k, b.v,
                                                                                 b.alpha, b.beta, j, out[j - 1])
                                                        for j in range(1, W + 1)], stream) for b in bufs]
                    g_upd = [capture_graph(lambda b=b: rs.sketchssm_update_window(d, S, P, U, b.k, b.v, b.alpha,
                                                                                  b.beta, W), stream) for b in bufs]
                    t_s, (t_dec, t_upd) = timed_windows([g_dec, g_upd], steps, warmup, stream, clocks, barrier)
                    del g_dec, g_upd, S, P
                    upd = kernel_entry(bm["update"], t_upd, steps, peak)
                    dec = kernel_entry(bm["decode_avg"], t_dec, steps * W, peak)
                    win_gbps = bm["sketch_step"] / (t_s / steps) / 1e9
                    points.append({
                        "B": B, "r": r, "W": W, "state": sdt, "value": steps * B * W / t_s,
                        "ms_per_step": 1e3 * t_s / steps,
                        "bytes_per_token_step": bm["sketch_step"] / (B * W),
                        "window_GBps": win_gbps, "window_frac": win_gbps / peak,
                        "update_us": upd["us_per_launch"], "update_GBps": upd["GBps"], "update_frac": upd["frac_of_peak"],
                        "decode_us": dec["us_per_launch"], "decode_GBps": dec["GBps"], "decode_frac": dec["frac_of_peak"],
                        "update_path": "tensor cores" if tc_update(cfg) else "cuda cores"})
                if W == 16:  # the full-read path does not depend on W or r
                    d = dims_of(cfgB)
                    bm = bytes_model(cfgB)
                    Sf = S0.clone()
                    g_full = [capture_graph(lambda t=t: fullread_window(d, Sf, t, out), stream) for t in toks]
                    t_f, _ = timed_windows([g_full], steps, warmup, stream, clocks, barrier)
                    del g_full, Sf
                    fk = kernel_entry(bm["fullread"], t_f, steps * W, peak)
                    fulls.append({"B": B, "state": sdt, "value": steps * B * W / t_f,
                                  "bytes_per_token_step": bm["full_step"] / (B * W),
                                  "us_per_step": fk["us_per_launch"], "GBps": fk["GBps"], "frac": fk["frac_of_peak"]})
                del S0, bufs, toks, out
                torch.cuda.empty_cache()
    for p in points:  # speed-up over the full-read path of the same batch and state dtype
        f = next(x for x in fulls if x["B"] == p["B"] and x["state"] == p["state"])
        p["speedup_vs_fullread"] = p["value"] / f["value"]
    return {"workload": "GDN sweep: H=32 dk=dv=128, q/k/v bf16; B x r x W x state dtype",
            "axes": {"B": list(SWEEP_B), "r": list(SWEEP_R), "W": list(SWEEP_W), "state": list(SWEEP_DT)},
            "steps_per_point": steps, "warmup_per_point": warmup, "unit": UNIT, "peak_GBps": peak,
            "points": points, "fullread": fulls}


# ---------------------------------------------------------------- GPU arm
def run_ours(args):
    import torch
    import torch.distributed as dist

    import recurrent_state_read_b200 as rs
    import workloads as wl
    from recurrent_state_read_b200.decode import WindowBuffer, prefill

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    rs.library()
    cfg = workload_of(args)
    d = rs.dims(cfg.kind, cfg.B, cfg.H, cfg.dk, cfg.dv, cfg.r, cfg.W, cfg.torch_state_dtype, cfg.torch_qkv_dtype)
    bm = bytes_model(cfg)
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.set_stream(stream)

    # start state: prefill through the library's window update
    S0 = torch.zeros(cfg.B, cfg.H, cfg.dv, cfg.dk, dtype=cfg.torch_state_dtype, device=dev)
    P = torch.empty(cfg.B, cfg.H, cfg.dv, cfg.r, device=dev)
    U0 = torch.zeros(cfg.H, cfg.r, cfg.dk, device=dev)
    prefill(d, S0, P, U0, lambda t0, n: wl.token_block(cfg, "prefill", t0, n, device=dev), cfg.prefill)
    # offline basis: the library's calibration on prefilled calibration sequences
    dc = rs.dims(cfg.kind, cfg.n_cal_seq, cfg.H, cfg.dk, cfg.dv, cfg.r, cfg.W, cfg.torch_state_dtype,
                 cfg.torch_qkv_dtype)
    S_cal = torch.zeros(cfg.n_cal_seq, cfg.H, cfg.dv, cfg.dk, dtype=cfg.torch_state_dtype, device=dev)
    P_cal = torch.empty(cfg.n_cal_seq, cfg.H, cfg.dv, cfg.r, device=dev)
    prefill(dc, S_cal, P_cal, U0, lambda t0, n: wl.token_block(cfg, "cal", t0, n, device=dev), cfg.prefill)
    q_cal = wl.calibration_queries(cfg, device=dev)
    U = torch.empty(cfg.H, cfg.r, cfg.dk, device=dev)  # basis rows
    R = torch.empty(cfg.H, cfg.r, cfg.dk, device=dev)
    rs.sketchssm_calibrate_basis(dc, q_cal, S_cal, U, R)
    if args.rank_avg:  # the same calibration data, ranks per head under an average-rank budget
        Uk = torch.empty_like(U)
        Rk = torch.empty_like(R)
        head_rank = torch.empty(cfg.H, dtype=torch.int32, device=dev)
        lam = torch.empty(cfg.H, cfg.r, dtype=torch.float64, device=dev)
        rs.sketchssm_calibrate_basis_ranked(dc, q_cal, S_cal, args.rank_avg, Uk, Rk, head_rank, lam)
    del S_cal, P_cal

    # NWIN distinct windows of decode tokens
    bufs, toks = [], []
    for i in range(NWIN):
        tok = wl.token_block(cfg, "decode", i * cfg.W, cfg.W, device=dev, with_query=True)  # time-major
        tok = {k: (None if v is None else v.contiguous()) for k, v in tok.items()}
        b = WindowBuffer.empty(d, device=dev)
        b.fill(tok)
        bufs.append(b)
        toks.append(tok)  # the full-read baseline reads one token plane per step
    out = torch.empty(cfg.W, cfg.B, cfg.H, cfg.dv, device=dev)
    out_f = torch.empty_like(out)
    S = S0.clone()
    Sf = S0.clone()
    rs.sketchssm_update_window(d, S, P, U, None, None, None, None, 0)
    torch.cuda.synchronize()

    # approximation error of the sketch against the exact read on the first window (information)
    from recurrent_state_read_b200.decode import fullread_window, sketch_window

    S_a, Sf_a, P_a = S.clone(), S.clone(), P.clone()
    sketch_window(d, S_a, P_a, U, R, bufs[0], out)
    fullread_window(d, Sf_a, toks[0], out_f)
    torch.cuda.synchronize()
    approx = float(torch.linalg.vector_norm((out - out_f).double()) / torch.linalg.vector_norm(out_f.double()))
    if args.rank_avg:
        S_k, P_k = S.clone(), torch.empty_like(P)
        rs.sketchssm_update_window_ranked(d, S_k, P_k, Uk, head_rank, None, None, None, None, 0)
        b0 = bufs[0]
        for j in range(1, cfg.W + 1):
            rs.sketchssm_decode_step_ranked(d, P_k, Rk, head_rank, b0.q[j - 1], b0.k, b0.v, b0.alpha, b0.beta, j,
                                            out[j - 1])
        torch.cuda.synchronize()
        approx_k = float(torch.linalg.vector_norm((out - out_f).double()) /
                         torch.linalg.vector_norm(out_f.double()))
        del S_k
    S_a, P_a = S.clone(), P.clone()
    sketch_window(d, S_a, P_a, U, R, bufs[0], out, exact_last=True)
    torch.cuda.synchronize()
    approx_x = float(torch.linalg.vector_norm((out - out_f).double()) / torch.linalg.vector_norm(out_f.double()))
    del S_a, Sf_a, P_a

    # CUDA graphs: per window buffer, the decode steps (sketch path) and the full-read steps
    def capture(fn):
        g = torch.cuda.CUDAGraph()
        fn()  # warm the launch path outside capture
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=stream):
            fn()
        return g

    def dec_fn(b):
        return lambda: [rs.sketchssm_decode_step(d, P, R, b.q[j - 1], b.k, b.v, b.alpha, b.beta, j, out[j - 1])
                        for j in range(1, cfg.W + 1)]

    def upd_fn(b):
        return lambda: rs.sketchssm_update_window(d, S, P, U, b.k, b.v, b.alpha, b.beta, cfg.W)

    def full_fn(tok):
        return lambda: fullread_window(d, Sf, tok, out_f)

    g_dec = [capture(dec_fn(b)) for b in bufs]
    g_upd = [capture(upd_fn(b)) for b in bufs]
    g_full = [capture(full_fn(tok)) for tok in toks]
    # the variant whose last step of each window is read exactly inside the window update
    g_x = [capture(lambda b=b: sketch_window(d, S, P, U, R, b, out, exact_last=True)) for b in bufs]
    # the staggered schedule: sequence b's windows run with a phase of b mod W steps; at every step the
    # sequences inside a window take a sketch step while those whose window ends are updated and read
    # exactly, on a second stream (W steps per graph = every sequence through one whole window)
    from recurrent_state_read_b200.decode import stagger_plan, staggered_step
    plan = stagger_plan(cfg.B, cfg.W, dev)
    share = tuple(int(x) for x in args.stagger_share.split(","))
    side = torch.cuda.Stream(device=dev)
    Sg, Pg = S.clone(), P.clone()

    def stagger_cycle(b):
        def fn():
            for st in range(cfg.W):
                fork = torch.cuda.Event()
                fork.record(stream)
                side.wait_event(fork)
                staggered_step(d, Sg, Pg, U, R, b, b.q[st], plan[st], out[st], share,
                               (stream.cuda_stream, side.cuda_stream))
                join = torch.cuda.Event()
                join.record(side)
                stream.wait_event(join)
        return fn

    g_st = [capture(stagger_cycle(b)) for b in bufs]
    g_wy = None
    if cfg.kind != "mamba2" and cfg.W <= 32:  # the delta rules' decode step in WY form
        Sw, Pw = S.clone(), P.clone()
        Gw = rs.wy_gram_buffer(d, dev)

        def wy_window(b):
            def fn():
                for j in range(1, cfg.W + 1):
                    rs.sketchssm_decode_step_wy(d, Pw, R, b.q[j - 1], b.k, b.v, b.alpha, b.beta, j, Gw, out[j - 1])
                rs.sketchssm_update_window(d, Sw, Pw, U, b.k, b.v, b.alpha, b.beta, cfg.W)
            return fn

        g_wy = [capture(wy_window(b)) for b in bufs]
    if args.rank_avg:  # the sketch path with a rank per head
        Sk = S.clone()
        Pk = torch.empty_like(P)
        rs.sketchssm_update_window_ranked(d, Sk, Pk, Uk, head_rank, None, None, None, None, 0)

        def ranked_window(b):
            def fn():
                for j in range(1, cfg.W + 1):
                    rs.sketchssm_decode_step_ranked(d, Pk, Rk, head_rank, b.q[j - 1], b.k, b.v, b.alpha, b.beta, j,
                                                    out[j - 1])
                rs.sketchssm_update_window_ranked(d, Sk, Pk, Uk, head_rank, b.k, b.v, b.alpha, b.beta, cfg.W)
            return fn

        g_rk = [capture(ranked_window(b)) for b in bufs]
    # the ReplaySSM-style baseline: W full-state reads of the window-start state + one update (no sketch)
    Sr = S0.clone()
    g_rdec = [capture(lambda b=b: [rs.sketchssm_replay_decode_step(d, Sr, b.q[j - 1], b.k, b.v, b.alpha, b.beta,
                                                                   j, out_f[j - 1]) for j in range(1, cfg.W + 1)])
              for b in bufs]
    g_rupd = [capture(lambda b=b: rs.sketchssm_update_window(d, Sr, None, None, b.k, b.v, b.alpha, b.beta, cfg.W))
              for b in bufs]

    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    clocks = ClockSampler(uuid)
    time.sleep(0.3)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def max_over_ranks(x):
        return reduce_max(x, dev)

    def ev():
        return torch.cuda.Event(enable_timing=True)

    # --- sketch path
    for i in range(args.warmup):
        g_dec[i % NWIN].replay()
        g_upd[i % NWIN].replay()
    barrier()
    evs = [(ev(), ev(), ev()) for _ in range(args.steps)]
    clocks.mark(True)
    for i in range(args.steps):
        e0, e1, e2 = evs[i]
        e0.record(stream)
        g_dec[i % NWIN].replay()
        e1.record(stream)
        g_upd[i % NWIN].replay()
        e2.record(stream)
    barrier()
    clocks.mark(False)
    t_sketch = evs[0][0].elapsed_time(evs[-1][2]) / 1e3
    t_dec = sum(e[0].elapsed_time(e[1]) for e in evs) / 1e3
    t_upd = sum(e[1].elapsed_time(e[2]) for e in evs) / 1e3
    t_sketch = max_over_ranks(t_sketch)

    # --- full-read baseline (same windows)
    for i in range(args.warmup):
        g_full[i % NWIN].replay()
    barrier()
    fe = [(ev(), ev()) for _ in range(args.steps)]
    clocks.mark(True)
    for i in range(args.steps):
        fe[i][0].record(stream)
        g_full[i % NWIN].replay()
        fe[i][1].record(stream)
    barrier()
    clocks.mark(False)
    t_full = max_over_ranks(fe[0][0].elapsed_time(fe[-1][1]) / 1e3)

    # --- sketch path with the exact last step fused into the window update
    for i in range(args.warmup):
        g_x[i % NWIN].replay()
    barrier()
    xe0, xe1 = ev(), ev()
    clocks.mark(True)
    xe0.record(stream)
    for i in range(args.steps):
        g_x[i % NWIN].replay()
    xe1.record(stream)
    barrier()
    clocks.mark(False)
    t_x = max_over_ranks(xe0.elapsed_time(xe1) / 1e3)

    # --- staggered schedule
    for i in range(args.warmup):
        g_st[i % NWIN].replay()
    barrier()
    se0, se1 = ev(), ev()
    clocks.mark(True)
    se0.record(stream)
    for i in range(args.steps):
        g_st[i % NWIN].replay()
    se1.record(stream)
    barrier()
    clocks.mark(False)
    t_st = max_over_ranks(se0.elapsed_time(se1) / 1e3)

    # --- rank per head
    t_rk = None
    if args.rank_avg:
        for i in range(args.warmup):
            g_rk[i % NWIN].replay()
        barrier()
        ke0, ke1 = ev(), ev()
        clocks.mark(True)
        ke0.record(stream)
        for i in range(args.steps):
            g_rk[i % NWIN].replay()
        ke1.record(stream)
        barrier()
        clocks.mark(False)
        t_rk = max_over_ranks(ke0.elapsed_time(ke1) / 1e3)

    # --- decode steps in WY form
    t_wy = None
    if g_wy is not None:
        for i in range(args.warmup):
            g_wy[i % NWIN].replay()
        barrier()
        we0, we1 = ev(), ev()
        clocks.mark(True)
        we0.record(stream)
        for i in range(args.steps):
            g_wy[i % NWIN].replay()
        we1.record(stream)
        barrier()
        clocks.mark(False)
        t_wy = max_over_ranks(we0.elapsed_time(we1) / 1e3)

    # --- ReplaySSM-style baseline
    for i in range(args.warmup):
        g_rdec[i % NWIN].replay()
        g_rupd[i % NWIN].replay()
    barrier()
    re_ = [(ev(), ev(), ev()) for _ in range(args.steps)]
    clocks.mark(True)
    for i in range(args.steps):
        re_[i][0].record(stream)
        g_rdec[i % NWIN].replay()
        re_[i][1].record(stream)
        g_rupd[i % NWIN].replay()
        re_[i][2].record(stream)
    barrier()
    clocks.mark(False)
    t_r = max_over_ranks(re_[0][0].elapsed_time(re_[-1][2]) / 1e3)
    t_rdec = sum(e[0].elapsed_time(e[1]) for e in re_) / 1e3

    # --- end to end: window inputs from pinned host memory, outputs back to host.  As a serving
    # loop would run it: the next window's inputs are copied in and the previous window's outputs
    # copied out on two copy streams while the current window computes (NWIN input buffers, two
    # output buffers; events order every reuse).
    e2e = None
    if not args.no_e2e:
        names = ("k", "v", "alpha", "beta", "q")
        host = []
        for b in bufs:
            host.append({n: getattr(b, n).cpu().pin_memory() for n in names if getattr(b, n) is not None})
        outs = [out, torch.empty_like(out)]
        out_h = [torch.empty(out.shape, dtype=out.dtype, pin_memory=True) for _ in range(2)]
        h2d = sum(t.numel() * t.element_size() for t in host[0].values())
        d2h = out.numel() * out.element_size()

        def dec_into(b, o):
            return lambda: [rs.sketchssm_decode_step(d, P, R, b.q[j - 1], b.k, b.v, b.alpha, b.beta, j, o[j - 1])
                            for j in range(1, cfg.W + 1)]

        g_dec_e = [capture(dec_into(bufs[i], outs[i % 2])) for i in range(NWIN)]
        up_s, down_s = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        h2d_ev = [torch.cuda.Event() for _ in range(NWIN)]
        comp_ev = [torch.cuda.Event() for _ in range(NWIN)]
        d2h_ev = [torch.cuda.Event() for _ in range(2)]

        def copy_in(i):
            b = i % NWIN
            up_s.wait_event(comp_ev[b])  # the buffer's previous window has been computed
            with torch.cuda.stream(up_s):
                for n, t in host[b].items():
                    getattr(bufs[b], n).copy_(t, non_blocking=True)
            h2d_ev[b].record(up_s)

        def compute(i):
            b, o = i % NWIN, i % 2
            stream.wait_event(h2d_ev[b])
            stream.wait_event(d2h_ev[o])  # the output buffer has been copied out
            g_dec_e[b].replay()
            g_upd[b].replay()
            comp_ev[b].record(stream)

        def copy_out(i):
            b, o = i % NWIN, i % 2
            down_s.wait_event(comp_ev[b])
            with torch.cuda.stream(down_s):
                out_h[o].copy_(outs[o], non_blocking=True)
            d2h_ev[o].record(down_s)

        def run_e2e(n, start=None):
            if start is not None:
                up_s.wait_event(start)
                down_s.wait_event(start)
            copy_in(0)
            for i in range(n):
                compute(i)
                if i + 1 < n:
                    copy_in(i + 1)
                copy_out(i)
            stream.wait_event(d2h_ev[(n - 1) % 2])

        run_e2e(min(args.warmup, 3))
        barrier()
        ee0, ee1 = ev(), ev()
        clocks.mark(True)
        ee0.record(stream)
        run_e2e(args.steps, ee0)
        ee1.record(stream)
        barrier()
        clocks.mark(False)
        t_e2e = max_over_ranks(ee0.elapsed_time(ee1) / 1e3)
        e2e = {"value": whole_job_rate(args.steps * cfg.B * cfg.W, world, t_e2e), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": 1e3 * t_e2e / args.steps,
               "pcie_GBps": (h2d + d2h) / (t_e2e / args.steps) / 1e9,
               "path": "python binding -> C ABI; every window's inputs copied in from pinned host memory and "
                       "its outputs copied out, inside the timed region, overlapped with the neighbouring "
                       "windows' compute on two copy streams (bound by the host link, not the kernels)"}
        del g_dec_e
    peak, peak_src = hbm_peak()

    # the other workloads and the GDN sweep (single GPU only; the scaling runs time the headline)
    extra = {}
    if world == 1 and not args.no_workloads:
        del g_st
        g_st = None
        extra["basis_ablation"] = basis_ablation(
            cfg, d, S, P, U, R, q_cal, bufs, toks, stream, clocks, barrier, max(3, args.workload_steps // 3), 3,
            {"approx_rel_l2_first_window": approx,
             "value": whole_job_rate(args.steps * cfg.B * cfg.W, world, t_sketch), "unit": UNIT})
        torch.cuda.empty_cache()
        extra["workloads"] = {}
        for name, wcfg in (("gdn", wl.workload(2)), ("kda_r4", wl.workload(3, r=4)), ("kda_r8", wl.workload(3, r=8)),
                           ("kda_r16", wl.workload(3, r=16))):
            extra["workloads"][name] = measure_workload(wcfg, dev, stream, clocks, barrier, args.workload_steps, 3, peak)
            torch.cuda.empty_cache()
    if world == 1 and not args.no_sweep:
        extra["sweep"] = run_sweep(dev, stream, clocks, barrier, args.sweep_steps, 3, peak)
        torch.cuda.empty_cache()
    clk = clocks.stop()

    tok_per_step = cfg.B * cfg.W
    value = whole_job_rate(args.steps * tok_per_step, world, t_sketch)
    value_full = whole_job_rate(args.steps * tok_per_step, world, t_full)
    upd_ms = 1e3 * t_upd / args.steps
    dec_ms = 1e3 * t_dec / (args.steps * cfg.W)
    full_ms = 1e3 * t_full / (args.steps * cfg.W)
    kernels = {
        "update_window": {"ms_per_launch": upd_ms, "algorithmic_bytes": bm["update"],
                          "GBps": bm["update"] / upd_ms / 1e6},
        "decode_step": {"ms_per_launch": dec_ms, "algorithmic_bytes": bm["decode_avg"],
                        "GBps": bm["decode_avg"] / dec_ms / 1e6},
        "fullread_decode": {"ms_per_launch": full_ms, "algorithmic_bytes": bm["fullread"],
                            "GBps": bm["fullread"] / full_ms / 1e6},
    }
    for k in kernels.values():
        k["frac_of_peak"] = k["GBps"] / peak
        k["nominal_8TBps_frac"] = k["GBps"] / 8000.0
    state_ratio = (2 * cfg.W * bm["S"]) / (2 * bm["S"] + (cfg.W + 1) * bm["P"])
    dominant = "update_window" if t_upd >= t_dec else "decode_step"
    kd = kernels[dominant]
    traffic = profiled_traffic(f"{dominant}_{cfg.kind}", cfg)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * t_sketch / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": config_json(cfg),
        "roofline": {"bound": "hbm", "kernel": dominant, "achieved": kd["GBps"], "peak": peak, "unit": "GB/s",
                     "frac": kd["GBps"] / peak, "traffic": traffic, "peak_source": peak_src,
                     "nominal_8TBps_frac": kd["GBps"] / 8000.0},
        "kernels": kernels,
        "fullread": {"value": value_full, "unit": UNIT, "ms_per_step": 1e3 * t_full / args.steps},
        "replay": {
            "value": whole_job_rate(args.steps * tok_per_step, world, t_r), "unit": UNIT,
            "ms_per_step": 1e3 * t_r / args.steps,
            "schedule": f"{cfg.W} decode steps that read the full window-start state + 1 window update "
                        "(no sketch): the ReplaySSM-style buffered baseline",
            "replay_step_GBps": bm["replay_avg"] / (1e3 * t_rdec / (args.steps * cfg.W)) / 1e6,
            "algorithmic_bytes_per_token_step": bm["replay_step"] / tok_per_step,
            "sketch_speedup": value / whole_job_rate(args.steps * tok_per_step, world, t_r)},
        **({"ranked": {
            "value": whole_job_rate(args.steps * tok_per_step, world, t_rk), "unit": UNIT,
            "ms_per_step": 1e3 * t_rk / args.steps, "r_avg": args.rank_avg, "r_max": cfg.r,
            "ranks": head_rank.cpu().tolist(),
            "schedule": "the sketch path with a rank per head (sketchssm_calibrate_basis_ranked, "
                        "*_ranked kernels), same windows",
            "approx_rel_l2_first_window": approx_k}} if args.rank_avg else {}),
        **({"wy_decode": {
            "value": whole_job_rate(args.steps * tok_per_step, world, t_wy), "unit": UNIT,
            "ms_per_step": 1e3 * t_wy / args.steps,
            "schedule": "the sketch path with the decode steps' backward pass in WY form "
                        "(sketchssm_decode_step_wy, per-head Gram buffer)"}} if t_wy is not None else {}),
        "staggered": {
            "value": whole_job_rate(args.steps * tok_per_step, world, t_st), "unit": UNIT,
            "ms_per_step": 1e3 * t_st / args.steps,
            "schedule": f"sequence b's windows offset by b mod {cfg.W} steps; per decode step the sequences "
                        f"inside a window take a sketch step (per-sequence step index) while about B/W "
                        f"sequences end their window: update + exact read, concurrently on a second stream; "
                        f"one step of this key = {cfg.W} decode steps = every sequence through one window",
            "ctas_per_sm": {"decode": share[0], "update": share[1]}},
        "exact_last_step": {
            "value": whole_job_rate(args.steps * tok_per_step, world, t_x), "unit": UNIT,
            "ms_per_step": 1e3 * t_x / args.steps,
            "schedule": f"{cfg.W - 1} sketch decode steps + 1 window update that also reads step {cfg.W} exactly",
            "approx_rel_l2_first_window": approx_x},
        "sketch_vs_fullread": {
            "speedup": value / value_full,
            "algorithmic_bytes_per_token_step": {"sketch": bm["sketch_step"] / tok_per_step,
                                                 "fullread": bm["full_step"] / tok_per_step},
            "algorithmic_bytes_ratio": bm["full_step"] / bm["sketch_step"],
            "state_bytes_ratio": state_ratio,
            "gate_on_state_bytes": {"bar": 0.8 * state_ratio, "met": value / value_full >= 0.8 * state_ratio},
            "gate_on_measured_bytes": measured_gate(cfg, value / value_full),
            "approx_rel_l2_first_window": approx,
        },
        "gpu_launches": args.steps * (cfg.W + 1),
        "clocks": clk,
    }
    if e2e is not None:
        line["e2e"] = e2e
    line.update(extra)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_oracle_rate(cfg, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    del g_dec, g_upd, g_full, g_x, g_rdec, g_rupd, g_st, g_wy
    if args.rank_avg:
        del g_rk
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
