"""Host-side logic of bench.py (CPU): the tensor-core dispatch predicate, the algorithmic byte model,
and the reading of committed ncu summaries (a summary counts only for the kernel sources and the
workload it was taken on)."""

import os

import pytest

import bench
import workloads as wl


def test_tc_update_predicate():
    assert bench.tc_update(wl.CONFIGS[2])                       # GDN, r = 8, W = 16, fp32 state
    assert bench.tc_update(wl.workload(4, r=16, W=12))
    assert not bench.tc_update(wl.CONFIGS[1])                   # Mamba-2
    assert not bench.tc_update(wl.CONFIGS[3])                   # KDA stays on the CUDA cores
    assert not bench.tc_update(wl.workload(4, W=8))             # too few tokens per window
    assert not bench.tc_update(wl.workload(4, W=32))            # more than 16 tokens
    assert not bench.tc_update(wl.workload(4, r=32))
    assert not bench.tc_update(wl.workload(4, state_dtype="bf16"))


def test_byte_model_closed_forms():
    cfg = wl.CONFIGS[2]  # GDN B=256 H=32 dk=dv=128 r=8 W=16, bf16 tokens, fp32 state
    bm = bench.bytes_model(cfg)
    NH = cfg.B * cfg.H
    assert bm["S"] == NH * 128 * 128 * 4
    assert bm["P"] == NH * 128 * 8 * 4
    assert bm["full_step"] == cfg.W * bm["fullread"]
    assert bm["sketch_step"] == bm["update"] + sum(bm["decode"])
    # decode step j reads j buffered tokens: the per-step bytes grow by one token slot per step
    steps = bm["decode"]
    assert len(steps) == cfg.W
    assert len({round(b - a) for a, b in zip(steps, steps[1:])}) == 1
    # state-only traffic ratio at r = 8, W = 16: 2 W S / (2 S + (W + 1) P)
    ratio = (2 * cfg.W * bm["S"]) / (2 * bm["S"] + (cfg.W + 1) * bm["P"])
    assert ratio == pytest.approx(10.449, rel=1e-3)


def _root(tmp_path, monkeypatch):
    """A bench root with its own profiles folder and the real kernel sources (for the hashes)."""
    (tmp_path / "profiles").mkdir()
    (tmp_path / "recurrent_state_read_b200").mkdir()
    (tmp_path / "recurrent_state_read_b200" / "csrc").symlink_to(
        os.path.join(os.path.dirname(os.path.abspath(bench.__file__)), "recurrent_state_read_b200", "csrc"))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))


def _summary(tmp_path, name, text):
    (tmp_path / "profiles" / name).write_text(text)


def test_measured_gate_reads_matching_summary_only(tmp_path, monkeypatch):
    cfg = wl.CONFIGS[1]
    _root(tmp_path, monkeypatch)
    body = ("kernel: whole windows\n"
            f"csrc_sha256: {bench.csrc_hash('window')}   (sources)\n"
            f"workload_key: {bench.workload_key(cfg)}\n"
            "sketch_dram_bytes_per_token_step: 1000\n"
            "fullread_dram_bytes_per_token_step: 6000\n")
    _summary(tmp_path, "traffic_gate_mamba2.txt", body)
    g = bench.measured_gate(cfg, 5.0)
    assert g["measured_bytes_ratio"] == pytest.approx(6.0)
    assert g["bar"] == pytest.approx(4.8) and g["met"]
    assert not bench.measured_gate(cfg, 4.0)["met"]
    # another workload or other kernel sources: the summary does not apply
    assert bench.measured_gate(wl.workload(1, B=128), 5.0) is None
    _summary(tmp_path, "traffic_gate_mamba2.txt", body.replace(bench.csrc_hash("window"), "0" * 16))
    assert bench.measured_gate(cfg, 5.0) is None


def test_profiled_traffic_keys_on_the_dispatched_kernel(tmp_path, monkeypatch):
    cfg = wl.CONFIGS[2]  # the GDN update runs on the tensor cores: keyed on that kernel's sources
    _root(tmp_path, monkeypatch)
    for key, expect in (("update_window_tc", 123.0), ("update_window", None)):
        _summary(tmp_path, "update_window_gdn.txt",
                 f"csrc_sha256: {bench.csrc_hash(key)}\nworkload_key: {bench.workload_key(cfg)}\n"
                 "dram_bytes_per_launch_full_size: 123\n")
        assert bench.profiled_traffic("update_window_gdn", cfg) == expect
