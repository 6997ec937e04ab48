"""The C ABI without a GPU: the library loads, exports every entry point its
header declares, and rejects invalid arguments on the host before any CUDA
call (every case below fails validation, so nothing is launched)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def rs():
    import recurrent_state_read_b200 as rs
    from recurrent_state_read_b200 import build

    build.build()
    return rs


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(sketchssm_\w+)\s*\(", src))
    return names


def test_exports_every_declared_symbol(rs):
    lib = rs.library()
    declared = _declared()
    assert {"sketchssm_update_window", "sketchssm_decode_step", "sketchssm_fullread_decode",
            "sketchssm_calibrate_basis"} <= declared
    for name in sorted(declared):
        assert hasattr(lib, name), name
    assert set(rs.EXPORTS) <= declared


def test_status_strings_and_version(rs):
    lib = rs.library()
    assert lib.sketchssm_status_string(0) == b"ok"
    for code in range(-7, 0):
        assert lib.sketchssm_status_string(code) != b"unknown status"
    assert lib.sketchssm_version() >= 10000


def _d(rs, **kw):
    base = dict(kind="gdn", B=2, H=3, dk=128, dv=128, r=8, W=16)
    base.update(kw)
    return rs.dims(**base)


FAKE = ctypes.c_void_p(1 << 20)  # never dereferenced: every call below fails validation first


@pytest.mark.parametrize("kw,code", [
    (dict(dk=96), -2), (dict(dv=32), -2), (dict(r=0), -2), (dict(r=33), -2), (dict(W=0), -2),
    (dict(W=65), -2), (dict(kind=3), -2), (dict(B=0), -2), (dict(H=0), -2),
])
def test_update_window_rejects_dims(rs, kw, code):
    lib = rs.library()
    d = _d(rs, **kw) if "kind" not in kw else _d(rs)
    if "kind" in kw:
        d.kind = kw["kind"]
    rc = lib.sketchssm_update_window(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, None)
    assert rc == code


def test_validation_codes(rs):
    lib = rs.library()
    d = _d(rs)
    uw = lib.sketchssm_update_window
    assert uw(None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, None) == -1
    assert uw(ctypes.byref(d), None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, None) == -1
    assert uw(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 17, None) == -3
    assert uw(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, -1, None) == -3
    assert uw(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 4, None) == -1  # GDN needs beta
    odd = ctypes.c_void_p((1 << 20) + 4)
    assert uw(ctypes.byref(d), odd, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, None) == -4
    bad = _d(rs)
    bad.state_dtype = 7
    assert uw(ctypes.byref(bad), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, None) == -5
    ur = lib.sketchssm_update_window_read
    assert ur(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, None, FAKE, None) == -1  # q
    assert ur(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, FAKE, None, None) == -1  # o
    assert ur(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 17, FAKE, FAKE, None) == -3
    assert ur(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, odd, FAKE, None) == -4
    assert ur(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, FAKE, odd, None) == -4
    assert ur(ctypes.byref(bad), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, FAKE, FAKE, None) == -5
    ds = lib.sketchssm_decode_step
    assert ds(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, FAKE, None) == -3
    assert ds(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 17, FAKE, None) == -3
    assert ds(ctypes.byref(d), FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE, 3, FAKE, None) == -1
    assert lib.sketchssm_selftest_wait_giveup(0, None) == -3
    assert lib.sketchssm_selftest_wait_giveup((1 << 20) + 1, None) == -3
    rp = lib.sketchssm_replay_decode_step
    assert rp(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, FAKE, None) == -3
    assert rp(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 17, FAKE, None) == -3
    assert rp(ctypes.byref(d), None, FAKE, FAKE, FAKE, FAKE, FAKE, 3, FAKE, None) == -1
    assert rp(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, None, 3, FAKE, None) == -1  # GDN needs beta
    assert rp(ctypes.byref(d), FAKE, odd, FAKE, FAKE, FAKE, FAKE, 3, FAKE, None) == -4
    assert uw(ctypes.byref(d), FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE, 4, None) == -1  # P without U
    fr = lib.sketchssm_fullread_decode
    assert fr(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, None) == -1
    assert fr(ctypes.byref(d), FAKE, FAKE, odd, FAKE, FAKE, FAKE, FAKE, None) == -4
    m = _d(rs, kind="mamba2")
    assert fr(ctypes.byref(m), None, FAKE, FAKE, FAKE, FAKE, None, FAKE, None) == -1
    cb = lib.sketchssm_calibrate_basis
    need = lib.sketchssm_calibrate_workspace_bytes(ctypes.byref(d), 100, 10)
    assert need == 3 * d.H * d.dk * d.dk * 8
    assert lib.sketchssm_calibrate_workspace_bytes(ctypes.byref(d), 0, 10) == 0
    assert cb(ctypes.byref(d), FAKE, 100, FAKE, 10, 1e-8, FAKE, FAKE, FAKE, need - 1, None) == -7
    assert cb(ctypes.byref(d), FAKE, 0, FAKE, 10, 1e-8, FAKE, FAKE, FAKE, need, None) == -3
    assert cb(ctypes.byref(d), FAKE, 100, FAKE, 10, -1.0, FAKE, FAKE, FAKE, need, None) == -3
    assert cb(ctypes.byref(d), FAKE, 100, FAKE, 10, 1e-8, FAKE, FAKE, None, need, None) == -7
