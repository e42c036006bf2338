"""The C-ABI library loads on a CPU-only host, exports every entry point include/carve.h
declares, and rejects malformed calls on the host before any launch (no GPU needed: every
call below fails validation, so no CUDA call is made)."""
import ctypes
import os
import re

import pytest

import chunk_gated_delta_b200 as carve
from chunk_gated_delta_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return carve.load()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "carve.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(carve_[a-z_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    assert declared_functions() == ["carve_bwd", "carve_bwd_noalloc", "carve_bwd_workspace_bytes", "carve_check",
                                    "carve_fwd", "carve_saved_bytes", "carve_selftest_timeout",
                                    "carve_status_string", "carve_step"]


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    out = os.popen(f"nm -D --defined-only {carve.library_path()}").read()
    for name in declared_functions():
        assert re.search(rf"\bT {name}\b", out), name


def test_status_strings(lib):
    for code, name in carve.STATUS.items():
        assert lib.carve_status_string(code).decode() == name


def good_dims(**kw):
    d = dict(B=2, H=3, T=128, dk=128, dv=64, rank=8, chunk=64, io=1, mc_mode=0)
    d.update(kw)
    return carve.Dims(**d)


def test_buffer_sizes(lib):
    d = good_dims()
    units = 2 * 3
    states = units * (128 // 16) * 64 * 128
    aux = units * 2 * (64 + 8 + 128)
    assert carve.saved_bytes(d) == 4 * (states + aux)
    assert carve.bwd_workspace_bytes(d) == 4 * units * (128 * 8 + 8 * 64 + 8)
    for bad in (dict(dk=96), dict(T=100), dict(chunk=48), dict(rank=65), dict(io=3), dict(mc_mode=2), dict(B=0),
                dict(T=0)):
        assert carve.saved_bytes(good_dims(**bad)) == 0, bad
        assert carve.bwd_workspace_bytes(good_dims(**bad)) == 0, bad


@pytest.mark.parametrize("bad,code", [(dict(dk=96), 2), (dict(dv=32), 2), (dict(T=100), 2), (dict(chunk=48), 2),
                                      (dict(rank=65), 2), (dict(io=7), 1), (dict(mc_mode=5), 1), (dict(H=0), 1),
                                      (dict(T=0), 1)])
def test_bad_dims_rejected(lib, bad, code):
    """Dimension checks run first, so the (fake) pointers below are never dereferenced."""
    d = good_dims(**bad)
    P = ctypes.c_void_p(4096)
    assert lib.carve_fwd(ctypes.byref(d), *([P] * 8), None, None, None, P, None, None, None, None) == code
    assert lib.carve_bwd(ctypes.byref(d), *([P] * 8), None, None, None, P, P, None, None, *([P] * 8), None, None,
                         None, P, None) == code
    if "T" not in bad and "chunk" not in bad:       # decode ignores T and (in mode 0) chunk
        assert lib.carve_step(ctypes.byref(d), *([P] * 8), None, P, None, None, P, None) == code


def test_null_and_misaligned_pointers_rejected(lib):
    """Every call below has valid dims and exactly one bad pointer, so it must be rejected on
    the host with CARVE_ERR_INVALID_ARG before any launch."""
    d = good_dims()
    P = ctypes.c_void_p(4096)
    fwd_ok = [P] * 8 + [None, None, None, P, None, None, None, None]
    for j in (0, 1, 2, 3, 4, 5, 6, 7, 11):              # each required forward pointer
        args = list(fwd_ok)
        args[j] = None
        assert lib.carve_fwd(ctypes.byref(d), *args) == 1, j
        args[j] = ctypes.c_void_p(4100)                 # misaligned
        assert lib.carve_fwd(ctypes.byref(d), *args) == 1, j
    for j in (8, 9, 10, 12, 13, 14):                    # optional pointers: misaligned is rejected
        args = list(fwd_ok)
        args[j] = ctypes.c_void_p(4104)
        assert lib.carve_fwd(ctypes.byref(d), *args) == 1, j
    # bwd: 8 inputs, Aw 8, S0 9, m_prev_in 10, saved 11, dO 12, dS_final 13, dm_prev_out 14,
    #      dq..dB 15-22, dAw 23, dS0 24, dm_prev_in 25, workspace 26, stream 27
    bwd_ok = [P] * 8 + [None, None, None, P, P, None, None] + [P] * 8 + [None, None, None, P, None]
    for j in (11, 12, 15, 16, 17, 18, 19, 20, 21, 22, 26):
        args = list(bwd_ok)
        args[j] = None
        assert lib.carve_bwd(ctypes.byref(d), *args) == 1, j
    args = list(bwd_ok)
    args[8] = P                                         # Aw without dAw
    assert lib.carve_bwd(ctypes.byref(d), *args) == 1
    args = list(bwd_ok)
    args[23] = P                                        # dAw without Aw
    assert lib.carve_bwd(ctypes.byref(d), *args) == 1
    ds = good_dims(mc_mode=1)
    assert lib.carve_step(ctypes.byref(ds), *([P] * 8), None, P, None, None, P, None) == 1   # needs mstate, pos
    assert lib.carve_step(ctypes.byref(d), *([P] * 8), None, None, None, None, P, None) == 1  # S missing
    assert lib.carve_step(ctypes.byref(d), *([P] * 8), ctypes.c_void_p(4104), P, None, None, P, None) == 1
    assert lib.carve_fwd(None, *fwd_ok) == 1


def test_selftest_timeout_bounds_checked_on_host(lib):
    """Out-of-range poll counts are rejected before any launch."""
    assert lib.carve_selftest_timeout(0, None) == 1
    assert lib.carve_selftest_timeout(1_000_001, None) == 1
