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
    assert declared_functions() == ["carve_bwd", "carve_bwd_noalloc", "carve_bwd_varlen", "carve_bwd_workspace_bytes",
                                    "carve_check", "carve_fwd", "carve_fwd_varlen", "carve_saved_bytes",
                                    "carve_selftest_stall", "carve_selftest_timeout", "carve_status_string",
                                    "carve_step"]


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
    assert carve.bwd_workspace_bytes(d) == 4 * units * (128 * 8 + 8 * 64 + 8 + 128 + 1)
    for bad in (dict(dk=96), dict(T=100), dict(chunk=48), dict(rank=65), dict(io=3), dict(mc_mode=2), dict(B=0),
                dict(T=0)):
        assert carve.saved_bytes(good_dims(**bad)) == 0, bad
        assert carve.bwd_workspace_bytes(good_dims(**bad)) == 0, bad


@pytest.mark.parametrize("bad,code", [(dict(dk=96), 2), (dict(dv=32), 2), (dict(T=100), 2), (dict(chunk=48), 2),
                                      (dict(rank=65), 2), (dict(io=7), 1), (dict(mc_mode=5), 1), (dict(H=0), 1),
                                      (dict(T=0), 1), (dict(chunk=1, mc_mode=1), 2),
                                      (dict(B=1 << 20, H=1, T=1 << 11, dk=64, dv=64), 2)])
def test_bad_dims_rejected(lib, bad, code):
    """Dimension checks run first, so the (fake) pointers below are never dereferenced."""
    d = good_dims(**bad)
    P = ctypes.c_void_p(4096)
    assert lib.carve_fwd(ctypes.byref(d), *fwd_args(P)) == code
    assert lib.carve_bwd(ctypes.byref(d), *bwd_args(P)) == code
    if "T" not in bad and "chunk" not in bad:       # decode ignores T and (in mode 0) chunk
        assert lib.carve_step(ctypes.byref(d), *step_args(P)) == code


# Valid argument lists (P: a 16-byte aligned placeholder; None where a pointer is optional).
# fwd: 8 inputs 0-7, Aw 8, A_dec 9, tau 10, S0 11, m_prev_in 12, o 13, S_final 14,
#      m_prev_out 15, saved 16, stream 17
def fwd_args(P):
    return [P] * 8 + [None] * 5 + [P, None, None, None, None]


# bwd: 8 inputs 0-7, Aw 8, A_dec 9, tau 10, S0 11, m_prev_in 12, saved 13, dO 14, dS_final 15,
#      dm_prev_out 16, dq..dB 17-24, dAw 25, dA_dec 26, dtau 27, dS0 28, dm_prev_in 29,
#      workspace 30, stream 31
def bwd_args(P):
    return [P] * 8 + [None] * 5 + [P, P, None, None] + [P] * 8 + [None] * 5 + [P, None]


# step: 8 inputs 0-7, Aw 8, A_dec 9, tau 10, S 11, mstate 12, pos 13, o 14, stream 15
def step_args(P):
    return [P] * 8 + [None] * 3 + [P, None, None, P, None]


def test_null_and_misaligned_pointers_rejected(lib):
    """Every call below has valid dims and exactly one bad pointer, so it must be rejected on
    the host with CARVE_ERR_INVALID_ARG before any launch."""
    d = good_dims()
    P = ctypes.c_void_p(4096)
    fwd_ok = fwd_args(P)
    for j in (0, 1, 2, 3, 4, 5, 6, 7, 13):              # each required forward pointer
        args = list(fwd_ok)
        args[j] = None
        assert lib.carve_fwd(ctypes.byref(d), *args) == 1, j
        args[j] = ctypes.c_void_p(4100)                 # misaligned
        assert lib.carve_fwd(ctypes.byref(d), *args) == 1, j
    for j in (8, 9, 10, 11, 12, 14, 15, 16):            # optional pointers: misaligned is rejected
        args = list(fwd_ok)
        args[j] = ctypes.c_void_p(4104)
        assert lib.carve_fwd(ctypes.byref(d), *args) == 1, j
    bwd_ok = bwd_args(P)
    for j in (13, 14, 17, 18, 19, 20, 21, 22, 23, 24, 30):
        args = list(bwd_ok)
        args[j] = None
        assert lib.carve_bwd(ctypes.byref(d), *args) == 1, j
    for x, dx in ((8, 25), (9, 26), (10, 27)):          # Aw / A_dec / tau and their gradients come in pairs
        args = list(bwd_ok)
        args[x] = P
        assert lib.carve_bwd(ctypes.byref(d), *args) == 1, (x, "without its gradient")
        args = list(bwd_ok)
        args[dx] = P
        assert lib.carve_bwd(ctypes.byref(d), *args) == 1, (dx, "without its parameter")
    ds = good_dims(mc_mode=1)
    assert lib.carve_step(ctypes.byref(ds), *step_args(P)) == 1   # needs mstate, pos
    args = step_args(P)
    args[11] = None                                     # S missing
    assert lib.carve_step(ctypes.byref(d), *args) == 1
    for j in (8, 9, 10):                                # misaligned Aw, A_dec, tau
        args = step_args(P)
        args[j] = ctypes.c_void_p(4104)
        assert lib.carve_step(ctypes.byref(d), *args) == 1, j
    assert lib.carve_fwd(None, *fwd_ok) == 1


def test_selftest_timeout_bounds_checked_on_host(lib):
    """Out-of-range poll counts are rejected before any launch (and arm nothing)."""
    assert lib.carve_selftest_timeout(0, None) == 1
    assert lib.carve_selftest_timeout(1_000_001, None) == 1
    assert lib.carve_selftest_stall(0) == 1
    assert lib.carve_selftest_stall(1_000_001) == 1


def test_varlen_arguments_checked_on_host(lib):
    """carve_fwd_varlen / carve_bwd_varlen: a missing or misaligned cu_seqlens and an
    out-of-range row count are rejected before any launch (the placeholder pointers are never
    used)."""
    P = ctypes.c_void_p(4096)
    d = good_dims()
    for cu, total, code in ((None, 64, 1), (ctypes.c_void_p(4100), 64, 1), (P, -1, 1), (P, 1 << 40, 1)):
        assert lib.carve_fwd_varlen(ctypes.byref(d), cu, total, *fwd_args(P)) == code, (cu, total)
        assert lib.carve_bwd_varlen(ctypes.byref(d), cu, total, *bwd_args(P)) == code, (cu, total)
    exact = good_dims(chunk=1)   # the exact recurrence has no packed form
    assert lib.carve_fwd_varlen(ctypes.byref(exact), P, 64, *fwd_args(P)) == 2
    assert lib.carve_bwd_varlen(ctypes.byref(exact), P, 64, *bwd_args(P)) == 2
