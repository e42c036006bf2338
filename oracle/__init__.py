"""CARVE fp64 reference oracle -- TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the benchmark's CPU-baseline / reference leg may import
this package.  The CUDA product path never imports it and shares no code with it.

`fwd`, `bwd` and `step` call the plain token-sequential C implementation in
`carve_oracle.c` (fp64, OpenMP over independent (batch, head) units).  `wy` holds a second,
independent fp64 restatement in chunked WY form, written in numpy.

Parity pins: see tests/test_oracle_pins.py and tests/test_oracle_wy.py.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "carve_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


class _Dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("B", "H", "T", "K", "V", "R", "L", "mc_mode", "content_off")]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain IEEE fp64: no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-shared",
                        "-fPIC", "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


def bind(path: str):
    """Load a compiled oracle library and declare its entry points."""
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    lib.orc_fwd.argtypes = [ctypes.POINTER(_Dims)] + [P] * 17
    lib.orc_bwd.argtypes = [ctypes.POINTER(_Dims)] + [P] * 30
    lib.orc_step.argtypes = [ctypes.POINTER(_Dims)] + [P] * 15
    for f in (lib.orc_fwd, lib.orc_bwd, lib.orc_step):
        f.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = bind(_LIB)
    return _lib


def _f64(x):
    if x is None:
        return None
    return np.ascontiguousarray(x, dtype=np.float64)


def _p(x):
    return None if x is None else x.ctypes.data_as(ctypes.c_void_p)


def _dims(inp, L, mc_mode, content_off, cu=None):
    B, T, H, K = inp["q"].shape
    V = inp["v"].shape[-1]
    R = inp["A"].shape[-1]
    if cu is not None:   # packed sequences: [1, T, H, *] tensors, len(cu) - 1 sequences
        assert B == 1, "packed sequences use a leading dimension of 1"
        B = len(cu) - 1
    return _Dims(B, H, T, K, V, R, L, mc_mode, int(content_off))


def _cu(cu_seqlens):
    return None if cu_seqlens is None else np.ascontiguousarray(cu_seqlens, dtype=np.int32)


_KEYS = ("q", "k", "v", "g_logit", "bx", "w_logit", "A", "B")


def fwd(inp: dict, L: int, mc_mode: int = 0, S0=None, m_prev=None, content_off: bool = False, cu_seqlens=None):
    """Forward over [B,T,H,*] inputs.  Optional entries: inp["Aw"] [H,R], the write gate's
    content term; inp["A_dec"] [H] and inp["tau"] [H,K], the decay's log-amplitude and bias.
    cu_seqlens ([N+1] ints): N sequences packed along the token axis of [1,T,H,*] inputs;
    S0, m_prev and the per-sequence outputs are then [N,H,...].
    Returns dict(o, S_final, m_prev_out) in fp64."""
    lib = _load()
    cu = _cu(cu_seqlens)
    d = _dims(inp, L, mc_mode, content_off, cu)
    a = [_f64(inp[k]) for k in _KEYS]
    Aw, S0, m_prev = _f64(inp.get("Aw")), _f64(S0), _f64(m_prev)
    A_dec, tau = _f64(inp.get("A_dec")), _f64(inp.get("tau"))
    o = np.zeros((1 if cu is not None else d.B, d.T, d.H, d.V))
    S = np.zeros((d.B, d.H, d.V, d.K))
    m = np.zeros((d.B, d.H, d.V))
    rc = lib.orc_fwd(ctypes.byref(d), *[_p(x) for x in a], _p(Aw), _p(A_dec), _p(tau), _p(S0), _p(m_prev), _p(o),
                     _p(S), _p(m), _p(cu))
    if rc:
        raise ValueError("oracle fwd: bad dims")
    return dict(o=o, S_final=S, m_prev_out=m)


def bwd(inp: dict, L: int, dO, mc_mode: int = 0, S0=None, m_prev=None, dS_final=None,
        dm_prev_out=None, content_off: bool = False, cu_seqlens=None):
    """Gradients of sum(dO*o) + sum(dS_final*S_final) + sum(dm_prev_out*m_prev_out).
    Returns dict(dq, dk, dv, dg_logit, dbx, dw_logit, dA, dB, dAw, dA_dec, dtau, dS0,
    dm_prev_in) in fp64 (dAw, dA_dec, dtau are zero when inp lacks "Aw", "A_dec", "tau")."""
    lib = _load()
    cu = _cu(cu_seqlens)
    d = _dims(inp, L, mc_mode, content_off, cu)
    a = [_f64(inp[k]) for k in _KEYS]
    Aw, A_dec, tau = _f64(inp.get("Aw")), _f64(inp.get("A_dec")), _f64(inp.get("tau"))
    S0, m_prev, dO = _f64(S0), _f64(m_prev), _f64(dO)
    dS_final, dm_prev_out = _f64(dS_final), _f64(dm_prev_out)
    B, T, H, K, V, R = d.B, d.T, d.H, d.K, d.V, d.R
    Bt = 1 if cu is not None else B   # leading dimension of the token tensors
    out = dict(dq=np.zeros((Bt, T, H, K)), dk=np.zeros((Bt, T, H, K)), dv=np.zeros((Bt, T, H, V)),
               dg_logit=np.zeros((Bt, T, H, K)), dbx=np.zeros((Bt, T, H, K)), dw_logit=np.zeros((Bt, T, H)),
               dA=np.zeros((H, K, R)), dB=np.zeros((H, R, V)), dAw=np.zeros((H, R)),
               dA_dec=np.zeros(H), dtau=np.zeros((H, K)), dS0=np.zeros((B, H, V, K)), dm_prev_in=np.zeros((B, H, V)))
    order = ("dq", "dk", "dv", "dg_logit", "dbx", "dw_logit", "dA", "dB", "dAw", "dA_dec", "dtau", "dS0",
             "dm_prev_in")
    rc = lib.orc_bwd(ctypes.byref(d), *[_p(x) for x in a], _p(Aw), _p(A_dec), _p(tau), _p(S0), _p(m_prev),
                     _p(dO), _p(dS_final),
                     _p(dm_prev_out), *[_p(out[k]) for k in order], _p(cu))
    if rc:
        raise ValueError("oracle bwd: bad dims")
    return out


def step(tok: dict, A, Bm, S, L: int = 1, mc_mode: int = 0, mstate=None, pos=None,
         content_off: bool = False, Aw=None, A_dec=None, tau=None):
    """One decode step.  tok holds q, k, g_logit, bx [B,H,K], v [B,H,V], w_logit [B,H]; Aw
    [H,R] (the write gate's content term), A_dec [H] and tau [H,K] (the decay's log-amplitude
    and bias) are optional.
    S [B,H,V,K] (fp64) is updated in place; mstate [B,H,2,V] and pos [B,H] (int32) too in
    mc_mode 1.  Returns o [B,H,V]."""
    lib = _load()
    B, H, K = tok["q"].shape
    V = tok["v"].shape[-1]
    R = np.shape(A)[-1]
    d = _Dims(B, H, 1, K, V, R, L, mc_mode, int(content_off))
    assert S.dtype == np.float64 and S.flags.c_contiguous
    if mstate is None:
        mstate = np.zeros((B, H, 2, V))
    if pos is None:
        pos = np.zeros((B, H), dtype=np.int32)
    assert mstate.dtype == np.float64 and pos.dtype == np.int32
    t = {k: _f64(tok[k]) for k in ("q", "k", "v", "g_logit", "bx", "w_logit")}
    A, Bm, Aw, A_dec, tau = _f64(A), _f64(Bm), _f64(Aw), _f64(A_dec), _f64(tau)
    o = np.zeros((B, H, V))
    rc = lib.orc_step(ctypes.byref(d), _p(t["q"]), _p(t["k"]), _p(t["v"]), _p(t["g_logit"]), _p(t["bx"]),
                      _p(t["w_logit"]), _p(A), _p(Bm), _p(Aw), _p(A_dec), _p(tau), _p(S), _p(mstate),
                      _p(pos), _p(o))
    if rc:
        raise ValueError("oracle step: bad dims")
    return o


def threads() -> int:
    """OpenMP threads the oracle uses (OMP_NUM_THREADS, else every host core)."""
    return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
