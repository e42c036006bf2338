"""Python binding of libcarve.so, the B200 (sm_100a) CARVE recurrence library.

Argument marshalling only: every step of the recurrence runs in the library's CUDA kernels
(include/carve.h).  PyTorch supplies device memory and the current stream.  There is no
CPU fallback: if libcarve.so is missing or fails to load, every call raises.

    import chunk_gated_delta_b200 as carve
    out  = carve.carve_fwd(q, k, v, g_logit, bx, w_logit, A, B, chunk=64)
    grads = carve.carve_bwd(q, k, v, g_logit, bx, w_logit, A, B, out["saved"], dO, chunk=64)
    o = carve.carve_step(q1, k1, v1, g1, bx1, w1, A, B, S)      # one decode token, S in place
"""
from __future__ import annotations

import ctypes
import os

__all__ = ["CarveError", "Dims", "load", "library_path", "carve_fwd", "carve_bwd", "carve_step",
           "saved_bytes", "bwd_workspace_bytes", "STATUS"]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libcarve.so")
_lib = None

STATUS = {0: "CARVE_OK", 1: "CARVE_ERR_INVALID_ARG", 2: "CARVE_ERR_UNSUPPORTED", 3: "CARVE_ERR_CUDA",
          4: "CARVE_ERR_TIMEOUT"}
IO_FP32, IO_BF16 = 0, 1


class CarveError(RuntimeError):
    def __init__(self, fn, code):
        super().__init__(f"{fn} failed: {STATUS.get(code, code)}")
        self.code = code


class Dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("B", "H", "T", "dk", "dv", "rank", "chunk", "io", "mc_mode")]


def library_path() -> str:
    return _LIB_PATH


def load():
    """Load libcarve.so (built by chunk_gated_delta_b200.build) and declare its entry points."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"{_LIB_PATH} is missing: build it with `python -m chunk_gated_delta_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    P, D = ctypes.c_void_p, ctypes.POINTER(Dims)
    lib.carve_status_string.argtypes = [ctypes.c_int]
    lib.carve_status_string.restype = ctypes.c_char_p
    for f in (lib.carve_saved_bytes, lib.carve_bwd_workspace_bytes):
        f.argtypes = [D]
        f.restype = ctypes.c_size_t
    lib.carve_fwd.argtypes = [D] + [P] * 18
    lib.carve_bwd.argtypes = [D] + [P] * 32
    lib.carve_step.argtypes = [D] + [P] * 16
    lib.carve_fwd_varlen.argtypes = [D, P, ctypes.c_int64] + [P] * 18
    lib.carve_bwd_varlen.argtypes = [D, P, ctypes.c_int64] + [P] * 32
    lib.carve_check.argtypes = [P]
    lib.carve_selftest_timeout.argtypes = [ctypes.c_uint32, P]
    lib.carve_selftest_stall.argtypes = [ctypes.c_uint32]
    for f in (lib.carve_fwd, lib.carve_bwd, lib.carve_fwd_varlen, lib.carve_bwd_varlen, lib.carve_step,
              lib.carve_check, lib.carve_selftest_timeout, lib.carve_selftest_stall):
        f.restype = ctypes.c_int
    _lib = lib
    return lib


# ---------------------------------------------------------------------------------------
# marshalling helpers (torch is imported lazily so that CPU-only tooling can import us)
# ---------------------------------------------------------------------------------------
def _torch():
    import torch
    return torch


def _ptr(x):
    if x is None:
        return None
    if not x.is_contiguous():
        raise ValueError("tensors passed to libcarve must be contiguous")
    return ctypes.c_void_p(x.data_ptr())


def _stream(stream):
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _io_of(x):
    torch = _torch()
    if x.dtype == torch.float32:
        return IO_FP32
    if x.dtype == torch.bfloat16:
        return IO_BF16
    raise TypeError(f"q/k/v must be float32 or bfloat16, got {x.dtype}")


def dims_of(q, v, A, chunk, mc_mode) -> Dims:
    B, T, H, K = q.shape
    return Dims(B, H, T, K, v.shape[-1], A.shape[-1], chunk, _io_of(q), mc_mode)


def dims_varlen(q, v, A, cu_seqlens, max_len, chunk, mc_mode) -> Dims:
    """Dims of a packed call: B = number of sequences, T = max_len rounded up to 64 (so that the
    tensor-core kernels, which tile sequences by 32 or 64 tokens, serve their shapes)."""
    T = max(64, (int(max_len) + 63) // 64 * 64)
    return Dims(cu_seqlens.numel() - 1, q.shape[-2], T, q.shape[-1], v.shape[-1], A.shape[-1], chunk, _io_of(q),
                mc_mode)


def _packed(cu_seqlens, max_len, q):
    """(cu pointer, row count) of a packed call; max_len None reads the lengths on the host."""
    torch = _torch()
    if cu_seqlens.dtype != torch.int32 or cu_seqlens.device != q.device:
        raise TypeError("cu_seqlens must be an int32 tensor on the device of q")
    if max_len is None:
        max_len = int((cu_seqlens[1:] - cu_seqlens[:-1]).max().item()) if cu_seqlens.numel() > 1 else 0
    return [_ptr(cu_seqlens), ctypes.c_int64(q.shape[-3])], max_len


def saved_bytes(d: Dims) -> int:
    return int(load().carve_saved_bytes(ctypes.byref(d)))


def bwd_workspace_bytes(d: Dims) -> int:
    return int(load().carve_bwd_workspace_bytes(ctypes.byref(d)))


def _check(fn, rc):
    if rc != 0:
        raise CarveError(fn, rc)


def carve_check(stream=None) -> int:
    """Wait for `stream` and return the library's status: 0 (CARVE_OK), or the code of a CUDA
    error or of a bounded device-side wait that gave up since the last check."""
    return int(load().carve_check(_stream(stream)))


def carve_fwd(q, k, v, g_logit, bx, w_logit, A, B, chunk: int, mc_mode: int = 0, S0=None, m_prev_in=None,
              save_for_bwd: bool = True, out: dict | None = None, stream=None, Aw=None, A_dec=None,
              tau=None) -> dict:
    """Forward over [B,T,H,*] device tensors.  Optional: Aw [H,rank], the write gate's content
    term; A_dec [H] and tau [H,dk], the decay's log-amplitude and bias.  Returns dict(o,
    S_final, m_prev_out, saved); `out` may supply preallocated buffers under the same keys."""
    return _fwd(dims_of(q, v, A, chunk, mc_mode), None, q, k, v, g_logit, bx, w_logit, A, B, S0, m_prev_in,
                save_for_bwd, out, stream, Aw, A_dec, tau)


def carve_fwd_varlen(q, k, v, g_logit, bx, w_logit, A, B, cu_seqlens, chunk: int, max_len=None, mc_mode: int = 0,
                     S0=None, m_prev_in=None, save_for_bwd: bool = True, out: dict | None = None, stream=None,
                     Aw=None, A_dec=None, tau=None) -> dict:
    """Forward over variable-length sequences packed along the token axis: q, k, g_logit, bx
    [total,H,dk]; v [total,H,dv]; w_logit [total,H]; cu_seqlens int32 [N+1] on the device
    (sequence n = rows cu[n]..cu[n+1]); max_len >= every length (None: read from cu_seqlens on
    the host).  S0, m_prev_in and the per-sequence outputs are [N,H,...]."""
    pk, max_len = _packed(cu_seqlens, max_len, q)
    d = dims_varlen(q, v, A, cu_seqlens, max_len, chunk, mc_mode)
    return _fwd(d, pk, q, k, v, g_logit, bx, w_logit, A, B, S0, m_prev_in, save_for_bwd, out, stream, Aw, A_dec,
                tau)


def _fwd(d, pk, q, k, v, g_logit, bx, w_logit, A, B, S0, m_prev_in, save_for_bwd, out, stream, Aw, A_dec, tau):
    torch = _torch()
    lib = load()
    out = dict(out or {})
    dev = q.device
    if "o" not in out:
        out["o"] = torch.empty(v.shape, dtype=q.dtype, device=dev)
    if "S_final" not in out:
        out["S_final"] = torch.empty((d.B, d.H, d.dv, d.dk), dtype=torch.float32, device=dev)
    if "m_prev_out" not in out:
        out["m_prev_out"] = torch.empty((d.B, d.H, d.dv), dtype=torch.float32, device=dev)
    if save_for_bwd and out.get("saved") is None:
        n = saved_bytes(d)
        if n == 0:
            raise CarveError("carve_saved_bytes", 1)
        out["saved"] = torch.empty(n, dtype=torch.uint8, device=dev)
    fn = lib.carve_fwd if pk is None else lib.carve_fwd_varlen
    rc = fn(ctypes.byref(d), *(pk or []), _ptr(q), _ptr(k), _ptr(v), _ptr(g_logit), _ptr(bx), _ptr(w_logit),
            _ptr(A), _ptr(B), _ptr(Aw), _ptr(A_dec), _ptr(tau), _ptr(S0), _ptr(m_prev_in), _ptr(out["o"]),
            _ptr(out["S_final"]), _ptr(out["m_prev_out"]), _ptr(out.get("saved") if save_for_bwd else None),
            _stream(stream))
    _check("carve_fwd" if pk is None else "carve_fwd_varlen", rc)
    return out


def carve_bwd(q, k, v, g_logit, bx, w_logit, A, B, saved, dO, chunk: int, mc_mode: int = 0, S0=None,
              m_prev_in=None, dS_final=None, dm_prev_out=None, want_dS0: bool = True, out: dict | None = None,
              workspace=None, stream=None, Aw=None, A_dec=None, tau=None) -> dict:
    """Reverse sweep.  Returns dict(dq, dk, dv, dg_logit, dbx, dw_logit, dA, dB, dS0, dm_prev_in),
    plus dAw, dA_dec, dtau when the forward had Aw, A_dec, tau."""
    return _bwd(dims_of(q, v, A, chunk, mc_mode), None, q, k, v, g_logit, bx, w_logit, A, B, saved, dO, S0,
                m_prev_in, dS_final, dm_prev_out, want_dS0, out, workspace, stream, Aw, A_dec, tau)


def carve_bwd_varlen(q, k, v, g_logit, bx, w_logit, A, B, saved, dO, cu_seqlens, chunk: int, max_len=None,
                     mc_mode: int = 0, S0=None, m_prev_in=None, dS_final=None, dm_prev_out=None,
                     want_dS0: bool = True, out: dict | None = None, workspace=None, stream=None, Aw=None,
                     A_dec=None, tau=None) -> dict:
    """Reverse sweep of carve_fwd_varlen (same packed layouts and the same max_len)."""
    pk, max_len = _packed(cu_seqlens, max_len, q)
    d = dims_varlen(q, v, A, cu_seqlens, max_len, chunk, mc_mode)
    return _bwd(d, pk, q, k, v, g_logit, bx, w_logit, A, B, saved, dO, S0, m_prev_in, dS_final, dm_prev_out,
                want_dS0, out, workspace, stream, Aw, A_dec, tau)


def _bwd(d, pk, q, k, v, g_logit, bx, w_logit, A, B, saved, dO, S0, m_prev_in, dS_final, dm_prev_out, want_dS0,
         out, workspace, stream, Aw, A_dec, tau):
    torch = _torch()
    lib = load()
    dev = q.device
    out = dict(out or {})
    shapes = dict(dq=(q.shape, q.dtype), dk=(k.shape, k.dtype), dv=(v.shape, v.dtype),
                  dg_logit=(g_logit.shape, torch.float32), dbx=(bx.shape, torch.float32),
                  dw_logit=(w_logit.shape, torch.float32), dA=(A.shape, torch.float32), dB=(B.shape, torch.float32),
                  dm_prev_in=((d.B, d.H, d.dv), torch.float32))
    if want_dS0:
        shapes["dS0"] = ((d.B, d.H, d.dv, d.dk), torch.float32)
    for name, x in (("dAw", Aw), ("dA_dec", A_dec), ("dtau", tau)):
        if x is not None:
            shapes[name] = (x.shape, torch.float32)
    for key, (shp, dt) in shapes.items():
        if key not in out:
            out[key] = torch.empty(shp, dtype=dt, device=dev)
    if workspace is None:
        workspace = torch.empty(bwd_workspace_bytes(d), dtype=torch.uint8, device=dev)
    fn = lib.carve_bwd if pk is None else lib.carve_bwd_varlen
    rc = fn(ctypes.byref(d), *(pk or []), _ptr(q), _ptr(k), _ptr(v), _ptr(g_logit), _ptr(bx), _ptr(w_logit), _ptr(A),
            _ptr(B), _ptr(Aw), _ptr(A_dec), _ptr(tau), _ptr(S0), _ptr(m_prev_in), _ptr(saved), _ptr(dO),
            _ptr(dS_final), _ptr(dm_prev_out), _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]),
            _ptr(out["dg_logit"]), _ptr(out["dbx"]), _ptr(out["dw_logit"]), _ptr(out["dA"]), _ptr(out["dB"]),
            _ptr(out.get("dAw") if Aw is not None else None),
            _ptr(out.get("dA_dec") if A_dec is not None else None),
            _ptr(out.get("dtau") if tau is not None else None), _ptr(out.get("dS0")),
            _ptr(out["dm_prev_in"]), _ptr(workspace), _stream(stream))
    _check("carve_bwd" if pk is None else "carve_bwd_varlen", rc)
    return out


def carve_step(q, k, v, g_logit, bx, w_logit, A, B, S, mc_mode: int = 0, chunk: int = 1, mstate=None, pos=None,
               o=None, stream=None, Aw=None, A_dec=None, tau=None):
    """One decode token for every (b,h): q, k, g_logit, bx [B,H,dk]; v [B,H,dv]; w_logit [B,H];
    Aw [H,rank], A_dec [H], tau [H,dk] optional; S [B,H,dv,dk] float32 updated in place (mstate/pos too in mc_mode 1).
    Returns o [B,H,dv]."""
    torch = _torch()
    lib = load()
    Bn, H, K = q.shape
    d = Dims(Bn, H, 1, K, v.shape[-1], A.shape[-1], chunk, _io_of(q), mc_mode)
    if o is None:
        o = torch.empty((Bn, H, d.dv), dtype=q.dtype, device=q.device)
    rc = lib.carve_step(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(g_logit), _ptr(bx), _ptr(w_logit), _ptr(A),
                        _ptr(B), _ptr(Aw), _ptr(A_dec), _ptr(tau), _ptr(S), _ptr(mstate), _ptr(pos), _ptr(o),
                        _stream(stream))
    _check("carve_step", rc)
    return o
