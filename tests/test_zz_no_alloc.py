"""carve_bwd_noalloc: the backward for callers that cannot allocate device memory.

Such callers (for instance a plugin running inside a host framework that owns all device
memory and hands it only input and output buffers, or a latency-critical loop that must not
pay for cudaMalloc's implicit synchronisation) get a backward whose scratch is a fixed 4 MiB
array inside the library.  These tests check that it gives the same gradients as carve_bwd,
call after call (the shared array keeps the previous call's contents, so a second call would
expose any state that is not cleared), and that problems too large for the array are
refused on the host.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest

import chunk_gated_delta_b200 as carve
from chunk_gated_delta_b200 import build
from chunk_gated_delta_b200 import inputs as I
from tests.helpers import TOL, host, rel_l2, to_dev

GRADS = ("dq", "dk", "dv", "dg_logit", "dbx", "dw_logit", "dA", "dB", "dS0", "dm_prev_in")


def _lib():
    build.build()
    lib = carve.load()
    f = lib.carve_bwd_noalloc
    f.argtypes = [ctypes.POINTER(carve.Dims)] + [ctypes.c_void_p] * 31
    f.restype = ctypes.c_int
    return lib


def test_too_large_for_the_array_is_refused_before_any_launch():
    """B*H*(dk*rank + rank*dv + rank + dk + 1) above 1,048,576 floats (4 MiB) returns
    CARVE_ERR_UNSUPPORTED.  The size check comes first, so the placeholder pointers are never
    used."""
    lib = _lib()
    d = carve.Dims(B=5, H=16, T=64, dk=128, dv=128, rank=64, chunk=64, io=1, mc_mode=0)
    assert carve.bwd_workspace_bytes(d) > 4 << 20
    P = ctypes.c_void_p(4096)
    args = [P] * 8 + [None] * 5 + [P, P, None, None] + [P] * 8 + [None] * 5 + [None]
    assert lib.carve_bwd_noalloc(ctypes.byref(d), *args) == 2
    fits = carve.Dims(B=3, H=16, T=64, dk=128, dv=128, rank=64, chunk=64, io=1, mc_mode=0)
    assert carve.bwd_workspace_bytes(fits) <= 4 << 20
    bad = carve.Dims(B=4, H=16, T=64, dk=96, dv=128, rank=64, chunk=64, io=1, mc_mode=0)
    assert lib.carve_bwd_noalloc(ctypes.byref(bad), *args) == 2      # same answer as carve_bwd


@pytest.mark.gpu
@pytest.mark.parametrize("io,mode", [("fp32", 1), ("bf16", 0)])
def test_noalloc_backward_matches_carve_bwd_twice(cuda_device, io, mode):
    import torch
    lib = _lib()
    w = I.Workload("noalloc_check", B=2, H=4, T=192, K=128, V=64, R=16, L=64, io=io, seed=4242)
    d = I.make_inputs(w)
    d["A"] *= 10.0
    d["B"] *= 10.0
    dd = to_dev(dict(d, dO=I.make_grad_out(w)), io, cuda_device)
    dSf = torch.from_numpy(I.normal(9, 9, (w.B, w.H, w.V, w.K)).astype(np.float32)).to(cuda_device)
    args = (dd["q"], dd["k"], dd["v"], dd["g_logit"], dd["bx"], dd["w_logit"], dd["A"], dd["B"])
    fwd = carve.carve_fwd(*args, chunk=w.L, mc_mode=mode)
    ref = carve.carve_bwd(*args, fwd["saved"], dd["dO"], chunk=w.L, mc_mode=mode, dS_final=dSf)
    dims = carve.dims_of(dd["q"], dd["v"], dd["A"], w.L, mode)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())   # noqa: E731
    for call in range(2):
        out = {k: torch.full_like(ref[k], float("nan")) for k in GRADS}
        grads = [p(out[k]) for k in GRADS]   # ... dA, dB, (dAw, dA_dec, dtau: none), dS0, dm_prev_in
        rc = lib.carve_bwd_noalloc(ctypes.byref(dims), *[p(t) for t in args], None, None, None, None, None,
                                   p(fwd["saved"]), p(dd["dO"]), p(dSf), None, *grads[:8], None, None, None,
                                   *grads[8:], stream)
        assert rc == 0, carve.STATUS.get(rc, rc)
        torch.cuda.synchronize()
        for k in GRADS:
            e = rel_l2(host(out[k]), host(ref[k]))
            assert e <= TOL[io], f"call {call + 1}: {k} rel-L2 {e:.2e}"
