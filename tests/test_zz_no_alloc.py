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


def test_tensor_core_workspace_formula():
    """The tensor-core backward's workspace is the size the header states: per unit
    NG*292 + 132 floats, plus ceil(B*NG/64)*H*257*rank floats of slice partials."""
    for B, H, T, R, L in ((2, 4, 192, 16, 64), (8, 16, 4096, 32, 64), (1, 16, 4096, 32, 32), (3, 2, 96, 8, 128)):
        d = carve.Dims(B=B, H=H, T=T, dk=128, dv=128, rank=R, chunk=L, io=1, mc_mode=0)
        NG = -(-T // L)
        floats = B * H * (NG * 292 + 132) + -(-(B * NG) // 64) * H * 257 * R
        assert carve.bwd_workspace_bytes(d) == 4 * floats, (B, H, T, R, L)


def _noalloc_case(cuda_device, w, mode, extras=False, bitwise=False):
    """carve_bwd_noalloc twice in a row against carve_bwd (and the oracle on the tensor-core
    shape): the fixed array keeps the first call's contents, so the second call shows whether
    anything that must start from zero is left over."""
    import torch
    import oracle
    lib = _lib()
    d = I.make_inputs(w)
    d["A"] *= 10.0
    d["B"] *= 10.0
    opt = {}
    if extras:
        d["Aw"] = I.normal(w.seed, 97, (w.H, w.R), 0.0, 2.0)
        d.update(I.make_decay(w))
        opt = {k: torch.from_numpy(np.asarray(d[k], dtype=np.float32)).to(cuda_device) for k in ("Aw", "A_dec", "tau")}
    dO = I.make_grad_out(w)
    dd = to_dev(dict(d, dO=dO), w.io, cuda_device)
    dSf_h = I.normal(9, 9, (w.B, w.H, w.V, w.K)).astype(np.float32)
    dSf = torch.from_numpy(dSf_h).to(cuda_device)
    args = (dd["q"], dd["k"], dd["v"], dd["g_logit"], dd["bx"], dd["w_logit"], dd["A"], dd["B"])
    fwd = carve.carve_fwd(*args, chunk=w.L, mc_mode=mode, **opt)
    ref = carve.carve_bwd(*args, fwd["saved"], dd["dO"], chunk=w.L, mc_mode=mode, dS_final=dSf, **opt)
    keys = GRADS + (("dAw", "dA_dec", "dtau") if extras else ())
    dims = carve.dims_of(dd["q"], dd["v"], dd["A"], w.L, mode)
    assert carve.bwd_workspace_bytes(dims) <= 4 << 20
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())   # noqa: E731
    rg = None
    if w.K == 128 and w.V == 128 and w.io == "bf16":   # the tensor-core shape: also against the oracle
        rg = oracle.bwd(d, w.L, dO, mc_mode=mode, dS_final=dSf_h)
    for call in range(2):
        out = {k: torch.full_like(ref[k], float("nan")) for k in keys}
        g = lambda k: p(out.get(k))   # noqa: E731
        rc = lib.carve_bwd_noalloc(ctypes.byref(dims), *[p(t) for t in args], p(opt.get("Aw")), p(opt.get("A_dec")),
                                   p(opt.get("tau")), None, None, p(fwd["saved"]), p(dd["dO"]), p(dSf), None,
                                   g("dq"), g("dk"), g("dv"), g("dg_logit"), g("dbx"), g("dw_logit"), g("dA"),
                                   g("dB"), g("dAw"), g("dA_dec"), g("dtau"), g("dS0"), g("dm_prev_in"), stream)
        assert rc == 0, carve.STATUS.get(rc, rc)
        torch.cuda.synchronize()
        for k in keys:
            if bitwise:   # the same deterministic kernels on the same inputs: the same bits
                assert torch.equal(out[k], ref[k]), f"call {call + 1}: {k} differs from carve_bwd"
            e = rel_l2(host(out[k]), host(ref[k]))
            assert e <= TOL[w.io], f"call {call + 1}: {k} rel-L2 {e:.2e}"
            if rg is not None and (k != "dm_prev_in" or mode == 1):
                e = rel_l2(host(out[k]), rg[k])
                assert e <= TOL[w.io], f"call {call + 1}: {k} rel-L2 {e:.2e} against the oracle"


@pytest.mark.gpu
@pytest.mark.parametrize("io,mode", [("fp32", 1), ("bf16", 0)])
def test_noalloc_backward_matches_carve_bwd_twice(cuda_device, io, mode):
    """The SIMT backward (dv = 64) through the fixed array."""
    w = I.Workload("noalloc_check", B=2, H=4, T=192, K=128, V=64, R=16, L=64, io=io, seed=4242)
    _noalloc_case(cuda_device, w, mode, bitwise=True)


@pytest.mark.gpu
@pytest.mark.parametrize("extras", [False, True])
@pytest.mark.parametrize("mode", [0, 1])
def test_noalloc_tensor_core_backward(cuda_device, mode, extras):
    """The tensor-core backward (bf16, dk = dv = 128, rank 16, gate chunk 64) through the fixed
    array: its per-gate-chunk records, dq readout vectors, slice partials of dA/dB/dAw and (with
    the decay's parameters) decay records all live in it.  Bit for bit equal to carve_bwd on two
    calls in a row, and within the bf16 tolerance of the oracle."""
    w = I.Workload("noalloc_tc", B=2, H=4, T=192, K=128, V=128, R=16, L=64, io="bf16", seed=4243 + mode)
    _noalloc_case(cuda_device, w, mode, extras=extras, bitwise=True)
