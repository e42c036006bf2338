"""Device status path: a bounded wait that gives up is reported by carve_check as
CARVE_ERR_TIMEOUT (then cleared), and the CUDA context stays usable afterwards: for the
dedicated one-thread wait, and for the barrier waits inside the tensor-core forward and
backward sweeps (carve_selftest_stall makes their first tile copy never arrive)."""
import dataclasses

import pytest

import chunk_gated_delta_b200 as carve
import oracle
from chunk_gated_delta_b200 import inputs as I
from tests.helpers import TOL, host, rel_l2, to_dev

pytestmark = pytest.mark.gpu


def _tiny_fwd(dev):
    w = I.TINY_FP32
    d = I.make_inputs(w)
    dd = to_dev(d, w.io, dev)
    out = carve.carve_fwd(dd["q"], dd["k"], dd["v"], dd["g_logit"], dd["bx"], dd["w_logit"], dd["A"], dd["B"],
                          chunk=w.L, save_for_bwd=False)
    return host(out["o"]), oracle.fwd(d, L=w.L)["o"]


def test_clean_run_reports_ok(cuda_device):
    got, want = _tiny_fwd(cuda_device)
    assert carve.carve_check() == 0
    assert rel_l2(got, want) <= TOL["fp32"]


def test_expired_wait_is_reported_and_context_survives(cuda_device):
    lib = carve.load()
    assert carve.carve_check() == 0
    assert lib.carve_selftest_timeout(1000, None) == 0
    assert carve.carve_check() == 4            # CARVE_ERR_TIMEOUT
    assert carve.carve_check() == 0            # the status word was cleared
    got, want = _tiny_fwd(cuda_device)         # and the context still computes correctly
    assert carve.carve_check() == 0
    assert rel_l2(got, want) <= TOL["fp32"]


def _tc_case(dev, mode):
    w = dataclasses.replace(I.FWD_1P3B, B=2, H=2, T=128, L=64, seed=331 + mode)
    d = I.make_inputs(w)
    d["A"] *= 10.0
    d["B"] *= 10.0
    dO = I.make_grad_out(w)
    dd = to_dev(dict(d, dO=dO), "bf16", dev)
    args = (dd["q"], dd["k"], dd["v"], dd["g_logit"], dd["bx"], dd["w_logit"], dd["A"], dd["B"])
    return w, d, dO, dd, args


@pytest.mark.parametrize("which", ["fwd_saving", "fwd_inference", "bwd"])
def test_tensor_core_wait_gives_up_and_context_survives(cuda_device, which):
    """A real tensor-core sweep whose first tile copy never arrives: every CTA's wait gives up
    after the armed 1000 polls, the sweep ends, carve_check reports CARVE_ERR_TIMEOUT once,
    and a following normal call matches the oracle."""
    import torch
    lib = carve.load()
    mode = 0
    w, d, dO, dd, args = _tc_case(cuda_device, mode)
    assert carve.carve_check() == 0
    save = which != "fwd_inference"
    out = carve.carve_fwd(*args, chunk=w.L, mc_mode=mode, save_for_bwd=save) if which == "bwd" else None
    assert carve.carve_check() == 0
    assert lib.carve_selftest_stall(1000) == 0
    if which == "bwd":
        carve.carve_bwd(*args, out["saved"], dd["dO"], chunk=w.L, mc_mode=mode)
    else:
        carve.carve_fwd(*args, chunk=w.L, mc_mode=mode, save_for_bwd=save)
    assert carve.carve_check() == 4            # CARVE_ERR_TIMEOUT
    assert carve.carve_check() == 0            # the status word was cleared
    # the one-shot was consumed: a normal training step matches the oracle
    out = carve.carve_fwd(*args, chunk=w.L, mc_mode=mode, save_for_bwd=True)
    g = carve.carve_bwd(*args, out["saved"], dd["dO"], chunk=w.L, mc_mode=mode)
    torch.cuda.synchronize()
    assert carve.carve_check() == 0
    r = oracle.fwd(d, L=w.L, mc_mode=mode)
    rg = oracle.bwd(d, w.L, dO, mc_mode=mode)
    assert rel_l2(host(out["o"]), r["o"]) <= TOL["bf16"]
    for k in ("dq", "dk", "dv", "dg_logit", "dbx", "dA", "dB"):
        assert rel_l2(host(g[k]), rg[k]) <= TOL["bf16"], k
