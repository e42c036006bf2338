"""Tensor-core forward path (bf16 q/k/v/o, dk = dv = 128) against the fp64 oracle.

Covers every gate chunk it serves (32, 64, 128), both readouts, carried state and signal,
and gates that decay hard (erase pre-activations far below zero), where the per-step
retention floor of e^-10 becomes active; the floor keeps the deviation far inside the bf16
tolerance.
"""
import dataclasses

import numpy as np
import pytest

import chunk_gated_delta_b200 as carve
import oracle
from chunk_gated_delta_b200 import inputs as I
from tests.helpers import TOL, host, rel_l2, to_dev

pytestmark = pytest.mark.gpu


def run(cuda_device, d, L, mode, S0=None, mp=None):
    import torch
    dd = to_dev(d, "bf16", cuda_device)
    tS0 = None if S0 is None else torch.from_numpy(S0).to(cuda_device)
    tmp = None if mp is None else torch.from_numpy(mp).to(cuda_device)
    out = carve.carve_fwd(dd["q"], dd["k"], dd["v"], dd["g_logit"], dd["bx"], dd["w_logit"], dd["A"], dd["B"],
                          chunk=L, mc_mode=mode, S0=tS0, m_prev_in=tmp, save_for_bwd=False)
    torch.cuda.synchronize()
    r = oracle.fwd(d, L=L, mc_mode=mode, S0=S0, m_prev=mp)
    errs = {k: rel_l2(host(out[k]), r[k]) for k in ("o", "S_final", "m_prev_out")}
    for k, e in errs.items():
        assert e <= TOL["bf16"], (k, e)
    return errs


@pytest.mark.parametrize("L", [32, 64, 128])
@pytest.mark.parametrize("mode", [0, 1])
def test_tc_forward(cuda_device, L, mode):
    w = dataclasses.replace(I.FWD_1P3B, B=2, H=3, T=384, seed=100 + L + mode)
    d = I.make_inputs(w)
    d["A"] *= 10.0
    d["B"] *= 10.0
    S0 = I.make_state(w, 0.1)
    mp = I.normal(5, 5, (w.B, w.H, w.V)).astype(np.float32)
    errs = run(cuda_device, d, L, mode, S0, mp)
    print(L, mode, {k: f"{v:.2e}" for k, v in errs.items()})


@pytest.mark.parametrize("bx_mean", [-6.0, -30.0])
def test_tc_forward_hard_erase(cuda_device, bx_mean):
    w = dataclasses.replace(I.FWD_1P3B, B=1, H=4, T=256, seed=7)
    d = I.make_inputs(w)
    d["bx"] = (d["bx"] + bx_mean).astype(np.float32)
    d["A"] *= 10.0
    d["B"] *= 10.0
    errs = run(cuda_device, d, 64, 0)
    print(bx_mean, {k: f"{v:.2e}" for k, v in errs.items()})
