"""Tensor-core path (bf16 q/k/v/o, dk = dv = 128) against the fp64 oracle.

Covers every gate chunk the forward serves (32, 64, 128), both readouts, carried state and
signal, and gates that decay hard (erase pre-activations far below zero, or a decay amplitude
that drives log g below -10), where the per-step retention floor of e^-10 becomes active: in
the forward alone, and through the training path (the saving forward and the backward), where
every output and gradient is compared.  The floor keeps the forward's deviation far inside the
bf16 tolerance, and the backward returns the exact recurrence's gate gradients where it binds.
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


GRADS = ("dq", "dk", "dv", "dg_logit", "dbx", "dw_logit", "dA", "dB", "dS0")


def train_case(cuda_device, w, d, mode):
    """Saving forward + backward on the GPU against the oracle: every output and gradient."""
    import torch
    dO = I.make_grad_out(w)
    S0 = I.make_state(w, 0.1)
    mp = I.normal(w.seed, 41, (w.B, w.H, w.V)).astype(np.float32)
    dSf = I.normal(w.seed, 43, (w.B, w.H, w.V, w.K)).astype(np.float32)
    dd = to_dev(dict(d, dO=dO), "bf16", cuda_device)
    extra = {k: torch.from_numpy(np.asarray(d[k], dtype=np.float32)).to(cuda_device)
             for k in ("A_dec", "tau") if k in d}
    tS0, tmp, tdS = (torch.from_numpy(x).to(cuda_device) for x in (S0, mp, dSf))
    args = (dd["q"], dd["k"], dd["v"], dd["g_logit"], dd["bx"], dd["w_logit"], dd["A"], dd["B"])
    out = carve.carve_fwd(*args, chunk=w.L, mc_mode=mode, S0=tS0, m_prev_in=tmp, save_for_bwd=True, **extra)
    g = carve.carve_bwd(*args, out["saved"], dd["dO"], chunk=w.L, mc_mode=mode, S0=tS0, m_prev_in=tmp,
                        dS_final=tdS, **extra)
    torch.cuda.synchronize()
    assert carve.carve_check() == 0
    r = oracle.fwd(d, L=w.L, mc_mode=mode, S0=S0, m_prev=mp)
    rg = oracle.bwd(d, w.L, dO, mc_mode=mode, S0=S0, m_prev=mp, dS_final=dSf)
    errs = {k: rel_l2(host(out[k]), r[k]) for k in ("o", "S_final", "m_prev_out")}
    keys = GRADS + tuple(k for k, x in (("dA_dec", "A_dec"), ("dtau", "tau")) if x in d)
    keys += ("dm_prev_in",) if mode == 1 else ()
    errs.update({k: rel_l2(host(g[k]), rg[k]) for k in keys})
    bad = {k: e for k, e in errs.items() if not e <= TOL["bf16"]}
    assert not bad, {k: f"{e:.3e}" for k, e in bad.items()}
    return errs


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("bx_shift", [-6.0, -30.0])
def test_tc_training_hard_erase(cuda_device, bx_shift, mode):
    """Erase gate pre-activations shifted by -6 (a ~ 2.5e-3 per step; the floor binds on the
    tail) and by -30 (a ~ 1e-13: the floor binds on every channel of every token, where the
    exact gradients of g_logit, bx, A and B are of order a)."""
    w = dataclasses.replace(I.FWD_1P3B, B=1, H=3, T=192, L=64, seed=311 + mode)
    d = I.make_inputs(w)
    d["bx"] = (d["bx"] + bx_shift).astype(np.float32)
    d["A"] *= 10.0
    d["B"] *= 10.0
    errs = train_case(cuda_device, w, d, mode)
    print(bx_shift, mode, {k: f"{v:.2e}" for k, v in errs.items()})


@pytest.mark.parametrize("mode", [0, 1])
def test_tc_training_decay_below_floor(cuda_device, mode):
    """The decay's amplitude drives log g below -10 on head 0 (amplitude 40 on softplus(g_logit
    + tau) ~ 0.3-1.3), near it on head 1 (amplitude 8) and leaves head 2 ordinary."""
    w = dataclasses.replace(I.FWD_1P3B, B=2, H=3, T=128, L=64, seed=317 + mode)
    d = I.make_inputs(w)
    d["A"] *= 10.0
    d["B"] *= 10.0
    d["A_dec"] = np.log(np.array([40.0, 8.0, 1.0])).astype(np.float32)
    d["tau"] = I.normal(w.seed, 45, (w.H, w.K), 2.0, 0.5).astype(np.float32)
    errs = train_case(cuda_device, w, d, mode)
    print(mode, {k: f"{v:.2e}" for k, v in errs.items()})
