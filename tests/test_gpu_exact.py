"""The exact content-aware recurrence (chunk = 1: the content signal of every token read from
the state right before it) against the oracle at L = 1, element by element: forward outputs,
final state and readout, and every gradient, with a carried state, upstream gradients on the
final state and readout, and (terms) the write gate's content term and the decay's amplitude
and bias.  T spans several 64-token checkpoint segments with a ragged last one."""
import dataclasses

import numpy as np
import pytest

import chunk_gated_delta_b200 as carve
import oracle
from chunk_gated_delta_b200 import inputs as I
from tests.helpers import TOL, host, rel_l2, to_dev

pytestmark = pytest.mark.gpu

GRADS = ("dq", "dk", "dv", "dg_logit", "dbx", "dw_logit", "dA", "dB", "dS0")


@pytest.mark.parametrize("io,K,V,T", [("fp32", 64, 64, 160), ("bf16", 128, 128, 144), ("fp32", 128, 64, 80)])
@pytest.mark.parametrize("terms", [False, True])
def test_exact_recurrence_matches_oracle(cuda_device, io, K, V, T, terms):
    import torch
    w = dataclasses.replace(I.TINY_FP32, B=2, H=2, T=T, K=K, V=V, R=16, L=1, io=io, seed=500 + K + T)
    d = I.make_inputs(w)
    d["A"] *= 10.0
    d["B"] *= 10.0
    grads = GRADS
    if terms:
        d["Aw"] = I.normal(w.seed, 97, (w.H, w.R), 0.0, 2.0).astype(np.float32)
        d.update(I.make_decay(w))
        grads = GRADS + ("dAw", "dA_dec", "dtau")
    dO = I.make_grad_out(w)
    S0 = I.make_state(w, 0.05)
    dSf = I.normal(6, 3, (w.B, w.H, V, K)).astype(np.float32)
    dmo = I.normal(6, 4, (w.B, w.H, V)).astype(np.float32)
    dd = to_dev(dict(d, dO=dO), io, cuda_device)
    extra = {k: dd[k] for k in ("Aw", "A_dec", "tau") if k in dd}
    tS0, tdS, tdm = (torch.from_numpy(x).to(cuda_device) for x in (S0, dSf, dmo))
    args = tuple(dd[k] for k in ("q", "k", "v", "g_logit", "bx", "w_logit", "A", "B"))
    out = carve.carve_fwd(*args, chunk=1, mc_mode=0, S0=tS0, **extra)
    g = carve.carve_bwd(*args, out["saved"], dd["dO"], chunk=1, mc_mode=0, S0=tS0, dS_final=tdS, dm_prev_out=tdm,
                        **extra)
    assert carve.carve_check() == 0
    od = {k: np.asarray(v, dtype=np.float64) for k, v in d.items()}
    r = oracle.fwd(od, L=1, mc_mode=0, S0=S0)
    rg = oracle.bwd(od, 1, dO, mc_mode=0, S0=S0, dS_final=dSf, dm_prev_out=dmo)
    tol = TOL[io]
    for key in ("o", "S_final", "m_prev_out"):
        e = rel_l2(host(out[key]), r[key])
        assert e <= tol, f"{key}: rel-L2 {e:.3e}"
    for key in grads:
        e = rel_l2(host(g[key]), rg[key])
        assert e <= tol, f"{key}: rel-L2 {e:.3e}"
    assert torch.all(g["dm_prev_in"] == 0)
