"""The chunked WY-form restatement (oracle/wy.py) against the token-sequential oracle.

The two share no code.  Agreement to ~1e-12 for every compute sub-chunk Lc dividing the
gate chunk L, with ragged chunks, both readout modes, carried state and carried content
signal, pins the chunk-parallel algebra (the single WY solve shared by all value channels,
CARVE blog section 2.3) that the GPU kernels implement, forward and backward.
"""
import dataclasses

import numpy as np
import pytest

import oracle
import oracle.wy as wy
from chunk_gated_delta_b200 import inputs as I


def case(T=37, K=8, V=6, R=3, seed=7):
    w = dataclasses.replace(I.TINY_FP32, B=2, H=2, T=T, K=K, V=V, R=R, L=16, seed=seed)
    d = {k: np.asarray(v, dtype=np.float64) for k, v in I.make_inputs(w).items()}
    d["A"] *= 40.0
    d["B"] *= 40.0
    S0 = I.make_state(w, 0.3).astype(np.float64)
    mp = I.normal(seed, 99, (w.B, w.H, w.V))
    return w, d, S0, mp


def rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def with_terms(w, d, terms):
    """Optional terms: the write gate's content term ("write") and the decay's amplitude and
    bias ("decay", scaled up so they matter at these sizes)."""
    d = dict(d)
    if "write" in terms:
        d["Aw"] = I.normal(w.seed, 98, (w.H, w.R), 0.0, 40.0 * 0.02)
    if "decay" in terms:
        d["A_dec"] = I.normal(w.seed, 97, (w.H,), 0.5, 0.5)
        d["tau"] = I.normal(w.seed, 96, (w.H, w.K), 1.0, 1.0)
    return d


@pytest.mark.parametrize("mc_mode", [0, 1])
@pytest.mark.parametrize("L,Lc", [(16, 16), (16, 8), (16, 4), (16, 1), (12, 4), (1, 1)])
@pytest.mark.parametrize("terms", ["", "write", "decay"])
def test_wy_forward_matches_sequential(mc_mode, L, Lc, terms):
    w, d, S0, mp = case()
    d = with_terms(w, d, terms)
    r = oracle.fwd(d, L=L, mc_mode=mc_mode, S0=S0, m_prev=mp)
    q = wy.fwd(d, L, Lc, mc_mode, S0=S0, m_prev=mp)
    for key in r:
        assert rel(q[key], r[key]) < 1e-12, key


@pytest.mark.parametrize("mc_mode", [0, 1])
@pytest.mark.parametrize("L,Lc", [(16, 16), (16, 4), (12, 6), (1, 1)])
@pytest.mark.parametrize("terms", ["", "write", "decay"])
def test_wy_backward_matches_bptt(mc_mode, L, Lc, terms):
    w, d, S0, mp = case(T=29)
    d = with_terms(w, d, terms)
    dO = I.normal(1, 2, (w.B, w.T, w.H, w.V))
    dSf = I.normal(1, 3, (w.B, w.H, w.V, w.K))
    dmo = I.normal(1, 4, (w.B, w.H, w.V))
    g = oracle.bwd(d, L, dO, mc_mode=mc_mode, S0=S0, m_prev=mp, dS_final=dSf, dm_prev_out=dmo)
    h = wy.bwd(d, L, dO, Lc, mc_mode, S0=S0, m_prev=mp, dS_final=dSf, dm_prev_out=dmo)
    for key in g:
        absent = (key == "dAw" and "write" not in terms) or (key in ("dA_dec", "dtau") and "decay" not in terms)
        if (mc_mode == 0 and key == "dm_prev_in") or absent:
            assert np.all(g[key] == 0) and np.all(h[key] == 0)
            continue
        assert rel(h[key], g[key]) < 1e-11, key


def test_wy_strong_decay_no_overflow():
    """Per-step log-retention near -20 (a ~ 2e-9): the decays of a 16-token chunk span
    e^-320, far outside fp64's exponent range if formed as 1/gamma; relative exponents
    exp(Lam_t - Lam_s) <= 1 keep the chunked form exact."""
    w, d, S0, mp = case(T=32)
    d["bx"][:] = -20.0
    r = oracle.fwd(d, L=16, S0=S0)
    q = wy.fwd(d, 16, 16, 0, S0=S0)
    assert np.all(np.isfinite(q["o"]))
    assert rel(q["o"], r["o"]) < 1e-12
