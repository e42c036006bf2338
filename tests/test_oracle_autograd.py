"""Two more checks of the fp64 oracle (test infrastructure only).

1. Its hand-derived BPTT backward against reverse-mode automatic differentiation: the
   recurrence is written out again as eager float64 torch operations on the CPU and
   torch.autograd produces the gradients of sum(dO*o) + sum(dS_final*S_final) +
   sum(dm_prev_out*m_prev_out) for every input (q, k, v, both gate logits, the write logit,
   the low-rank factors A and B, the write gate's content factor Aw, the decay's
   log-amplitude A_dec and bias tau, the initial state and the carried content signal), in
   both readout modes, with a ragged last chunk.  The gradient arithmetic comes from
   autograd, not from the oracle's derivation, so a slip in any adjoint fails here.
2. The precision of the oracle's fp64 evaluation: the same definition evaluated in 50-digit
   arithmetic (mpmath) on tiny inputs must agree to 1e-13.  This re-types the forward
   definition, so it checks rounding and the stable forms of softplus / sigmoid, not the
   formula itself (the formula is pinned in test_oracle_pins.py).
"""
import dataclasses

import numpy as np
import pytest

import oracle
from chunk_gated_delta_b200 import inputs as I


def _case(seed, B=2, H=2, T=7, K=4, V=3, R=2, L=3):
    w = dataclasses.replace(I.TINY_FP32, B=B, H=H, T=T, K=K, V=V, R=R, L=L, seed=seed)
    d = {k: np.asarray(v, dtype=np.float64) for k, v in I.make_inputs(w).items()}
    d["A"] *= 30.0
    d["B"] *= 30.0
    S0 = I.make_state(w, 0.4).astype(np.float64)
    mp = I.normal(seed, 7, (B, H, V))
    return w, d, S0, mp


def _torch_forward(torch, x, L, mc_mode):
    """The recurrence as written in the definition (per unit, token-sequential)."""
    q, k, v, gl, bx, wl, A, Bm, Aw, A_dec, tau, S0, mp = (
        x[n] for n in ("q", "k", "v", "g_logit", "bx", "w_logit", "A", "B", "Aw", "A_dec", "tau", "S0", "m_prev"))
    B, T, H, K = q.shape
    V = v.shape[-1]
    sp = torch.nn.functional.softplus
    outs, finals, means = [], [], []
    for b in range(B):
        ob, fb, mb = [], [], []
        for h in range(H):
            S = S0[b, h]
            prev_mean = mp[b, h]
            o_unit = []
            for t0 in range(0, T, L):
                t1 = min(T, t0 + L)
                if mc_mode == 0:
                    m = S @ q[b, t0:t1, h].mean(dim=0)
                else:
                    m = prev_mean
                z = Bm[h] @ m
                delta = A[h] @ z
                dw = Aw[h] @ z   # the write gate's content term
                o_chunk = []
                for t in range(t0, t1):
                    decay = torch.exp(-torch.exp(A_dec[h]) * sp(gl[b, t, h] + tau[h]))
                    a = decay * torch.sigmoid(bx[b, t, h] + delta)
                    wt = torch.sigmoid(wl[b, t, h] + dw)
                    P = S * a[None, :]
                    e = v[b, t, h] - P @ k[b, t, h]
                    S = P + wt * torch.outer(e, k[b, t, h])
                    o_chunk.append(S @ q[b, t, h])
                o_chunk = torch.stack(o_chunk)
                prev_mean = o_chunk.mean(dim=0)
                o_unit.append(o_chunk)
            ob.append(torch.cat(o_unit))
            fb.append(S)
            mb.append(prev_mean)
        outs.append(torch.stack(ob, dim=1))
        finals.append(torch.stack(fb))
        means.append(torch.stack(mb))
    return torch.stack(outs), torch.stack(finals), torch.stack(means)


@pytest.mark.parametrize("mc_mode", [0, 1])
def test_backward_matches_autograd(mc_mode):
    torch = pytest.importorskip("torch")
    w, d, S0, mp = _case(31 + mc_mode)
    d["Aw"] = I.normal(31, 8, (w.H, w.R), 0.0, 3.0)
    d["A_dec"] = I.normal(31, 9, (w.H,), 0.0, 0.7)
    d["tau"] = I.normal(31, 10, (w.H, w.K), 0.0, 1.0)
    dO = I.normal(5, 1, (w.B, w.T, w.H, w.V))
    dSf = I.normal(5, 2, (w.B, w.H, w.V, w.K))
    dmo = I.normal(5, 3, (w.B, w.H, w.V))
    x = {n: torch.tensor(d[n], dtype=torch.float64, requires_grad=True) for n in
         ("q", "k", "v", "g_logit", "bx", "w_logit", "A", "B", "Aw", "A_dec", "tau")}
    x["S0"] = torch.tensor(S0, dtype=torch.float64, requires_grad=True)
    x["m_prev"] = torch.tensor(mp, dtype=torch.float64, requires_grad=True)
    o, Sf, mo = _torch_forward(torch, x, w.L, mc_mode)
    ref = oracle.fwd(d, L=w.L, mc_mode=mc_mode, S0=S0, m_prev=mp)
    np.testing.assert_allclose(o.detach().numpy(), ref["o"], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(Sf.detach().numpy(), ref["S_final"], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(mo.detach().numpy(), ref["m_prev_out"], rtol=1e-12, atol=1e-13)
    loss = (o * torch.from_numpy(dO)).sum() + (Sf * torch.from_numpy(dSf)).sum() + (mo * torch.from_numpy(dmo)).sum()
    names = ["q", "k", "v", "g_logit", "bx", "w_logit", "A", "B", "Aw", "A_dec", "tau", "S0", "m_prev"]
    grads = torch.autograd.grad(loss, [x[n] for n in names], allow_unused=True)   # m_prev: mode 1 only
    g = oracle.bwd(d, w.L, dO, mc_mode=mc_mode, S0=S0, m_prev=mp, dS_final=dSf, dm_prev_out=dmo)
    keys = ["dq", "dk", "dv", "dg_logit", "dbx", "dw_logit", "dA", "dB", "dAw", "dA_dec", "dtau", "dS0",
            "dm_prev_in"]
    for n, gk, ga in zip(names, keys, grads):
        if ga is None:   # the input does not reach the loss: the oracle must report zeros
            assert np.all(g[gk] == 0.0), gk
            continue
        ga = ga.numpy()
        err = np.linalg.norm(g[gk] - ga) / max(np.linalg.norm(ga), 1e-300)
        assert err <= 1e-11, f"{gk}: rel {err:.2e} against autograd"


def _mp_forward(mp, d, L, mc_mode):
    """The definition in 50-digit arithmetic (B = H = 1)."""
    T, K = d["q"].shape[1], d["q"].shape[3]
    V = d["v"].shape[3]

    def M(x):
        return mp.mpf(float(x))

    def softplus(x):
        return mp.log1p(mp.exp(x)) if x < 0 else x + mp.log1p(mp.exp(-x))

    def sigmoid(x):
        return 1 / (1 + mp.exp(-x))

    R = d["A"].shape[2]
    A = [[M(d["A"][0, i, r]) for r in range(R)] for i in range(K)]
    Bm = [[M(d["B"][0, r, j]) for j in range(V)] for r in range(R)]
    S = [[mp.mpf(0) for _ in range(K)] for _ in range(V)]
    prev_mean = [mp.mpf(0)] * V
    o = []
    for t0 in range(0, T, L):
        t1 = min(T, t0 + L)
        if mc_mode == 0:
            qbar = [sum(M(d["q"][0, t, 0, i]) for t in range(t0, t1)) / (t1 - t0) for i in range(K)]
            m = [sum(S[j][i] * qbar[i] for i in range(K)) for j in range(V)]
        else:
            m = prev_mean
        z = [sum(Bm[r][j] * m[j] for j in range(V)) for r in range(R)]
        delta = [sum(A[i][r] * z[r] for r in range(R)) for i in range(K)]
        oc = []
        for t in range(t0, t1):
            q = [M(d["q"][0, t, 0, i]) for i in range(K)]
            k = [M(d["k"][0, t, 0, i]) for i in range(K)]
            v = [M(d["v"][0, t, 0, j]) for j in range(V)]
            a = [mp.exp(-softplus(M(d["g_logit"][0, t, 0, i]))) * sigmoid(M(d["bx"][0, t, 0, i]) + delta[i])
                 for i in range(K)]
            wt = sigmoid(M(d["w_logit"][0, t, 0]))
            P = [[S[j][i] * a[i] for i in range(K)] for j in range(V)]
            e = [v[j] - sum(P[j][i] * k[i] for i in range(K)) for j in range(V)]
            S = [[P[j][i] + wt * e[j] * k[i] for i in range(K)] for j in range(V)]
            oc.append([sum(S[j][i] * q[i] for i in range(K)) for j in range(V)])
        prev_mean = [sum(row[j] for row in oc) / len(oc) for j in range(V)]
        o.extend(oc)
    return o, S


@pytest.mark.parametrize("mc_mode", [0, 1])
def test_fp64_evaluation_matches_50_digits(mc_mode):
    mp = pytest.importorskip("mpmath").mp
    mp.dps = 50
    w, d, _, _ = _case(41 + mc_mode, B=1, H=1, T=5, K=3, V=2, R=2, L=2)
    d["g_logit"][0, 1, 0, 0] = 40.0      # a channel erased almost completely in one step
    d["bx"][0, 3, 0, 1] = -40.0
    o_mp, S_mp = _mp_forward(mp, d, w.L, mc_mode)
    ref = oracle.fwd(d, L=w.L, mc_mode=mc_mode)
    o_mp = np.array([[float(x) for x in row] for row in o_mp])
    S_mp = np.array([[float(x) for x in row] for row in S_mp])
    np.testing.assert_allclose(ref["o"][0, :, 0], o_mp, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(ref["S_final"][0, 0], S_mp, rtol=1e-13, atol=1e-15)
