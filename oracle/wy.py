"""Chunked WY-form restatement of the CARVE recurrence, fp64 numpy -- TEST INFRASTRUCTURE ONLY.

A second CPU restatement, independent of `carve_oracle.c` (no shared code): it evaluates
the same recurrence chunk-parallel, the way the pages say the method is trained (CARVE blog,
section 2.3: the key-axis retention gamma lives on the key axis only, so the coupling
matrix M_ts of a chunk is shared by every value channel and one triangular solve U = M^-1 R
serves them all; paperdance abstract: "one unmodified WY-form solve").

Notation per chunk of n tokens with start state S0 (V x K), everything relative to the
chunk (or compute sub-chunk) start:
  l_t      = log a_t = -e^{A_dec} softplus(g_logit_t + tau) - softplus(-(bx_t + Delta))   (key axis;
             A_dec = 0, tau = 0 unless the decay's amplitude and bias are given)
  Lam_t    = sum_{s<=t} l_s            (inclusive cumulative log-retention)
  D[t,s,i] = exp(Lam_t,i - Lam_s,i) for s <= t   (decay from token s to token t)
  Akk[t,s] = sum_i k_t,i k_s,i D[t,s,i]   (s < t)        Aqk[t,s] = sum_i q_t,i k_s,i D[t,s,i]  (s <= t)
  Qt = q*exp(Lam), Kt = k*exp(Lam), Kb = k*exp(Lam_n - Lam)
  (I + Diag(w) Akk) U = Diag(w) (V - Kt S0^T)          -- the WY solve
  O  = Qt S0^T + Aqk U
  S1 = S0 Diag(exp(Lam_n)) + U^T Kb
Row t of U equals w_t (v_t - S_{t-1} Diag(a_t) k_t) of the token-sequential form.

The gate grouping L (which tokens share one content signal) is part of the model; the
compute sub-chunk Lc (any divisor of L) is not: results must agree for every Lc.
"""
from __future__ import annotations

import numpy as np
from scipy.linalg import solve_triangular


def _softplus(x):
    return np.logaddexp(0.0, x)


def _sigmoid(x):
    return 0.5 * (1.0 + np.tanh(0.5 * x))


def _sub_fwd(S0, q, k, v, gl, bx, wl, delta, dec):
    """One compute sub-chunk (dec = (A_dec, tau [K]) of the head).  Returns O, S1 and the
    intermediates the backward needs."""
    n = q.shape[0]
    beta = bx + delta[None, :]
    log_g = -np.exp(dec[0]) * _softplus(gl + dec[1][None, :])
    ell = log_g - _softplus(-beta)
    Lam = np.cumsum(ell, axis=0)
    w = _sigmoid(wl)
    diff = Lam[:, None, :] - Lam[None, :, :]                 # [t,s,i]
    low = np.tril(np.ones((n, n), dtype=bool))
    D = np.where(low[:, :, None], np.exp(np.where(low[:, :, None], diff, 0.0)), 0.0)
    strict = np.tril(np.ones((n, n)), -1)
    Akk = np.einsum("ti,si,tsi->ts", k, k, D) * strict
    Aqk = np.einsum("ti,si,tsi->ts", q, k, D)
    eL = np.exp(Lam)
    Qt, Kt = q * eL, k * eL
    Kb = k * np.exp(Lam[-1][None, :] - Lam)
    M = np.eye(n) + w[:, None] * Akk
    R = v - Kt @ S0.T
    U = solve_triangular(M, w[:, None] * R, lower=True, unit_diagonal=True)
    O = Qt @ S0.T + Aqk @ U
    gam = np.exp(Lam[-1])
    S1 = S0 * gam[None, :] + U.T @ Kb
    return O, S1, dict(beta=beta, log_g=log_g, Lam=Lam, w=w, D=D, Akk=Akk, Aqk=Aqk, Qt=Qt, Kt=Kt, Kb=Kb,
                       M=M, R=R, U=U, gam=gam)


def _content(S, qbar, mprev, A, Bm, mc_mode):
    m = S @ qbar if mc_mode == 0 else mprev.copy()
    z = Bm @ m
    return m, z, A @ z


def _decay(dec, K):
    return (0.0, np.zeros(K)) if dec is None else (float(dec[0]), np.asarray(dec[1], dtype=np.float64))


def fwd_unit(q, k, v, gl, bx, wl, A, Bm, S0, m_prev, L, Lc, mc_mode=0, aw=None, dec=None):
    """One (batch, head) unit: q, k, gl, bx [T,K]; v [T,V]; wl [T]; A [K,R]; Bm [R,V];
    S0 [V,K]; m_prev [V]; aw [R] or None (the write gate's content term: the chunk's write
    logits are shifted by aw . z); dec = (A_dec, tau [K]) or None (the decay's log-amplitude
    and bias).  Returns o [T,V], S_final, m_prev_out."""
    T = q.shape[0]
    dec = _decay(dec, q.shape[1])
    S = S0.copy()
    mprev = m_prev.copy()
    o = np.zeros((T, v.shape[1]))
    for t0 in range(0, T, L):
        t1 = min(t0 + L, T)
        _, z, delta = _content(S, q[t0:t1].mean(axis=0), mprev, A, Bm, mc_mode)
        wls = wl + (0.0 if aw is None else float(aw @ z))
        for s0 in range(t0, t1, Lc):
            s1 = min(s0 + Lc, t1)
            O, S, _ = _sub_fwd(S, q[s0:s1], k[s0:s1], v[s0:s1], gl[s0:s1], bx[s0:s1], wls[s0:s1], delta, dec)
            o[s0:s1] = O
        mprev = o[t0:t1].mean(axis=0)
    return o, S, mprev


def _sub_bwd(S0, q, k, gl, it, dO, dS1, dec):
    """Backward of one compute sub-chunk.  Returns dq, dk, dv, dgl, dbeta, dw_logit, dS0 and
    the sub-chunk's contribution to the gradient of A_dec."""
    Lam, w, D, Akk, Aqk = it["Lam"], it["w"], it["D"], it["Akk"], it["Aqk"]
    Qt, Kt, Kb, M, R, U, gam = it["Qt"], it["Kt"], it["Kb"], it["M"], it["R"], it["U"], it["gam"]
    n = q.shape[0]
    # O = Qt S0^T + Aqk U ;  S1 = S0 Diag(gam) + U^T Kb
    dU = Aqk.T @ dO + Kb @ dS1.T
    dAqk = np.tril(dO @ U.T)
    dQt = dO @ S0
    dS0 = dO.T @ Qt + dS1 * gam[None, :]
    dKb = U @ dS1
    dgam = np.sum(S0 * dS1, axis=0)
    # M U = Diag(w) R
    dY = solve_triangular(M.T, dU, lower=False, unit_diagonal=True)
    dM = -np.tril(dY @ U.T, -1)
    dAkk = w[:, None] * dM
    dw = np.sum(dM * Akk, axis=1) + np.sum(dY * R, axis=1)
    dR = w[:, None] * dY
    dv = dR
    dKt = -dR @ S0
    dS0 -= dR.T @ Kt
    # Akk, Aqk through D = exp(Lam_t - Lam_s)
    dq_a = np.einsum("ts,si,tsi->ti", dAqk, k, D)
    dk_row = np.einsum("ts,si,tsi->ti", dAkk, k, D)
    dk_col = np.einsum("ts,ti,tsi->si", dAqk, q, D) + np.einsum("ts,ti,tsi->si", dAkk, k, D)
    eL = np.exp(Lam)
    eb = np.exp(Lam[-1][None, :] - Lam)
    dq = dq_a + dQt * eL
    dk = dk_row + dk_col + dKt * eL + dKb * eb
    dLam = q * dq_a + k * dk_row - k * dk_col + dQt * Qt + dKt * Kt - dKb * Kb
    dLam[-1] += np.sum(dKb * Kb, axis=0) + dgam * gam
    dell = np.cumsum(dLam[::-1], axis=0)[::-1]
    # log g = -e^{A_dec} softplus(gl + tau): d/dgl = d/dtau = -e^{A_dec} sigmoid(gl + tau),
    # d/dA_dec = log g
    dgl = -np.exp(dec[0]) * _sigmoid(gl + dec[1][None, :]) * dell
    dbeta = _sigmoid(-it["beta"]) * dell
    dwl = dw * w * (1.0 - w)
    return dq, dk, dv, dgl, dbeta, dwl, dS0, float(np.sum(dell * it["log_g"]))


def bwd_unit(q, k, v, gl, bx, wl, A, Bm, S0, m_prev, L, Lc, dO, dS_final, dm_prev_out, mc_mode=0, aw=None,
             dec=None):
    """Reverse sweep over chunks (and compute sub-chunks inside each chunk).
    Returns dq, dk, dv, dgl, dbx, dwl, dA, dB, dS0, dm_prev_in, daw, dA_dec, dtau for one unit."""
    T, K = q.shape
    dec = _decay(dec, K)
    V = v.shape[1]
    # forward: chunk-start states, content signals
    S = S0.copy()
    mprev = m_prev.copy()
    starts, ms, zs, deltas, qbars, wlss = [], [], [], [], [], []
    o = np.zeros((T, V))
    for t0 in range(0, T, L):
        t1 = min(t0 + L, T)
        qbar = q[t0:t1].mean(axis=0)
        m, z, delta = _content(S, qbar, mprev, A, Bm, mc_mode)
        wls = wl + (0.0 if aw is None else float(aw @ z))
        starts.append(S.copy()); ms.append(m); zs.append(z); deltas.append(delta); qbars.append(qbar)
        wlss.append(wls)
        for s0 in range(t0, t1, Lc):
            s1 = min(s0 + Lc, t1)
            O, S, _ = _sub_fwd(S, q[s0:s1], k[s0:s1], v[s0:s1], gl[s0:s1], bx[s0:s1], wls[s0:s1], delta, dec)
            o[s0:s1] = O
        mprev = o[t0:t1].mean(axis=0)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dgl, dbx, dwl = np.zeros_like(gl), np.zeros_like(bx), np.zeros_like(wl)
    dA, dB = np.zeros_like(A), np.zeros_like(Bm)
    daw = np.zeros(A.shape[1])
    da_dec = 0.0
    dS = dS_final.copy()
    dO = dO.copy()
    nch = len(starts)
    if nch:
        t0 = (nch - 1) * L
        dO[t0:] += dm_prev_out[None, :] / (T - t0)
    dm_prev_in = np.zeros(V)
    for c in range(nch - 1, -1, -1):
        t0, t1 = c * L, min(c * L + L, T)
        delta, wls = deltas[c], wlss[c]
        subs = list(range(t0, t1, Lc))
        sub_states, its = [], []
        Sx = starts[c]
        for s0 in subs:
            s1 = min(s0 + Lc, t1)
            sub_states.append(Sx)
            _, Sx, it = _sub_fwd(Sx, q[s0:s1], k[s0:s1], v[s0:s1], gl[s0:s1], bx[s0:s1], wls[s0:s1], delta, dec)
            its.append(it)
        ddelta = np.zeros(K)
        for j in range(len(subs) - 1, -1, -1):
            s0 = subs[j]
            s1 = min(s0 + Lc, t1)
            r = _sub_bwd(sub_states[j], q[s0:s1], k[s0:s1], gl[s0:s1], its[j], dO[s0:s1], dS, dec)
            dq[s0:s1], dk[s0:s1], dv[s0:s1], dgl[s0:s1], dbx[s0:s1], dwl[s0:s1], dS = r[:7]
            da_dec += r[7]
            ddelta += r[4].sum(axis=0)
        dz = A.T @ ddelta
        if aw is not None:   # the chunk's write logits were shifted by aw . z
            ddw = dwl[t0:t1].sum()
            dz = dz + aw * ddw
            daw += ddw * zs[c]
        dA += np.outer(ddelta, zs[c])
        dm = Bm.T @ dz
        dB += np.outer(dz, ms[c])
        if mc_mode == 0:
            dS = dS + np.outer(dm, qbars[c])
            dq[t0:t1] += (starts[c].T @ dm)[None, :] / (t1 - t0)
        elif c > 0:
            dO[(c - 1) * L:c * L] += dm[None, :] / L
        else:
            dm_prev_in = dm
    return dq, dk, dv, dgl, dbx, dwl, dA, dB, dS, dm_prev_in, daw, da_dec, dgl.sum(axis=0)


def _units(inp):
    B, T, H, K = inp["q"].shape
    for b in range(B):
        for h in range(H):
            yield b, h


def _head_decay(f, h, K):
    if "A_dec" not in f and "tau" not in f:
        return None
    return (f["A_dec"][h] if "A_dec" in f else 0.0, f["tau"][h] if "tau" in f else np.zeros(K))


def fwd(inp, L, Lc=None, mc_mode=0, S0=None, m_prev=None):
    """Whole-tensor forward (loops over units).  Same layouts as the C oracle."""
    Lc = L if Lc is None else Lc
    B, T, H, K = inp["q"].shape
    V = inp["v"].shape[-1]
    f = {k: np.asarray(inp[k], dtype=np.float64) for k in inp}
    o = np.zeros((B, T, H, V)); Sf = np.zeros((B, H, V, K)); mo = np.zeros((B, H, V))
    for b, h in _units(inp):
        s0 = np.zeros((V, K)) if S0 is None else np.asarray(S0[b, h], dtype=np.float64)
        mp = np.zeros(V) if m_prev is None else np.asarray(m_prev[b, h], dtype=np.float64)
        o[b, :, h], Sf[b, h], mo[b, h] = fwd_unit(
            f["q"][b, :, h], f["k"][b, :, h], f["v"][b, :, h], f["g_logit"][b, :, h], f["bx"][b, :, h],
            f["w_logit"][b, :, h], f["A"][h], f["B"][h], s0, mp, L, Lc, mc_mode,
            None if "Aw" not in f else f["Aw"][h], _head_decay(f, h, K))
    return dict(o=o, S_final=Sf, m_prev_out=mo)


def bwd(inp, L, dO, Lc=None, mc_mode=0, S0=None, m_prev=None, dS_final=None, dm_prev_out=None):
    Lc = L if Lc is None else Lc
    B, T, H, K = inp["q"].shape
    V = inp["v"].shape[-1]
    f = {k: np.asarray(inp[k], dtype=np.float64) for k in inp}
    out = dict(dq=np.zeros((B, T, H, K)), dk=np.zeros((B, T, H, K)), dv=np.zeros((B, T, H, V)),
               dg_logit=np.zeros((B, T, H, K)), dbx=np.zeros((B, T, H, K)), dw_logit=np.zeros((B, T, H)),
               dA=np.zeros_like(f["A"]), dB=np.zeros_like(f["B"]), dAw=np.zeros(f["A"].shape[::2]),
               dA_dec=np.zeros(H), dtau=np.zeros((H, K)), dS0=np.zeros((B, H, V, K)), dm_prev_in=np.zeros((B, H, V)))
    for b, h in _units(inp):
        s0 = np.zeros((V, K)) if S0 is None else np.asarray(S0[b, h], dtype=np.float64)
        mp = np.zeros(V) if m_prev is None else np.asarray(m_prev[b, h], dtype=np.float64)
        dsf = np.zeros((V, K)) if dS_final is None else np.asarray(dS_final[b, h], dtype=np.float64)
        dmo = np.zeros(V) if dm_prev_out is None else np.asarray(dm_prev_out[b, h], dtype=np.float64)
        r = bwd_unit(f["q"][b, :, h], f["k"][b, :, h], f["v"][b, :, h], f["g_logit"][b, :, h],
                     f["bx"][b, :, h], f["w_logit"][b, :, h], f["A"][h], f["B"][h], s0, mp, L, Lc,
                     np.asarray(dO[b, :, h], dtype=np.float64), dsf, dmo, mc_mode,
                     None if "Aw" not in f else f["Aw"][h], _head_decay(f, h, K))
        (out["dq"][b, :, h], out["dk"][b, :, h], out["dv"][b, :, h], out["dg_logit"][b, :, h],
         out["dbx"][b, :, h], out["dw_logit"][b, :, h]) = r[:6]
        out["dA"][h] += r[6]
        out["dB"][h] += r[7]
        out["dS0"][b, h] = r[8]
        out["dm_prev_in"][b, h] = r[9]
        out["dAw"][h] += r[10]
        if "A_dec" in f:
            out["dA_dec"][h] += r[11]
        if "tau" in f:
            out["dtau"][h] += r[12]
    return out
