"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

Each test ties the oracle to a closed form, a textbook special case, an invariant proved
from the recurrence, an alternative evaluation order named on the pages, or finite
differences, chosen so that a dropped term, a wrong sign, a wrong index or a transposed
operand in the oracle fails at least one of them.
"""
import dataclasses

import numpy as np
import pytest

import oracle
from chunk_gated_delta_b200 import inputs as I

BIG = 800.0  # sigmoid(+BIG) == 1.0 and softplus(-BIG) == 0.0 exactly in fp64


def tiny(B=1, H=2, T=12, K=6, V=5, R=3, L=4, seed=11):
    w = dataclasses.replace(I.TINY_FP32, B=B, H=H, T=T, K=K, V=V, R=R, L=L, seed=seed)
    d = {k: np.asarray(v, dtype=np.float64) for k, v in I.make_inputs(w).items()}
    return w, d


def sig(x):
    return np.exp(-np.logaddexp(0.0, -x))


# ---------------------------------------------------------------------------------------
# 1. Alternative evaluation: transition-matrix form + the (U_b S) qbar fold
# ---------------------------------------------------------------------------------------
def transition_form(d, L, mc_mode):
    """S_t = S_{t-1} Phi_t + w_t v_t k_t^T with Phi_t = Diag(a_t)(I - w_t k_t k_t^T) (the
    delta rule rewritten as an affine map; CARVE blog section 2.1), and the content signal
    folded as (U_b S) qbar with U_b = A B formed explicitly (paperdance abstract:
    U(Sq) = (US)q).  Gates via g = 1/(1+exp(g_logit)), the closed form of
    exp(-softplus(x))."""
    B, T, H, K = d["q"].shape
    V = d["v"].shape[-1]
    o = np.zeros((B, T, H, V))
    Sf = np.zeros((B, H, V, K))
    for b in range(B):
        for h in range(H):
            Ub = d["A"][h] @ d["B"][h]                       # K x V
            S = np.zeros((V, K))
            mprev = np.zeros(V)
            for t0 in range(0, T, L):
                t1 = min(T, t0 + L)
                if mc_mode == 0:
                    delta = (Ub @ S) @ d["q"][b, t0:t1, h].mean(axis=0)
                else:
                    delta = Ub @ mprev
                for t in range(t0, t1):
                    k = d["k"][b, t, h]
                    g = 1.0 / (1.0 + np.exp(d["g_logit"][b, t, h]))
                    a = g * sig(d["bx"][b, t, h] + delta)
                    w = sig(d["w_logit"][b, t, h])
                    Phi = np.diag(a) @ (np.eye(K) - w * np.outer(k, k))
                    S = S @ Phi + w * np.outer(d["v"][b, t, h], k)
                    o[b, t, h] = S @ d["q"][b, t, h]
                mprev = o[b, t0:t1, h].mean(axis=0)
            Sf[b, h] = S
    return o, Sf


@pytest.mark.parametrize("mc_mode", [0, 1])
def test_transition_matrix_form(mc_mode):
    w, d = tiny(T=14, L=4)
    d["A"] *= 40.0
    d["B"] *= 40.0            # make the content path matter
    r = oracle.fwd(d, L=4, mc_mode=mc_mode)
    o, Sf = transition_form(d, 4, mc_mode)
    assert np.abs(r["o"] - o).max() < 1e-12
    assert np.abs(r["S_final"] - Sf).max() < 1e-12
    # the content path is live: switching it off changes the result
    r0 = oracle.fwd(d, L=4, mc_mode=mc_mode, content_off=True)
    assert np.abs(r0["o"] - r["o"]).max() > 1e-6


# ---------------------------------------------------------------------------------------
# 2. Subsumption special cases (CARVE blog Table 1; gist.science summary, Theorem 1)
# ---------------------------------------------------------------------------------------
def test_retention_one_is_plain_delta_rule():
    """a == 1 (g_logit -> -inf, bx -> +inf) reduces CARVE to the delta rule
    S <- S + w (v - S k) k^T (Widrow-Hoff update of a linear associative memory)."""
    w, d = tiny(T=10)
    d["g_logit"][:] = -BIG
    d["bx"][:] = BIG
    S0 = I.make_state(w, 0.3).astype(np.float64)
    r = oracle.fwd(d, L=4, S0=S0)
    for b in range(w.B):
        for h in range(w.H):
            S = S0[b, h].copy()
            for t in range(w.T):
                k, v, q = d["k"][b, t, h], d["v"][b, t, h], d["q"][b, t, h]
                beta = sig(d["w_logit"][b, t, h])
                S = S + beta * np.outer(v - S @ k, k)
                assert np.allclose(r["o"][b, t, h], S @ q, rtol=0, atol=1e-13)
            assert np.allclose(r["S_final"][b, h], S, rtol=0, atol=1e-13)


def test_write_zero_is_pure_decay():
    """w == 0 with U_b = 0: S_t = S0 Diag(prod_{s<=t} a_s), a = sigmoid(-g_logit) sigmoid(bx)."""
    w, d = tiny(T=9)
    d["w_logit"][:] = -BIG
    d["A"][:] = 0.0
    S0 = I.make_state(w, 0.5).astype(np.float64)
    r = oracle.fwd(d, L=4, S0=S0)
    loga = -np.log1p(np.exp(d["g_logit"])) - np.log1p(np.exp(-d["bx"]))     # [B,T,H,K]
    cum = np.cumsum(loga, axis=1)
    for t in range(w.T):
        St = S0 * np.exp(cum[:, t])[:, :, None, :]                      # [B,H,V,K]
        assert np.allclose(r["o"][:, t], np.einsum("bhvk,bhk->bhv", St, d["q"][:, t]), rtol=1e-12, atol=1e-14)
    assert np.allclose(r["S_final"], S0 * np.exp(cum[:, -1])[:, :, None, :], rtol=1e-12, atol=1e-14)


def test_decay_amplitude_and_bias_closed_form():
    """The fused decay (CARVE blog section 2.3: log-decay amplitude A_dec per head, bias tau,
    g <= 0 in the log domain): with w == 0 and U_b = 0,
    S_t = S0 Diag(prod_{s<=t} a_s), log a = -e^{A_dec[h]} log(1 + e^{g_logit + tau[h]}) - log(1 + e^{-bx}).
    Two heads with different amplitudes and biases pin the sign of the amplitude, the bias
    inside the softplus and the head index of both."""
    w, d = tiny(T=9)
    d["w_logit"][:] = -BIG
    d["A"][:] = 0.0
    d["A_dec"] = np.array([np.log(0.5), np.log(3.0)])
    d["tau"] = I.normal(5, 77, (w.H, w.K), 0.0, 1.5)
    S0 = I.make_state(w, 0.5).astype(np.float64)
    r = oracle.fwd(d, L=4, S0=S0)
    amp = np.exp(d["A_dec"])[None, None, :, None]
    loga = -amp * np.log1p(np.exp(d["g_logit"] + d["tau"][None, None])) - np.log1p(np.exp(-d["bx"]))
    cum = np.cumsum(loga, axis=1)
    for t in range(w.T):
        St = S0 * np.exp(cum[:, t])[:, :, None, :]
        assert np.allclose(r["o"][:, t], np.einsum("bhvk,bhk->bhv", St, d["q"][:, t]), rtol=1e-12, atol=1e-14)
    assert np.allclose(r["S_final"], S0 * np.exp(cum[:, -1])[:, :, None, :], rtol=1e-12, atol=1e-14)
    # the parameters matter in this construction
    base = oracle.fwd({k: v for k, v in d.items() if k not in ("A_dec", "tau")}, L=4, S0=S0)
    assert np.abs(base["S_final"] - r["S_final"]).max() > 1e-3


def test_exact_write_with_unit_keys():
    """w == 1, a == 1, ||k|| = 1: the delta rule stores v_t exactly under k_t, S_t k_t = v_t."""
    w, d = tiny(T=7, V=4)
    d["w_logit"][:] = BIG
    d["g_logit"][:] = -BIG
    d["bx"][:] = BIG
    d["k"] /= np.linalg.norm(d["k"], axis=-1, keepdims=True)   # unit norm in fp64
    for t in range(1, w.T + 1):
        r = oracle.fwd({k: (v[:, :t] if v.ndim >= 3 and k not in ("A", "B") else v) for k, v in d.items()}, L=4)
        Sk = np.einsum("bhvk,bhk->bhv", r["S_final"], d["k"][:, t - 1])
        assert np.abs(Sk - d["v"][:, t - 1]).max() < 1e-13


def test_orthogonal_keys_give_linear_attention():
    """With a == 1, w == 1, S0 = 0 and mutually orthogonal unit keys the delta correction
    vanishes and o_t = sum_{s<=t} v_s (k_s . q_t): linear attention."""
    w, d = tiny(T=6, K=6, L=3)
    d["w_logit"][:] = BIG
    d["g_logit"][:] = -BIG
    d["bx"][:] = BIG
    rng = np.random.default_rng(3)
    Q, _ = np.linalg.qr(rng.standard_normal((6, 6)))
    for b in range(w.B):
        for h in range(w.H):
            d["k"][b, :, h] = Q.T[rng.permutation(6)]
    r = oracle.fwd(d, L=3)
    for t in range(w.T):
        att = np.einsum("bshk,bhk->bsh", d["k"][:, :t + 1], d["q"][:, t])
        ref = np.einsum("bsh,bshv->bhv", att, d["v"][:, :t + 1])
        assert np.abs(r["o"][:, t] - ref).max() < 1e-13


# ---------------------------------------------------------------------------------------
# 3. Zero-initialised content projection (CARVE blog section 2.2 and Table 2;
#    paperdance abstract: bit-identical to the baseline at init)
# ---------------------------------------------------------------------------------------
@pytest.mark.parametrize("mc_mode", [0, 1])
@pytest.mark.parametrize("zero", ["A", "B"])
def test_zero_projection_is_bit_identical(mc_mode, zero):
    w, d = tiny(T=13, L=4)
    d[zero][:] = 0.0
    S0 = I.make_state(w, 0.2).astype(np.float64)
    r = oracle.fwd(d, L=4, mc_mode=mc_mode, S0=S0)
    base = oracle.fwd(d, L=4, mc_mode=mc_mode, S0=S0, content_off=True)
    assert np.array_equal(r["o"], base["o"])
    assert np.array_equal(r["S_final"], base["S_final"])


@pytest.mark.parametrize("mc_mode", [0, 1])
def test_zero_write_projection_is_bit_identical(mc_mode):
    """Aw = 0 (zero-initialised, like U_b): sigmoid(w_logit + 0) = sigmoid(w_logit) exactly, so
    the forward and every backward output equal those without the write term, bit for bit,
    and d(Aw) is still the true gradient (compared against finite differences elsewhere)."""
    w, d = tiny(T=13, L=4)
    d["A"] *= 30.0
    d["B"] *= 30.0
    S0 = I.make_state(w, 0.2).astype(np.float64)
    dO = I.normal(8, 1, (w.B, w.T, w.H, w.V))
    dz = dict(d, Aw=np.zeros((w.H, w.R)))
    r, base = oracle.fwd(dz, L=4, mc_mode=mc_mode, S0=S0), oracle.fwd(d, L=4, mc_mode=mc_mode, S0=S0)
    for key in r:
        assert np.array_equal(r[key], base[key]), key
    g, gb = oracle.bwd(dz, 4, dO, mc_mode=mc_mode, S0=S0), oracle.bwd(d, 4, dO, mc_mode=mc_mode, S0=S0)
    for key in g:
        if key != "dAw":
            assert np.array_equal(g[key], gb[key]), key
    assert np.all(gb["dAw"] == 0.0) and np.abs(g["dAw"]).max() > 0.0


@pytest.mark.parametrize("mc_mode", [0, 1])
def test_zero_decay_parameters_are_bit_identical(mc_mode):
    """A_dec = 0 and tau = 0: e^0 softplus(g_logit + 0) is exactly softplus(g_logit), so every
    output equals the run without the parameters bit for bit; their gradients are the true
    ones (finite differences elsewhere), and d tau = sum over batch and tokens of d g_logit
    because tau enters only through g_logit + tau."""
    w, d = tiny(B=2, T=13, L=4)
    d["A"] *= 30.0
    d["B"] *= 30.0
    S0 = I.make_state(w, 0.2).astype(np.float64)
    dO = I.normal(8, 2, (w.B, w.T, w.H, w.V))
    dz = dict(d, A_dec=np.zeros(w.H), tau=np.zeros((w.H, w.K)))
    r, base = oracle.fwd(dz, L=4, mc_mode=mc_mode, S0=S0), oracle.fwd(d, L=4, mc_mode=mc_mode, S0=S0)
    for key in r:
        assert np.array_equal(r[key], base[key]), key
    g, gb = oracle.bwd(dz, 4, dO, mc_mode=mc_mode, S0=S0), oracle.bwd(d, 4, dO, mc_mode=mc_mode, S0=S0)
    for key in g:
        if key not in ("dA_dec", "dtau"):
            assert np.array_equal(g[key], gb[key]), key
    assert np.all(gb["dA_dec"] == 0.0) and np.all(gb["dtau"] == 0.0)
    assert np.abs(g["dA_dec"]).min() > 0.0
    np.testing.assert_allclose(g["dtau"], g["dg_logit"].sum(axis=(0, 1)), rtol=1e-12, atol=1e-15)


def test_chunk_size_enters_only_through_the_content_signal():
    """With U_b = 0 the gate grouping is irrelevant: every L gives the same bits."""
    w, d = tiny(T=16)
    d["A"][:] = 0.0
    ref = oracle.fwd(d, L=1)
    for L in (3, 4, 16, 40):
        r = oracle.fwd(d, L=L)
        assert np.array_equal(r["o"], ref["o"]) and np.array_equal(r["S_final"], ref["S_final"])
    d2 = dict(d)
    d2["A"] = tiny(T=16)[1]["A"] * 50
    assert np.abs(oracle.fwd(d2, L=1)["o"] - oracle.fwd(d2, L=4)["o"]).max() > 1e-8


# ---------------------------------------------------------------------------------------
# 4. The content signal in closed form (which state, which mean, which factor order)
# ---------------------------------------------------------------------------------------
@pytest.mark.parametrize("mc_mode", [0, 1])
@pytest.mark.parametrize("write_term", [False, True])
def test_content_signal_closed_form(mc_mode, write_term):
    """Chunk 0 (L = 4 tokens) with a == 1, w == 1 and keys e_0..e_3 gives
    S_[0] = sum_t v_t e_t^T and o_t = sum_{s<=t} v_s q_t[s] in closed form.  The first token
    of chunk 1 (ragged: 3 tokens) then sees m_1 = S_[0] mean(q over chunk 1) (mode 0:
    boundary state, mean over the CURRENT chunk incl. later tokens; paperdance abstract)
    or m_1 = mean(o over chunk 0) (mode 1; CARVE blog section 2.2), Delta = A (B m_1), and
    with the write gate's content term w = sigmoid(w_logit + Aw . (B m_1)) (the same
    low-rank projection of m_1 gives the erase and the write bias, blog section 2.2)."""
    K = V = 5
    w, d = tiny(B=1, H=1, T=7, K=K, V=V, R=2, L=4)
    d["A"] *= 60.0
    d["B"] *= 60.0
    if write_term:
        d["Aw"] = np.array([[25.0, -40.0]])
    d["w_logit"][:, :4] = BIG
    d["g_logit"][:, :4] = -BIG
    d["bx"][:, :4] = BIG
    for t in range(4):
        d["k"][0, t, 0] = np.eye(K)[t]
    r = oracle.fwd(d, L=4, mc_mode=mc_mode)
    vv, qq = d["v"][0, :, 0], d["q"][0, :, 0]
    S0 = sum(np.outer(vv[t], np.eye(K)[t]) for t in range(4))
    o0 = np.array([sum(vv[s] * qq[t][s] for s in range(t + 1)) for t in range(4)])
    assert np.abs(r["o"][0, :4, 0] - o0).max() < 1e-13
    m = S0 @ qq[4:7].mean(axis=0) if mc_mode == 0 else o0.mean(axis=0)
    z = d["B"][0] @ m
    delta = d["A"][0] @ z
    k, t = d["k"][0, 4, 0], 4
    a = sig(-d["g_logit"][0, t, 0]) * sig(d["bx"][0, t, 0] + delta)
    wt = sig(d["w_logit"][0, t, 0] + (d["Aw"][0] @ z if write_term else 0.0))
    if write_term:   # the term matters in this construction
        assert abs(wt - sig(d["w_logit"][0, t, 0])) > 1e-3
    e = vv[t] - S0 @ (a * k)
    S1 = S0 * a[None, :] + wt * np.outer(e, k)
    assert np.abs(r["o"][0, 4, 0] - S1 @ qq[4]).max() < 1e-13
    # a plausible slip -- reading the state after the first token -- is distinguishable
    assert np.abs(delta).max() > 1e-3


# ---------------------------------------------------------------------------------------
# 5. Lyapunov-type bound (CARVE blog section 2.3; gist.science Theorem 4), derived:
#    ||k|| = 1, w in [0,1], a in (0,1]  =>  ||S_t||_F <= max_i a_t,i ||S_{t-1}||_F + w_t ||v_t||
# ---------------------------------------------------------------------------------------
def test_state_norm_bound_every_token():
    w = dataclasses.replace(I.TINY_FP32, B=2, H=2, T=200, K=16, V=12, R=4, L=1, seed=5)
    d = {k: np.asarray(v, dtype=np.float64) for k, v in I.make_inputs(w).items()}
    d["A"] *= 30.0
    d["B"] *= 30.0
    S = I.make_state(w, 1.0).astype(np.float64)
    A, Bm = d["A"], d["B"]
    worst = -np.inf
    for t in range(w.T):
        tok = {k: d[k][:, t] for k in ("q", "k", "v", "g_logit", "bx", "w_logit")}
        Sprev = S.copy()
        m = np.einsum("bhvk,bhk->bhv", Sprev, tok["q"])
        delta = np.einsum("hkr,bhr->bhk", A, np.einsum("hrv,bhv->bhr", Bm, m))
        amax = (sig(-tok["g_logit"]) * sig(tok["bx"] + delta)).max(axis=-1)
        oracle.step(tok, A, Bm, S, L=1)
        lhs = np.linalg.norm(S, axis=(2, 3))
        rhs = amax * np.linalg.norm(Sprev, axis=(2, 3)) + sig(tok["w_logit"]) * np.linalg.norm(tok["v"], axis=-1)
        worst = max(worst, float((lhs - rhs).max()))
    assert worst <= 1e-12


# ---------------------------------------------------------------------------------------
# 6. Decode step == sequence forward (L = 1 readout in mode 0; running block mean in mode 1)
# ---------------------------------------------------------------------------------------
@pytest.mark.parametrize("mc_mode,L", [(0, 1), (1, 3)])
@pytest.mark.parametrize("decay", [False, True])
def test_step_equals_sequence(mc_mode, L, decay):
    w, d = tiny(T=11, L=L)
    d["A"] *= 40.0
    d["B"] *= 40.0
    dec = {}
    if decay:
        dec = {k: np.asarray(v, dtype=np.float64) for k, v in I.make_decay(w).items()}
        d.update(dec)
    S0 = I.make_state(w, 0.3).astype(np.float64)
    mp = I.normal(9, 1, (w.B, w.H, w.V))
    r = oracle.fwd(d, L=L, mc_mode=mc_mode, S0=S0, m_prev=mp)
    S = S0.copy()
    ms = np.zeros((w.B, w.H, 2, w.V))
    ms[:, :, 1] = mp
    pos = np.zeros((w.B, w.H), dtype=np.int32)
    for t in range(w.T):
        tok = {k: d[k][:, t] for k in ("q", "k", "v", "g_logit", "bx", "w_logit")}
        o = oracle.step(tok, d["A"], d["B"], S, L=L, mc_mode=mc_mode, mstate=ms, pos=pos, **dec)
        assert np.abs(o - r["o"][:, t]).max() < 1e-12
    assert np.abs(S - r["S_final"]).max() < 1e-12
    assert np.all(pos == w.T)


# ---------------------------------------------------------------------------------------
# 7. Gradients: central finite differences of the forward (every input, both modes)
# ---------------------------------------------------------------------------------------
@pytest.mark.parametrize("mc_mode", [0, 1])
def test_gradients_central_differences(mc_mode):
    w, d = tiny(B=2, H=1, T=7, K=3, V=3, R=2, L=3, seed=21)
    d["A"] *= 30.0
    d["B"] *= 30.0
    d["Aw"] = I.normal(21, 9, (w.H, w.R), 0.0, 3.0)
    d["A_dec"] = np.array([0.7])
    d["tau"] = I.normal(21, 10, (w.H, w.K), 0.0, 1.0)
    S0 = I.make_state(w, 0.4).astype(np.float64)
    mp = I.normal(3, 3, (w.B, w.H, w.V))
    dO = I.normal(4, 4, (w.B, w.T, w.H, w.V))
    dSf = I.normal(4, 5, (w.B, w.H, w.V, w.K))
    dmo = I.normal(4, 6, (w.B, w.H, w.V))

    def loss(dd, s0, m0):
        r = oracle.fwd(dd, L=3, mc_mode=mc_mode, S0=s0, m_prev=m0)
        return np.sum(dO * r["o"]) + np.sum(dSf * r["S_final"]) + np.sum(dmo * r["m_prev_out"])

    g = oracle.bwd(d, 3, dO, mc_mode=mc_mode, S0=S0, m_prev=mp, dS_final=dSf, dm_prev_out=dmo)
    eps = 1e-6
    names = [("q", "dq"), ("k", "dk"), ("v", "dv"), ("g_logit", "dg_logit"), ("bx", "dbx"),
             ("w_logit", "dw_logit"), ("A", "dA"), ("B", "dB"), ("Aw", "dAw"), ("A_dec", "dA_dec"),
             ("tau", "dtau"), ("S0", "dS0"),
             ("m_prev", "dm_prev_in")]
    for x, gx in names:
        base = S0 if x == "S0" else mp if x == "m_prev" else d[x]
        num = np.zeros_like(base)
        for idx in np.ndindex(base.shape):
            vals = []
            for sgn in (1, -1):
                pert = base.copy()
                pert[idx] += sgn * eps
                if x == "S0":
                    vals.append(loss(d, pert, mp))
                elif x == "m_prev":
                    vals.append(loss(d, S0, pert))
                else:
                    dd = dict(d)
                    dd[x] = pert
                    vals.append(loss(dd, S0, mp))
            num[idx] = (vals[0] - vals[1]) / (2 * eps)
        err = np.abs(num - g[gx]).max() / max(np.abs(num).max(), 1e-3)
        assert err < 1e-6, (x, err)
    if mc_mode == 0:
        assert np.all(g["dm_prev_in"] == 0.0)


# ---------------------------------------------------------------------------------------
# 8. Packed variable-length sequences: each sequence is an independent recurrence with its own
#    state, content signal and chunk grid (chunks restart at its first token)
# ---------------------------------------------------------------------------------------
def packed_case(lens, seed, H=2, K=6, V=5, R=3):
    """Sequences of the given lengths, drawn separately, and their packing along the token axis."""
    seqs = []
    for n, T in enumerate(lens):
        w = dataclasses.replace(I.TINY_FP32, B=1, H=H, T=T, K=K, V=V, R=R, L=4, seed=seed + n)
        d = {k: np.asarray(v, dtype=np.float64) for k, v in I.make_inputs(w).items()}
        seqs.append(d)
    shared = {k: seqs[0][k] * 40.0 for k in ("A", "B")}
    for d in seqs:
        d.update(shared)
    Ttot = sum(lens) + 3   # three trailing rows that belong to no sequence
    packed = dict(shared)
    for k in ("q", "k", "v", "g_logit", "bx", "w_logit"):
        tail = np.full((1, 3) + seqs[0][k].shape[2:], 7.0)
        packed[k] = np.concatenate([d[k] for d in seqs] + [tail], axis=1)
        assert packed[k].shape[1] == Ttot
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return seqs, packed, cu


@pytest.mark.parametrize("mc_mode", [0, 1])
def test_packed_sequences_equal_separate_calls(mc_mode):
    """Forward and backward over packed sequences (lengths with an empty one, a one-token one,
    ragged last chunks) give, bit for bit, what separate calls give per sequence; dA and dB
    are the per-sequence sums in order; rows past the last sequence stay zero."""
    lens = [7, 0, 13, 1, 8]
    seqs, packed, cu = packed_case(lens, 300 + mc_mode)
    N, H, K, V = len(lens), 2, 6, 5
    S0 = I.normal(9, 10, (N, H, V, K), 0.0, 0.3)
    mp = I.normal(9, 11, (N, H, V))
    dO = I.normal(9, 12, (1, cu[-1] + 3, H, V))
    dSf = I.normal(9, 13, (N, H, V, K))
    dmo = I.normal(9, 14, (N, H, V))
    r = oracle.fwd(packed, L=4, mc_mode=mc_mode, S0=S0, m_prev=mp, cu_seqlens=cu)
    g = oracle.bwd(packed, 4, dO, mc_mode=mc_mode, S0=S0, m_prev=mp, dS_final=dSf, dm_prev_out=dmo, cu_seqlens=cu)
    dA = np.zeros_like(packed["A"])
    dB = np.zeros_like(packed["B"])
    for n, d in enumerate(seqs):
        a, b = cu[n], cu[n + 1]
        if b == a:   # an empty sequence passes its state and content signal through
            assert np.array_equal(r["S_final"][n], S0[n]) and np.array_equal(r["m_prev_out"][n], mp[n])
            assert np.array_equal(g["dS0"][n], dSf[n])
            assert np.array_equal(g["dm_prev_in"][n], dmo[n])
            continue
        rs = oracle.fwd(d, L=4, mc_mode=mc_mode, S0=S0[n:n + 1], m_prev=mp[n:n + 1])
        gs = oracle.bwd(d, 4, dO[:, a:b], mc_mode=mc_mode, S0=S0[n:n + 1], m_prev=mp[n:n + 1],
                        dS_final=dSf[n:n + 1], dm_prev_out=dmo[n:n + 1])
        assert np.array_equal(r["o"][:, a:b], rs["o"])
        assert np.array_equal(r["S_final"][n], rs["S_final"][0])
        assert np.array_equal(r["m_prev_out"][n], rs["m_prev_out"][0])
        for key in ("dq", "dk", "dv", "dg_logit", "dbx", "dw_logit"):
            assert np.array_equal(g[key][:, a:b], gs[key]), key
        for key in ("dS0", "dm_prev_in"):
            assert np.array_equal(g[key][n], gs[key][0]), key
        dA += gs["dA"]
        dB += gs["dB"]
    assert np.array_equal(g["dA"], dA) and np.array_equal(g["dB"], dB)
    assert np.all(r["o"][:, cu[-1]:] == 0.0) and np.all(g["dq"][:, cu[-1]:] == 0.0)


def test_packed_sequences_rejected_when_malformed():
    _, packed, cu = packed_case([4, 4], 310)
    for bad in ([1, 4, 8], [0, 5, 4], [0, 4, 100]):
        with pytest.raises(ValueError):
            oracle.fwd(packed, L=4, cu_seqlens=np.array(bad))
