"""GPU (libcarve.so through its C ABI) against the fp64 oracle, element by element.

Tolerance: relative L2 over each whole tensor, 1e-5 with fp32 I/O and 2e-2 with bf16
q/k/v/o (fp32 gates, state and accumulation).  The oracle reads the bf16-rounded inputs
exactly.  Full-size workloads are compared on sampled (batch, head) units, which are
independent except for dA/dB (sampled heads keep every batch element so those sums are
exact).
"""
import dataclasses

import numpy as np
import pytest

import chunk_gated_delta_b200 as carve
import oracle
from chunk_gated_delta_b200 import inputs as I
from tests.helpers import TOL, host, rel_l2, sub_units, to_dev

pytestmark = pytest.mark.gpu

GRADS = ("dq", "dk", "dv", "dg_logit", "dbx", "dw_logit", "dA", "dB")


def gpu_fwd(dev, dd, L, mode, S0=None, mp=None, save=True):
    return carve.carve_fwd(dd["q"], dd["k"], dd["v"], dd["g_logit"], dd["bx"], dd["w_logit"], dd["A"], dd["B"],
                           chunk=L, mc_mode=mode, S0=S0, m_prev_in=mp, save_for_bwd=save)


def gpu_bwd(dd, saved, L, mode, dS_final=None, dm_prev_out=None):
    return carve.carve_bwd(dd["q"], dd["k"], dd["v"], dd["g_logit"], dd["bx"], dd["w_logit"], dd["A"], dd["B"],
                           saved, dd["dO"], chunk=L, mc_mode=mode, dS_final=dS_final, dm_prev_out=dm_prev_out)


def check(name, got, ref, tol):
    e = rel_l2(got, ref)
    assert e <= tol, f"{name}: rel-L2 {e:.3e} > {tol:.1e}"
    return e


def run_case(cuda_device, w, d, dO, L, mode, S0=None, mp=None, dSf=None, dmo=None, units=None, bwd=True):
    """GPU fwd(+bwd) on the whole workload; oracle on `units` = (bs, hs) (all by default)."""
    import torch
    dd = to_dev(d if dO is None else dict(d, dO=dO), w.io, cuda_device)
    tS0 = None if S0 is None else torch.from_numpy(S0).to(cuda_device)
    tmp = None if mp is None else torch.from_numpy(mp).to(cuda_device)
    out = gpu_fwd(cuda_device, dd, L, mode, tS0, tmp, save=bwd)
    g = None
    if bwd:
        tdS = None if dSf is None else torch.from_numpy(dSf).to(cuda_device)
        tdm = None if dmo is None else torch.from_numpy(dmo).to(cuda_device)
        g = gpu_bwd(dd, out["saved"], L, mode, tdS, tdm)
    torch.cuda.synchronize()
    bs, hs = units if units is not None else (slice(None), slice(None))
    od = sub_units(d, bs, hs)
    sl = lambda x: None if x is None else x[bs][:, hs]   # noqa: E731
    r = oracle.fwd(od, L=L, mc_mode=mode, S0=sl(S0), m_prev=sl(mp))
    tol = TOL[w.io]
    errs = {}
    errs["o"] = check("o", host(out["o"])[bs][:, :, hs], r["o"], tol)
    errs["S_final"] = check("S_final", host(out["S_final"])[bs][:, hs], r["S_final"], tol)
    errs["m_prev_out"] = check("m_prev_out", host(out["m_prev_out"])[bs][:, hs], r["m_prev_out"], tol)
    if bwd:
        rg = oracle.bwd(od, L, dO[bs][:, :, hs], mc_mode=mode, S0=sl(S0), m_prev=sl(mp), dS_final=sl(dSf),
                        dm_prev_out=sl(dmo))
        for key in GRADS:
            gk = host(g[key])
            gk = gk[hs] if key in ("dA", "dB") else gk[bs][:, :, hs]
            errs[key] = check(key, gk, rg[key], tol)
        errs["dS0"] = check("dS0", host(g["dS0"])[bs][:, hs], rg["dS0"], tol)
        if mode == 1:
            errs["dm_prev_in"] = check("dm_prev_in", host(g["dm_prev_in"])[bs][:, hs], rg["dm_prev_in"], tol)
    return errs


def small(w, **kw):
    w = dataclasses.replace(w, **kw)
    d = I.make_inputs(w)
    dO = I.make_grad_out(w)
    return w, d, dO


# ---------------------------------------------------------------------------------------
# tiny fp32 workload (B1 H2 T256 d64 L64, rank 16): forward and backward at 1e-5
# ---------------------------------------------------------------------------------------
@pytest.mark.parametrize("mode", [0, 1])
def test_tiny_fp32(cuda_device, mode):
    w, d, dO = small(I.TINY_FP32)
    errs = run_case(cuda_device, w, d, dO, w.L, mode)
    print(w.name, mode, {k: f"{v:.2e}" for k, v in errs.items()})


@pytest.mark.parametrize("mode", [0, 1])
def test_tiny_fp32_carried_state_and_signal(cuda_device, mode):
    """Non-zero S0, m_prev_in, dS_final and dm_prev_out, a ragged last chunk (T = 80, L = 32)."""
    w, d, dO = small(I.TINY_FP32, T=80, L=32, seed=77)
    d["A"] *= 10.0
    d["B"] *= 10.0
    S0 = I.make_state(w, 0.1)
    mp = I.normal(1, 2, (w.B, w.H, w.V)).astype(np.float32)
    dSf = I.normal(1, 3, (w.B, w.H, w.V, w.K)).astype(np.float32)
    dmo = I.normal(1, 4, (w.B, w.H, w.V)).astype(np.float32)
    run_case(cuda_device, w, d, dO, 32, mode, S0=S0, mp=mp, dSf=dSf, dmo=dmo)


@pytest.mark.parametrize("K,V", [(64, 128), (128, 64), (128, 128)])
@pytest.mark.parametrize("io", ["fp32", "bf16"])
def test_shapes_and_dtypes(cuda_device, K, V, io):
    w, d, dO = small(I.TINY_FP32, B=2, H=3, T=96, K=K, V=V, R=8, L=32, io=io, seed=K + V)
    d["A"] *= 10.0
    d["B"] *= 10.0
    for mode in (0, 1):
        run_case(cuda_device, w, d, dO, 32, mode)


@pytest.mark.parametrize("L", [16, 32, 64, 128])
def test_chunk_lengths_bf16(cuda_device, L):
    w, d, dO = small(I.FWD_1P3B, B=1, H=4, T=384, L=L, seed=5 + L)
    d["A"] *= 10.0
    d["B"] *= 10.0
    for mode in (0, 1):
        run_case(cuda_device, w, d, dO, L, mode)


@pytest.mark.parametrize("T,L", [(352, 64), (352, 128), (320, 128), (448, 64)])
def test_saved_state_paths_bf16(cuda_device, T, L):
    """Gate chunks of 64 and 128 tokens over the 32-token chunks that the training path saves
    and reverses, with T a multiple of 64 or only of 32 (gate chunks of 128 may end ragged).
    Carried S0, m_prev_in, dS_final and dm_prev_out."""
    w, d, dO = small(I.FWD_1P3B, B=1, H=3, T=T, L=L, seed=T + L)
    d["A"] *= 10.0
    d["B"] *= 10.0
    S0 = I.make_state(w, 0.05)
    mp = I.normal(2, 2, (w.B, w.H, w.V)).astype(np.float32)
    dSf = I.normal(2, 3, (w.B, w.H, w.V, w.K)).astype(np.float32)
    dmo = I.normal(2, 4, (w.B, w.H, w.V)).astype(np.float32)
    for mode in (0, 1):
        run_case(cuda_device, w, d, dO, L, mode, S0=S0, mp=mp, dSf=dSf, dmo=dmo)


def test_zero_projection_is_chunk_length_invariant(cuda_device):
    """U_b = 0 (A = 0): the erase gate is sigmoid(bx + 0) = sigmoid(bx) exactly, so the gate
    grouping L cannot matter.  Kernels that split the sequence into the same compute chunks
    (L = 64 and 128 on the tensor-core path, both readouts) agree bitwise; every L agrees with
    the oracle's key-axis baseline (content path removed) within tolerance."""
    import torch
    w, d, dO = small(I.FWD_1P3B, B=2, H=2, T=256, seed=9)
    d["A"][:] = 0.0
    dd = to_dev(d, w.io, cuda_device)
    same = [gpu_fwd(cuda_device, dd, 64, 0, save=False), gpu_fwd(cuda_device, dd, 128, 0, save=False),
            gpu_fwd(cuda_device, dd, 64, 1, save=False), gpu_fwd(cuda_device, dd, 128, 1, save=False)]
    torch.cuda.synchronize()
    for x in same[1:]:
        assert torch.equal(x["o"], same[0]["o"]) and torch.equal(x["S_final"], same[0]["S_final"])
    base = oracle.fwd(d, L=64, content_off=True)
    for L in (16, 32, 64, 128):
        for save in (False, True):
            x = gpu_fwd(cuda_device, dd, L, 0, save=save)
            check(f"o L={L} save={save}", host(x["o"]), base["o"], TOL["bf16"])
            check(f"S L={L} save={save}", host(x["S_final"]), base["S_final"], TOL["bf16"])


@pytest.mark.parametrize("mode", [0, 1])
def test_chaining_is_bitwise(cuda_device, mode):
    """fwd(T) == fwd(first half) then fwd(second half) carrying S and m (checkpoint/resume)."""
    import torch
    w, d, dO = small(I.FWD_1P3B, B=2, H=3, T=512, seed=31)
    d["A"] *= 10.0
    d["B"] *= 10.0
    dd = to_dev(d, w.io, cuda_device)
    full = gpu_fwd(cuda_device, dd, 64, mode, save=False)
    half = {k: (v[:, :256].contiguous() if v.dim() >= 3 and k not in ("A", "B") else v) for k, v in dd.items()}
    rest = {k: (v[:, 256:].contiguous() if v.dim() >= 3 and k not in ("A", "B") else v) for k, v in dd.items()}
    a = gpu_fwd(cuda_device, half, 64, mode, save=False)
    b = gpu_fwd(cuda_device, rest, 64, mode, S0=a["S_final"], mp=a["m_prev_out"], save=False)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat([a["o"], b["o"]], dim=1), full["o"])
    assert torch.equal(b["S_final"], full["S_final"])
    assert torch.equal(b["m_prev_out"], full["m_prev_out"])


# ---------------------------------------------------------------------------------------
# full-size workloads
# ---------------------------------------------------------------------------------------
def test_fwd_1p3b_layer(cuda_device):
    """B4 H16 T2048 d128 L64 rank 32, bf16 forward; 8 sampled units."""
    w = I.FWD_1P3B
    d = I.make_inputs(w)
    errs = run_case(cuda_device, w, d, None, w.L, 0, units=([0, 3], [0, 5, 10, 15]), bwd=False)
    print(w.name, {k: f"{v:.2e}" for k, v in errs.items()})


def test_train_1p3b_layer(cuda_device):
    """B8 H16 T4096 d128 L64 rank 32, bf16 forward + backward; heads 0 and 9 (every batch)."""
    w = I.TRAIN_1P3B
    d = I.make_inputs(w)
    dO = I.make_grad_out(w)
    errs = run_case(cuda_device, w, d, dO, w.L, 0, units=(list(range(w.B)), [0, 9]))
    print(w.name, {k: f"{v:.2e}" for k, v in errs.items()})


@pytest.fixture(scope="module")
def long_inputs():
    w = I.long_context(64, 0)
    return I.make_inputs(w), I.make_grad_out(w)


@pytest.mark.parametrize("L", [32, 64, 128])
@pytest.mark.parametrize("mode", [0, 1])
def test_long_context(cuda_device, long_inputs, L, mode):
    """B1 H16 T65536 d128, bf16 forward + backward at L in {32, 64, 128}, both readouts;
    one sampled head (the oracle is sequential per unit)."""
    w = I.long_context(L, mode)
    d, dO = long_inputs
    errs = run_case(cuda_device, w, d, dO, L, mode, units=([0], [3]))
    print(w.name, {k: f"{v:.2e}" for k, v in errs.items()})


@pytest.mark.parametrize("mode", [0, 1])
def test_decode_1000_steps(cuda_device, mode):
    """B256 H16 d128: 1000 consecutive decode steps, fp32 state ~ N(0, 0.05^2) in place,
    bf16 q/k/v, per-token gates (a pool of 64 seeded token sets cycled).  Six sampled units
    are replayed by the oracle step by step; every step's output and the final state are
    compared."""
    import torch
    w = I.DECODE
    L = 64
    pool = I.make_decode_pool(w, pool=64)
    S_np = I.make_state(w, 0.05)
    dev = cuda_device
    tp = to_dev({k: pool[k] for k in ("q", "k", "v", "g_logit", "bx", "w_logit")}, "bf16", dev)
    A = torch.from_numpy(pool["A"]).to(dev)
    Bm = torch.from_numpy(pool["B"]).to(dev)
    S = torch.from_numpy(S_np).to(dev)
    mstate = torch.zeros((w.B, w.H, 2, w.V), dtype=torch.float32, device=dev)
    pos = torch.zeros((w.B, w.H), dtype=torch.int32, device=dev)
    units = [(0, 0), (17, 3), (100, 8), (128, 15), (200, 1), (255, 12)]
    bi = [u[0] for u in units]
    hi = [u[1] for u in units]
    outs = []
    for j in range(w.steps):
        p = j % 64
        o = carve.carve_step(tp["q"][p], tp["k"][p], tp["v"][p], tp["g_logit"][p], tp["bx"][p], tp["w_logit"][p], A,
                             Bm, S, mc_mode=mode, chunk=L, mstate=mstate, pos=pos)
        outs.append(o[bi, hi].float())
    torch.cuda.synchronize()
    go = torch.stack(outs).cpu().numpy()
    # oracle: the same units, token by token
    Sr = S_np[bi, hi][:, None].astype(np.float64).copy()          # [6,1,V,K]
    A_r = pool["A"][hi][:, None]                                    # per-unit head factors
    ms = np.zeros((len(units), 1, 2, w.V))
    ps = np.zeros((len(units), 1), dtype=np.int32)
    ref = np.zeros_like(go)
    for n, (b, h) in enumerate(units):
        Sn = Sr[n:n + 1]
        msn, psn = ms[n:n + 1], ps[n:n + 1]
        for j in range(w.steps):
            p = j % 64
            tok = {k: pool[k][p][b:b + 1, h:h + 1] for k in ("q", "k", "v", "g_logit", "bx", "w_logit")}
            tok = {k: np.asarray(v, dtype=np.float64) for k, v in tok.items()}
            ref[j, n] = oracle.step(tok, A_r[n], pool["B"][h][None], Sn, L=L, mc_mode=mode, mstate=msn, pos=psn)[0, 0]
    check("o (all steps)", go, ref, TOL["bf16"])
    check("S after 1000 steps", host(S)[bi, hi], Sr[:, 0], TOL["bf16"])
    if mode == 1:
        assert torch.all(pos == w.steps)


@pytest.mark.parametrize("K,V", [(64, 64), (64, 128), (128, 64), (128, 128)])
@pytest.mark.parametrize("io", ["fp32", "bf16"])
def test_decode_shapes_all_units(cuda_device, K, V, io):
    """336 (b,h) units (more than one per SM, so every CTA cycles its state stages), rank 48
    (two passes of the z product), 40 steps in each mode (mc_mode 1 with 4-token blocks);
    every unit's outputs and final state against the oracle."""
    import torch
    w = dataclasses.replace(I.DECODE, B=3, H=112, K=K, V=V, R=48, io=io, seed=900 + K + V)
    steps, L = 40, 4
    pool = I.make_decode_pool(w, pool=steps)
    for mode in (0, 1):
        S_np = I.make_state(w, 0.05)
        tp = to_dev({k: pool[k] for k in ("q", "k", "v", "g_logit", "bx", "w_logit")}, io, cuda_device)
        A = torch.from_numpy(pool["A"]).to(cuda_device)
        Bm = torch.from_numpy(pool["B"]).to(cuda_device)
        S = torch.from_numpy(S_np).to(cuda_device)
        mstate = torch.zeros((w.B, w.H, 2, V), dtype=torch.float32, device=cuda_device)
        pos = torch.zeros((w.B, w.H), dtype=torch.int32, device=cuda_device)
        outs = []
        for j in range(steps):
            o = carve.carve_step(tp["q"][j], tp["k"][j], tp["v"][j], tp["g_logit"][j], tp["bx"][j], tp["w_logit"][j],
                                 A, Bm, S, mc_mode=mode, chunk=L, mstate=mstate, pos=pos)
            outs.append(host(o))
        assert carve.carve_check() == 0
        Sr = S_np.astype(np.float64).copy()
        ms = np.zeros((w.B, w.H, 2, V))
        ps = np.zeros((w.B, w.H), dtype=np.int32)
        ref = [oracle.step({k: pool[k][j] for k in ("q", "k", "v", "g_logit", "bx", "w_logit")}, pool["A"], pool["B"],
                           Sr, L=L, mc_mode=mode, mstate=ms, pos=ps) for j in range(steps)]
        check(f"o mode {mode}", np.stack(outs), np.stack(ref), TOL[io])
        check(f"S mode {mode}", host(S), Sr, TOL[io])
        if mode == 1:
            check("mstate", host(mstate), ms, TOL[io])
            assert torch.all(pos == steps)


# ---------------------------------------------------------------------------------------
# content term of the write gate: w = sigmoid(w_logit + Aw . z_c), and the decay's amplitude
# and bias: g = exp(-e^{A_dec} softplus(g_logit + tau))  (both kernel paths, decode)
# ---------------------------------------------------------------------------------------
def _terms_case(cuda_device, w, L, mode, write=True, decay=False):
    import torch
    d = I.make_inputs(w)
    d["A"] *= 10.0
    d["B"] *= 10.0
    extra, grads = {}, ()
    if write:
        d["Aw"] = I.normal(w.seed, 97, (w.H, w.R), 0.0, 2.0)
        grads += ("dAw",)
    if decay:
        d.update(I.make_decay(w))
        grads += ("dA_dec", "dtau")
    dO = I.make_grad_out(w)
    S0 = I.make_state(w, 0.05)
    mp = I.normal(3, 2, (w.B, w.H, w.V)).astype(np.float32)
    dSf = I.normal(3, 3, (w.B, w.H, w.V, w.K)).astype(np.float32)
    dd = to_dev(dict(d, dO=dO), w.io, cuda_device)
    for key in ("Aw", "A_dec", "tau"):
        if key in d:
            extra[key] = torch.from_numpy(np.asarray(d[key], dtype=np.float32)).to(cuda_device)
    tS0, tmp, tdS = (torch.from_numpy(x).to(cuda_device) for x in (S0, mp, dSf))
    args = (dd["q"], dd["k"], dd["v"], dd["g_logit"], dd["bx"], dd["w_logit"], dd["A"], dd["B"])
    out = carve.carve_fwd(*args, chunk=L, mc_mode=mode, S0=tS0, m_prev_in=tmp, **extra)
    g = carve.carve_bwd(*args, out["saved"], dd["dO"], chunk=L, mc_mode=mode, S0=tS0, m_prev_in=tmp,
                        dS_final=tdS, **extra)
    torch.cuda.synchronize()
    r = oracle.fwd(d, L=L, mc_mode=mode, S0=S0, m_prev=mp)
    rg = oracle.bwd(d, L, dO, mc_mode=mode, S0=S0, m_prev=mp, dS_final=dSf)
    tol = TOL[w.io]
    check("o", host(out["o"]), r["o"], tol)
    check("S_final", host(out["S_final"]), r["S_final"], tol)
    for key in GRADS + grads + ("dS0",):
        check(key, host(g[key]), rg[key], tol)
    if decay and mode == 0:   # the forward-only path (64-token compute chunks on the tensor cores)
        f = carve.carve_fwd(*args, chunk=L, mc_mode=mode, S0=tS0, m_prev_in=tmp, save_for_bwd=False, **extra)
        torch.cuda.synchronize()
        check("o (forward only)", host(f["o"]), r["o"], tol)
    return d, dd, args, tS0, tmp, tdS


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("path", ["tensor_core", "simt"])
def test_write_gate_term(cuda_device, path, mode):
    if path == "tensor_core":
        w = dataclasses.replace(I.FWD_1P3B, B=1, H=3, T=256, L=64, seed=61 + mode)
    else:
        w = dataclasses.replace(I.TINY_FP32, B=2, H=2, T=96, L=32, seed=63 + mode)
    _terms_case(cuda_device, w, w.L, mode)


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("path", ["tensor_core", "simt"])
def test_decay_amplitude_and_bias(cuda_device, path, mode):
    if path == "tensor_core":
        w = dataclasses.replace(I.FWD_1P3B, B=2, H=3, T=256, L=64, seed=71 + mode)
    else:
        w = dataclasses.replace(I.TINY_FP32, B=2, H=2, T=96, L=32, seed=73 + mode)
    _terms_case(cuda_device, w, w.L, mode, write=False, decay=True)


def test_decay_with_write_gate_term(cuda_device):
    """Both optional terms at once on the tensor-core path, with a ragged last gate chunk."""
    w = dataclasses.replace(I.FWD_1P3B, B=2, H=2, T=224, L=64, seed=75)
    _terms_case(cuda_device, w, w.L, 0, write=True, decay=True)


def test_zero_write_factor_is_bit_identical(cuda_device):
    """Aw = 0 on the tensor-core path: every output equals the run without the term, bit for bit."""
    import torch
    w = dataclasses.replace(I.FWD_1P3B, B=1, H=2, T=128, L=64, seed=65)
    d = I.make_inputs(w)
    d["A"] *= 10.0
    d["B"] *= 10.0
    dd = to_dev(dict(d, dO=I.make_grad_out(w)), w.io, cuda_device)
    args = (dd["q"], dd["k"], dd["v"], dd["g_logit"], dd["bx"], dd["w_logit"], dd["A"], dd["B"])
    zero = torch.zeros((w.H, w.R), dtype=torch.float32, device=cuda_device)
    f0 = carve.carve_fwd(*args, chunk=w.L)
    f1 = carve.carve_fwd(*args, chunk=w.L, Aw=zero)
    g0 = carve.carve_bwd(*args, f0["saved"], dd["dO"], chunk=w.L)
    g1 = carve.carve_bwd(*args, f1["saved"], dd["dO"], chunk=w.L, Aw=zero)
    torch.cuda.synchronize()
    assert torch.equal(f0["o"], f1["o"]) and torch.equal(f0["S_final"], f1["S_final"])
    for key in GRADS:
        assert torch.equal(g0[key], g1[key]), key


@pytest.mark.parametrize("K,V,io", [(128, 128, "bf16"), (64, 64, "fp32")])
@pytest.mark.parametrize("decay", [False, True])
def test_decode_write_gate_term(cuda_device, K, V, io, decay):
    """The decode step with the write gate's content term, and (decay) also the decay's
    amplitude and bias."""
    import torch
    w = dataclasses.replace(I.DECODE, B=4, H=8, K=K, V=V, R=16, io=io, seed=700 + K)
    steps, L = 12, 4
    pool = I.make_decode_pool(w, pool=steps)
    Aw_np = I.normal(w.seed, 96, (w.H, w.R), 0.0, 3.0)
    dec_np = I.make_decay(w) if decay else {}
    dec = {k: torch.from_numpy(v).to(cuda_device) for k, v in dec_np.items()}
    for mode in (0, 1):
        S_np = I.make_state(w, 0.05)
        tp = to_dev({k: pool[k] for k in ("q", "k", "v", "g_logit", "bx", "w_logit")}, io, cuda_device)
        A = torch.from_numpy(pool["A"]).to(cuda_device)
        Bm = torch.from_numpy(pool["B"]).to(cuda_device)
        Aw = torch.from_numpy(Aw_np.astype(np.float32)).to(cuda_device)
        S = torch.from_numpy(S_np).to(cuda_device)
        mstate = torch.zeros((w.B, w.H, 2, V), dtype=torch.float32, device=cuda_device)
        pos = torch.zeros((w.B, w.H), dtype=torch.int32, device=cuda_device)
        outs = [host(carve.carve_step(tp["q"][j], tp["k"][j], tp["v"][j], tp["g_logit"][j], tp["bx"][j],
                                      tp["w_logit"][j], A, Bm, S, mc_mode=mode, chunk=L, mstate=mstate, pos=pos,
                                      Aw=Aw, **dec)) for j in range(steps)]
        Sr = S_np.astype(np.float64).copy()
        ms = np.zeros((w.B, w.H, 2, V))
        ps = np.zeros((w.B, w.H), dtype=np.int32)
        ref = [oracle.step({k: pool[k][j] for k in ("q", "k", "v", "g_logit", "bx", "w_logit")}, pool["A"],
                           pool["B"], Sr, L=L, mc_mode=mode, mstate=ms, pos=ps, Aw=Aw_np,
                           **{k: v.astype(np.float64) for k, v in dec_np.items()}) for j in range(steps)]
        check(f"o mode {mode}", np.stack(outs), np.stack(ref), TOL[io])
        check(f"S mode {mode}", host(S), Sr, TOL[io])
