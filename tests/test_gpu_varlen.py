"""Packed variable-length sequences (carve_fwd_varlen / carve_bwd_varlen) against the oracle's
packed evaluation, element by element.

The sequences are drawn separately and packed along the token axis without padding; their
lengths include an empty sequence, a one-token sequence, lengths that end inside a 16-token
compute sub-chunk and inside a gate chunk, and one of exactly the bound.  The rows after the
last sequence hold NaN: a kernel that read a row it does not own would carry NaN into its
outputs.  Rows that belong to no sequence are not compared (they are not written).
"""
import dataclasses

import numpy as np
import pytest

import chunk_gated_delta_b200 as carve
import oracle
from chunk_gated_delta_b200 import inputs as I
from tests.helpers import TOL, host, rel_l2, to_dev

pytestmark = pytest.mark.gpu

TOKEN_KEYS = ("q", "k", "v", "g_logit", "bx", "w_logit")
TAIL = 5   # rows owned by no sequence, filled with NaN


def packed_case(lens, K, V, R, H, io, seed, L):
    seqs = []
    for n, T in enumerate(lens):
        w = dataclasses.replace(I.TINY_FP32, B=1, H=H, T=T, K=K, V=V, R=R, L=L, io=io, seed=seed + n)
        d = I.make_inputs(w)
        d["dO"] = I.make_grad_out(w)
        seqs.append(d)
    packed = {k: seqs[0][k] * 10.0 for k in ("A", "B")}
    for k in TOKEN_KEYS + ("dO",):
        tail = np.full((1, TAIL) + seqs[0][k].shape[2:], np.nan, dtype=np.float32)
        packed[k] = np.concatenate([d[k] for d in seqs] + [tail], axis=1)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return packed, cu


@pytest.mark.parametrize("io,K,V,L", [("fp32", 64, 64, 32), ("bf16", 128, 64, 32), ("bf16", 128, 128, 64),
                                      ("bf16", 128, 128, 32)])
@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("terms", [False, True])
def test_packed_sequences_match_oracle(cuda_device, io, K, V, L, mode, terms):
    """(bf16, 128, 128): the tensor-core kernels (32-token chunks saving for the backward, and
    the forward-only kernel with 64-token chunks when L = 64); the others: the SIMT kernels."""
    import torch
    lens = [37, 0, 64, 1, 100, 16, 45, 128]
    H, R = 2, 16
    packed, cu = packed_case(lens, K, V, R, H, io, 900 + 10 * mode + K, L)
    N = len(lens)
    extra = {}
    if terms:   # the write gate's content term and the decay's amplitude and bias
        w = dataclasses.replace(I.TINY_FP32, H=H, K=K, R=R, seed=77)
        extra = dict(Aw=I.normal(77, 5, (H, R), 0.0, 2.0).astype(np.float32), **I.make_decay(w))
    S0 = I.normal(5, 1, (N, H, V, K), 0.0, 0.05).astype(np.float32)
    mp = I.normal(5, 2, (N, H, V)).astype(np.float32)
    dSf = I.normal(5, 3, (N, H, V, K)).astype(np.float32)
    dmo = I.normal(5, 4, (N, H, V)).astype(np.float32)
    dd = to_dev(packed, io, cuda_device)
    tcu = torch.from_numpy(cu).to(cuda_device)
    tex = {k: torch.from_numpy(v).to(cuda_device) for k, v in extra.items()}
    tS0, tmp, tdS, tdm = (torch.from_numpy(x).to(cuda_device) for x in (S0, mp, dSf, dmo))
    args = tuple(dd[k] for k in ("q", "k", "v", "g_logit", "bx", "w_logit", "A", "B"))
    out = carve.carve_fwd_varlen(*args, tcu, chunk=L, max_len=max(lens), mc_mode=mode, S0=tS0, m_prev_in=tmp,
                                 **tex)
    g = carve.carve_bwd_varlen(*args, out["saved"], dd["dO"], tcu, chunk=L, max_len=max(lens), mc_mode=mode,
                               S0=tS0, m_prev_in=tmp, dS_final=tdS, dm_prev_out=tdm, **tex)
    assert carve.carve_check() == 0
    od = {k: np.asarray(v, dtype=np.float64) for k, v in packed.items() if k != "dO"}
    od.update({k: np.asarray(v, dtype=np.float64) for k, v in extra.items()})
    r = oracle.fwd(od, L=L, mc_mode=mode, S0=S0, m_prev=mp, cu_seqlens=cu)
    rg = oracle.bwd(od, L, packed["dO"], mc_mode=mode, S0=S0, m_prev=mp, dS_final=dSf, dm_prev_out=dmo,
                    cu_seqlens=cu)
    n_rows = cu[-1]
    tol = TOL[io]
    for key, got, ref in [("o", out["o"], r["o"]), ("S_final", out["S_final"], r["S_final"]),
                          ("m_prev_out", out["m_prev_out"], r["m_prev_out"])]:
        x = host(got)
        x = x[:, :n_rows] if key == "o" else x
        ref = ref[:, :n_rows] if key == "o" else ref
        e = rel_l2(x, ref)
        assert e <= tol, f"{key}: rel-L2 {e:.3e}"
    grads = ["dq", "dk", "dv", "dg_logit", "dbx", "dw_logit", "dA", "dB", "dS0", "dm_prev_in"]
    if terms:
        grads += ["dAw", "dA_dec", "dtau"]
    for key in grads:
        x = host(g[key])
        ref = rg[key]
        if key in ("dq", "dk", "dv", "dg_logit", "dbx", "dw_logit"):
            x, ref = x[:, :n_rows], ref[:, :n_rows]
        e = rel_l2(x, ref)
        assert e <= tol, f"{key}: rel-L2 {e:.3e}"
    if L == 64:   # the forward-only path (64-token compute chunks on the tensor cores)
        f = carve.carve_fwd_varlen(*args, tcu, chunk=L, max_len=max(lens), mc_mode=mode, S0=tS0, m_prev_in=tmp,
                                   save_for_bwd=False, **tex)
        assert carve.carve_check() == 0
        e = rel_l2(host(f["o"])[:, :n_rows], r["o"][:, :n_rows])
        assert e <= tol, f"o (forward only): rel-L2 {e:.3e}"
        e = rel_l2(host(f["S_final"]), r["S_final"])
        assert e <= tol, f"S_final (forward only): rel-L2 {e:.3e}"
    # the empty sequence passes its state and content signal (and their gradients) through
    assert np.array_equal(host(out["S_final"])[1], S0[1].astype(np.float64))
    assert np.array_equal(host(g["dS0"])[1], dSf[1].astype(np.float64))
    assert np.array_equal(host(g["dm_prev_in"])[1], dmo[1].astype(np.float64))


def test_out_of_range_offsets_are_reported(cuda_device):
    """A sequence whose rows run past the packed tensor is computed as empty (no access outside
    the tensors) and carve_check reports CARVE_ERR_INVALID_ARG once; the other sequences are
    unaffected and the next call is clean."""
    import torch
    lens = [20, 30]
    packed, cu = packed_case(lens, 64, 64, 8, 2, "fp32", 950, 16)
    dd = to_dev(packed, "fp32", cuda_device)
    args = tuple(dd[k] for k in ("q", "k", "v", "g_logit", "bx", "w_logit", "A", "B"))
    good = torch.from_numpy(cu).to(cuda_device)
    bad = torch.tensor([0, 20, 20 + 30 + TAIL + 1], dtype=torch.int32, device=cuda_device)   # past the rows
    ref = carve.carve_fwd_varlen(*args, good, chunk=16, max_len=64, save_for_bwd=False)
    assert carve.carve_check() == 0
    out = carve.carve_fwd_varlen(*args, bad, chunk=16, max_len=64, save_for_bwd=False)
    assert carve.carve_check() == 1   # CARVE_ERR_INVALID_ARG
    assert torch.equal(out["o"][:, :20], ref["o"][:, :20])
    assert torch.all(out["S_final"][1] == 0)   # treated as empty: S0 = 0 passed through
    carve.carve_fwd_varlen(*args, good, chunk=16, max_len=64, save_for_bwd=False)
    assert carve.carve_check() == 0
