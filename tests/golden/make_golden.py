"""Writes tests/golden/oracle_tiny.json from the fp64 oracle alone.

The pages print no worked numerical example, so the stored values here are the oracle's
own (regression guard against unintended changes of the oracle's arithmetic); they are
pinned indirectly by the closed forms and invariants of tests/test_oracle_pins.py.
Run:  python tests/golden/make_golden.py
"""
import dataclasses
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from chunk_gated_delta_b200 import inputs as I  # noqa: E402

CASE = dict(B=1, H=1, T=6, K=3, V=3, R=2, L=4, seed=424242)


def compute():
    w = dataclasses.replace(I.TINY_FP32, **CASE)
    d = {k: np.asarray(v, dtype=np.float64) for k, v in I.make_inputs(w).items()}
    d["A"] *= 50.0
    d["B"] *= 50.0
    out = {"case": CASE, "A_B_scale": 50.0}
    for mode in (0, 1):
        r = oracle.fwd(d, L=w.L, mc_mode=mode)
        out[f"mc{mode}"] = {"o": r["o"].ravel().tolist(), "S_final": r["S_final"].ravel().tolist()}
    # the optional terms: the write gate's content factor and the decay's amplitude and bias
    dt = dict(d, Aw=np.array([[2.0, -3.0]]), A_dec=np.array([0.4]), tau=np.array([[0.5, -1.0, 0.25]]))
    r = oracle.fwd(dt, L=w.L, mc_mode=0)
    g = oracle.bwd(dt, w.L, np.ones_like(r["o"]), mc_mode=0)
    out["terms"] = {"o": r["o"].ravel().tolist(), "S_final": r["S_final"].ravel().tolist(),
                    "dAw": g["dAw"].ravel().tolist(), "dA_dec": g["dA_dec"].ravel().tolist(),
                    "dtau": g["dtau"].ravel().tolist()}
    # the exact recurrence (L = 1) and two packed sequences (4 + 2 tokens)
    r = oracle.fwd(d, L=1, mc_mode=0)
    out["exact"] = {"o": r["o"].ravel().tolist(), "S_final": r["S_final"].ravel().tolist()}
    r = oracle.fwd(d, L=w.L, mc_mode=1, cu_seqlens=np.array([0, 4, 6]))
    out["packed"] = {"o": r["o"].ravel().tolist(), "S_final": r["S_final"].ravel().tolist()}
    return out


if __name__ == "__main__":
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_tiny.json"), "w") as f:
        json.dump(compute(), f, indent=1)
