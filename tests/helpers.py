"""Helpers shared by the GPU parity tests: device transfer, the error metric, sampled oracle runs."""
from __future__ import annotations

import numpy as np

from chunk_gated_delta_b200 import inputs as I

# Tolerances (relative L2 over a whole tensor, in fp64), as fixed for this recurrence:
# fp32 I/O with fp32 arithmetic: 1e-5; bf16 q/k/v/o with fp32 gates, state and accumulation: 2e-2.
TOL = {"fp32": 1e-5, "bf16": 2e-2}


def rel_l2(x, ref) -> float:
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / (den if den > 0 else 1.0))


def to_dev(d: dict, io: str, device):
    """float32 numpy inputs -> torch device tensors (q/k/v in the I/O dtype)."""
    import torch
    out = {}
    for key, val in d.items():
        t = torch.from_numpy(np.ascontiguousarray(val, dtype=np.float32)).to(device)
        if key in ("q", "k", "v", "dO") and io == "bf16":
            t = t.to(torch.bfloat16)
        out[key] = t.contiguous()
    return out


def host(t) -> np.ndarray:
    import torch
    return t.detach().to(torch.float32).cpu().numpy().astype(np.float64)


def sub_units(d: dict, bs, hs) -> dict:
    """Restrict [B,T,H,*] inputs (and per-head A, B) to batches bs and heads hs."""
    out = {}
    for key, val in d.items():
        if key in ("A", "B"):
            out[key] = val[hs]
        elif val.ndim >= 3:
            out[key] = val[bs][:, :, hs]
        else:
            out[key] = val
    return out


def workload_inputs(w: I.Workload, T: int | None = None):
    return I.make_inputs(w, T=T)
