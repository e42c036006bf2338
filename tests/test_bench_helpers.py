"""Host-side pieces of bench.py and the input recipe that the benchmark lines depend on."""
import dataclasses
import json
import os

import numpy as np

import bench
from chunk_gated_delta_b200 import inputs as I

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_launch_counts():
    w = I.TRAIN_1P3B
    assert bench.launches_per_step(w, fwd_only=True) == 1
    # mode 0: chunk-mean prologue + forward; backward + dq readout + two reduction passes
    assert bench.launches_per_step(w, fwd_only=False) == 2 + 3
    assert bench.launches_per_step(dataclasses.replace(w, mc_mode=1), fwd_only=False) == 1 + 2
    assert bench.launches_per_step(w, fwd_only=False, decay=True) == 2 + 3 + 1
    assert bench.launches_per_step(dataclasses.replace(w, L=1), fwd_only=False) == 3


def test_packed_lengths_fill_the_budget_exactly():
    for total, lo, hi, seed in ((32768, 512, 8192, 5), (1000, 10, 30, 1), (64, 64, 64, 2), (5, 16, 32, 3)):
        lens = I.make_lengths(total, lo, hi, seed)
        assert lens.sum() == total and lens.dtype == np.int32
        assert np.all(lens[:-1] >= lo) and np.all(lens <= hi) and lens[-1] >= 1
        assert np.array_equal(lens, I.make_lengths(total, lo, hi, seed))   # seeded


def test_committed_traffic_matches_the_workload_names():
    """The DRAM traffic of the committed captures is keyed by workload name and ABI call; the
    default training and decode lines must find theirs."""
    tr = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    for w, call in ((I.TRAIN_1P3B, "carve_fwd"), (I.TRAIN_1P3B, "carve_bwd"), (I.DECODE, "carve_step")):
        assert bench.load_traffic(w.name, call) == tr[f"{w.name}/{call}"] > 0
    assert bench.load_traffic(I.FWD_1P3B.name, "carve_fwd") is None


def test_algorithmic_bytes_per_token_head():
    # forward: q, k, v, o (bf16) + gates (fp32) = 2052 B, plus the saved state 4 d^2 / L
    assert bench.fwd_bytes(128, 64) == 2052 + 4 * 128 * 128 / 64
    assert bench.bwd_bytes(128, 64) == 3848 + 4 * 128 * 128 / 64


def test_kernel_rooflines():
    """Per-call rates: bytes and FLOPs over the call's own time, against the peaks."""
    peaks = {"hbm": 6650.0, "bf16": 1590.0}
    kern = {"carve_fwd": (0.5, 1.0e9), "carve_bwd": (2.0, 4.0e9)}
    flops = {"carve_fwd": 2.0e11, "carve_bwd": 1.0e12}
    r = bench.kernel_rooflines(kern, flops, peaks)
    assert set(r) == {"carve_fwd", "carve_bwd"}
    assert abs(r["carve_fwd"]["hbm_gbs"] - 2000.0) < 1e-9 and abs(r["carve_bwd"]["hbm_gbs"] - 2000.0) < 1e-9
    assert abs(r["carve_fwd"]["tflops"] - 400.0) < 1e-9 and abs(r["carve_bwd"]["tflops"] - 500.0) < 1e-9
    assert abs(r["carve_bwd"]["hbm_frac"] - 2000.0 / 6650.0) < 1e-12
    assert abs(r["carve_fwd"]["tensor_frac"] - 400.0 / 1590.0) < 1e-12
