"""Benchmark of the CARVE recurrence library on B200.

Default workload: the 1.3B-layer training step (B=8, H=16, T=4096, d=128, chunk 64, rank 32,
bf16 q/k/v/o, fp32 gates) -- one step = carve_fwd (saving what the backward needs) + carve_bwd
against a seeded upstream gradient.  Prints ONE JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl carve|reference]
                  [--workload train|fwd|decode] [--no-e2e] [--no-cpu-baseline]

Timing: CUDA events on the launch stream, W untimed warm-up steps, then K timed steps
bracketed by a barrier and a device synchronize, max over ranks.  The working set of a step
(about 3 GB) is far larger than the 126 MB L2, so no explicit flush is needed between steps.
`--impl reference` times the fp64 CPU oracle on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import copy
import dataclasses
import json
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from chunk_gated_delta_b200 import inputs as I  # noqa: E402

VARLEN_LO, VARLEN_HI = 512, 8192   # lengths of the packed variable-length benchmark
METRIC = "fwd+bwd tokens/s per layer (B200, 16 heads, d=128) & % bf16 tensor peak"

# Algorithmic HBM bytes per (token, head) at d = 128 with bf16 q/k/v/o and fp32 gates:
#   forward : q,k,v 768 + g_logit,bx 1024 + w 4 + o 256                      = 2052
#             + chunk-boundary state saved for the backward, 4 d^2 / L          (1024 at L=64)
#   backward: inputs 1796 + dO 256 + boundary state 4 d^2 / L + dq,dk,dv 768
#             + dg_logit,dbx 1024 + dw 4                                        = 3848 + 4 d^2 / L
# FLOPs per (token, head), triangular halves only (forward exact for the WY algorithm,
# backward counted from its GEMM list):
#   forward : 5 L d + 6 d^2 + L^2/3 + (2 d^2 + 4 r d)/L
#   backward: 14 L d + 14 d^2 + L^2
def fwd_bytes(d, L):
    return 2052 + 4 * d * d / L


def bwd_bytes(d, L):
    return 3848 + 4 * d * d / L


def fwd_flops(d, L, r):
    return 5 * L * d + 6 * d * d + L * L / 3 + (2 * d * d + 4 * r * d) / L


def bwd_flops(d, L, r):
    return 14 * L * d + 14 * d * d + L * L


def launches_per_step(w, fwd_only, decay=False):
    """Kernels one step launches on the tensor-core path (bf16, d = 128): the forward (plus the
    chunk-mean prologue when it saves for the backward in mode 0); the backward, the dq
    readout pass (mode 0), the dA/dB reduction and (with the decay's parameters) the d tau /
    d A_dec reduction."""
    if fwd_only:
        return 1
    if w.L == 1:   # the exact recurrence: its forward, its backward and the per-unit reduction
        return 3
    return (2 if w.mc_mode == 0 else 1) + (3 if w.mc_mode == 0 else 2) + (1 if decay else 0)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        return dict(hbm=j["hbm_gbs"], bf16=j["bf16_tflops"], bf16_sustained=j.get("bf16_tflops_sustained"),
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


# ---------------------------------------------------------------------------------------
class ClockSampler:
    """SM clock, power and throttle reasons of this process's GPU, polled through NVML every
    `period` seconds on a host thread during the timed region (read-only queries); with
    `--clocks-csv PATH` the samples are also written to PATH (rank i: PATH.rank<i>)."""
    NAMES = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
             ("sw_power_cap", 0x4))

    csv_path = None   # set from --clocks-csv

    def __init__(self, index: int, period: float = 0.005):
        self.index, self.period = index, period
        self.rows, self.err = [], None
        self.path = None if self.csv_path is None else (
            self.csv_path if index == 0 else f"{self.csv_path}.rank{index}")

    def _handle(self, nv):
        import torch
        try:
            p = torch.cuda.get_device_properties(self.index)
            bus = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
            return nv.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:   # noqa: BLE001 - older torch without PCI fields: CUDA order
            return nv.nvmlDeviceGetHandleByIndex(self.index)

    def _run(self):
        nv = self.nv
        reasons_fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self.stop.is_set():
            try:
                self.rows.append((time.time(), nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM),
                                  nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0, int(reasons_fn(self.h))))
            except Exception as e:   # noqa: BLE001
                self.err = str(e)
                return
            self.stop.wait(self.period)

    def __enter__(self):
        import threading
        try:
            import pynvml as nv
            nv.nvmlInit()
            self.nv, self.h = nv, self._handle(nv)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
        except Exception as e:   # noqa: BLE001
            self.nv, self.err = None, f"nvml: {e}"
            return self
        self.stop = threading.Event()
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()
        return self

    def __exit__(self, *exc):
        if self.nv is None:
            return
        self.stop.set()
        self.thread.join(timeout=5)
        try:
            if self.path is None:
                raise OSError("no csv requested")
            os.makedirs(os.path.dirname(os.path.abspath(self.path)), exist_ok=True)
            with open(self.path, "w") as f:
                f.write("time,sm_mhz,sm_max_mhz,power_w,reasons_mask\n")
                for t, mhz, pw, rs in self.rows:
                    f.write(f"{t:.3f},{mhz},{self.max_mhz},{pw:.1f},{rs:#x}\n")
        except OSError:
            pass
        self.nv.nvmlShutdown()

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled: " + str(self.err)]}
        reasons = sorted({n for _, _, _, rs in self.rows for n, bit in self.NAMES if rs & bit})
        return {"sm_mhz": statistics.median(r[1] for r in self.rows), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.rows), "power_w_max": max(r[2] for r in self.rows)}


# ---------------------------------------------------------------------------------------
def dist_setup():
    from chunk_gated_delta_b200 import dist as cdist
    return cdist.setup("nccl")


def barrier_sync(ws):
    import torch
    from chunk_gated_delta_b200 import dist as cdist
    cdist.barrier(torch.device("cuda", torch.cuda.current_device()))


def max_over_ranks(x: float, ws: int) -> float:
    import torch
    from chunk_gated_delta_b200 import dist as cdist
    return cdist.max_over_ranks(x, torch.device("cuda", torch.cuda.current_device()))


def cpu_oracle_sample(w, d, dO, target_s=12.0, max_T=None, fwd_only=False):
    """Time the fp64 oracle (fwd + bwd) on batch element 0 (all heads) over a prefix of the
    sequence, doubling the prefix until the run takes at least target_s / 2 seconds.
    Returns (tokens/s of the whole layer, cores used, sample description)."""
    import oracle
    T = 128
    max_T = w.T if max_T is None else max_T
    while True:
        sub = {k: (v[:1, :T] if v.ndim >= 3 and k not in ("A", "B") else v) for k, v in d.items()}
        t0 = time.perf_counter()
        oracle.fwd(sub, L=w.L, mc_mode=w.mc_mode)
        if not fwd_only:
            oracle.bwd(sub, w.L, dO[:1, :T], mc_mode=w.mc_mode)
        dt = time.perf_counter() - t0
        if dt >= target_s / 2 or T >= max_T:
            break
        T = min(max_T, T * 2)
    what = "fwd" if fwd_only else "fwd+bwd"
    return T / dt, oracle.threads(), f"oracle {what}, batch 0 (all {w.H} heads), first {T} of {w.T} tokens"


# ---------------------------------------------------------------------------------------
def run_reference(args, w):
    """The reference arm: the fp64 oracle on the host cores, one bounded sample per step (batch
    element 0, every head: 256 tokens for the sequence workloads, batch 0-15 for decode),
    reported in this workload's metric and unit."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if ws > 1 and rank != 0:
        return
    import oracle
    decode = args.workload == "decode"
    fwd_only = args.workload == "fwd"
    if decode:
        Bs, P = 16, 64
        pool = I.make_decode_pool(w, pool=P)
        S64 = I.make_state(w, 0.05)[:Bs].astype(np.float64)
        keys = ("q", "k", "v", "g_logit", "bx", "w_logit")

        def one(j):
            oracle.step({k: pool[k][j % P][:Bs] for k in keys}, pool["A"], pool["B"], S64, L=1, mc_mode=w.mc_mode)
    else:
        Tp = 256
        d = I.make_inputs(w, T=Tp)
        dO = I.make_grad_out(w, T=Tp)
        sub = {k: (v[:1] if v.ndim >= 3 and k not in ("A", "B") else v) for k, v in d.items()}

        def one(j):
            oracle.fwd(sub, L=w.L, mc_mode=w.mc_mode)
            if not fwd_only:
                oracle.bwd(sub, w.L, dO[:1], mc_mode=w.mc_mode)
    for j in range(args.warmup):
        one(j)
    t0 = time.perf_counter()
    for j in range(args.steps):
        one(j)
    dt = (time.perf_counter() - t0) / args.steps
    if decode:
        v, unit, metric = Bs / w.B / dt, "steps/s", "decode steps/s (B200, B=256, 16 heads, d=128)"
        sample = f"oracle decode step on batch 0-{Bs - 1} of {w.B} (all {w.H} heads), scaled to {w.B}"
    else:
        v, unit = Tp / dt, "tokens/s"
        metric = "fwd tokens/s per layer (B200, 16 heads, d=128)" if fwd_only else METRIC
        sample = f"oracle {'fwd' if fwd_only else 'fwd+bwd'} on batch 0 (all {w.H} heads), {Tp} tokens per step"
    line = {"impl": "reference", "metric": metric, "value": v, "unit": unit, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "sample": sample},
            "cpu_baseline": {"value": v, "unit": unit, "cores": oracle.threads(), "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_train(args, w, fwd_only=False):
    ws, rank, local = dist_setup()
    line = measure_train(args, w, ws, rank, local, fwd_only)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_long(args):
    """The long-context workload: B1 H16 T65536 d128, the training step (fwd + bwd) at every
    gate chunk L in {32, 64, 128} with both content readouts.  One JSON line: the headline
    fields are those of L = 64 with the boundary-state readout; `runs` holds all six."""
    ws, rank, local = dist_setup()
    runs, head = {}, None
    for L in (32, 64, 128):
        for mode in (0, 1):
            w = I.long_context(L, mode)
            if args.seq_len:
                w = dataclasses.replace(w, T=args.seq_len, name=w.name.replace("_T65536_", f"_T{args.seq_len}_"))
            sub = copy.copy(args)
            sub.no_e2e = args.no_e2e or (L, mode) != (64, 0)   # end to end: the headline run only
            sub.cpu_target_s = 6.0
            line = measure_train(sub, w, ws, rank, local, False)
            runs[f"L{L}_mc{mode}"] = {k: line[k] for k in ("value", "ms_per_step", "tensor_frac", "kernels_ms")}
            runs[f"L{L}_mc{mode}"].update(hbm_frac=line["roofline"]["frac"], roofline_kernel=line["roofline"]["kernel"],
                                          cpu_baseline=None if line["cpu_baseline"] is None
                                          else line["cpu_baseline"]["value"])
            if (L, mode) == (64, 0):
                head = line
    head["config"]["workload"] = head["config"]["workload"].replace("_L64_mc0", "")
    head["config"]["runs_of"] = "gate chunk L in {32, 64, 128} x readout mc in {0, 1}; headline: L64 mc0"
    head["runs"] = runs
    head["gpu_launches"] = sum(launches_per_step(dataclasses.replace(w, L=int(k[1:k.index('_')]),
                                                                     mc_mode=int(k[-1])), False) * args.steps
                               for k in runs)
    if rank == 0:
        print(json.dumps(head), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def measure_train(args, w, ws, rank, local, fwd_only=False):
    import torch
    import chunk_gated_delta_b200 as carve
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    seed = w.seed + 7919 * rank      # each rank holds its own batch shard (weak scaling)
    d = I.make_inputs(w, seed=seed)
    dO = I.make_grad_out(w, seed=seed)
    bf = torch.bfloat16 if w.io == "bf16" else torch.float32
    host = {}
    for k, v in dict(d, dO=dO).items():
        t = torch.from_numpy(v)
        if k in ("q", "k", "v", "dO"):
            t = t.to(bf)
        host[k] = t.pin_memory()
    dv_ = {k: v.to(dev, non_blocking=True) for k, v in host.items()}
    torch.cuda.synchronize()
    L, mode = w.L, w.mc_mode
    opt = {}   # the optional terms of the recurrence
    if args.write_gate:   # a seeded content factor of the write gate, N(0, 0.02^2) like A and B
        opt["Aw"] = torch.from_numpy(I.normal(w.seed, 95, (w.H, w.R), 0.0, 0.02).astype(np.float32)).to(dev)
    if args.decay:        # the decay's log-amplitude [H] and bias [H, dk]
        opt.update({k: torch.from_numpy(v).to(dev) for k, v in I.make_decay(w).items()})
    packed, lens = {}, None   # packed variable-length sequences: the w.T tokens cut into sequences
    if args.varlen:
        lens = I.make_lengths(w.T, VARLEN_LO, VARLEN_HI, w.seed + 7919 * rank)
        cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
        packed = dict(cu_seqlens=torch.from_numpy(cu).to(dev), max_len=int(lens.max()))
    fwd_fn = carve.carve_fwd_varlen if packed else carve.carve_fwd
    bwd_fn = carve.carve_bwd_varlen if packed else carve.carve_bwd
    fwd_out = fwd_fn(dv_["q"], dv_["k"], dv_["v"], dv_["g_logit"], dv_["bx"], dv_["w_logit"], dv_["A"],
                     dv_["B"], chunk=L, mc_mode=mode, save_for_bwd=not fwd_only, **opt, **packed)
    bwd_out = None
    if not fwd_only:
        from chunk_gated_delta_b200 import dist as cdist
        # every per-head parameter gradient in one flat buffer: the step's one all-reduce
        dAB, pviews = cdist.param_grad_buffer(w.H, w.K, w.V, w.R, dev, write_term="Aw" in opt,
                                              decay="A_dec" in opt)
        bwd_out = bwd_fn(dv_["q"], dv_["k"], dv_["v"], dv_["g_logit"], dv_["bx"], dv_["w_logit"], dv_["A"],
                         dv_["B"], fwd_out["saved"], dv_["dO"], chunk=L, mc_mode=mode,
                         out=dict(pviews), **opt, **packed)
    dims = (carve.dims_varlen(dv_["q"], dv_["v"], dv_["A"], packed["cu_seqlens"], packed["max_len"], L, mode)
            if packed else carve.dims_of(dv_["q"], dv_["v"], dv_["A"], L, mode))
    workspace = torch.empty(carve.bwd_workspace_bytes(dims), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(x, ev=None):
        if ev is not None:
            ev[0].record(stream)
        fwd_fn(x["q"], x["k"], x["v"], x["g_logit"], x["bx"], x["w_logit"], x["A"], x["B"], chunk=L,
               mc_mode=mode, out=fwd_out, save_for_bwd=not fwd_only, **opt, **packed)
        if ev is not None:
            ev[1].record(stream)
        if fwd_only:
            if ev is not None:
                ev[2].record(stream)
            return
        bwd_fn(x["q"], x["k"], x["v"], x["g_logit"], x["bx"], x["w_logit"], x["A"], x["B"],
               fwd_out["saved"], x["dO"], chunk=L, mc_mode=mode, out=bwd_out, workspace=workspace, **opt, **packed)
        if ev is not None:
            ev[2].record(stream)
        if ws > 1:
            cdist.allreduce_(dAB)

    for _ in range(args.warmup):
        step(dv_)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier_sync(ws)
        start.record(stream)
        for j in range(args.steps):
            step(dv_, evs[j])
        end.record(stream)
        barrier_sync(ws)
    ms = max_over_ranks(start.elapsed_time(end), ws) / args.steps
    fwd_ms = sum(e[0].elapsed_time(e[1]) for e in evs) / args.steps
    bwd_ms = sum(e[1].elapsed_time(e[2]) for e in evs) / args.steps
    tokens = w.B * w.T * ws
    value = tokens / (ms * 1e-3)

    th = w.B * w.T * w.H          # token-heads of one rank's launch
    dd = w.K
    # bytes per token-head: the exact recurrence (L = 1) keeps its state on chip and saves it
    # every 64 tokens, so its state term is that of a 64-token save interval
    Lb = 64 if L == 1 else L
    if fwd_only:
        kern = {"carve_fwd": (fwd_ms, 2052 * th)}
    else:
        kern = {"carve_fwd": (fwd_ms, fwd_bytes(dd, Lb) * th), "carve_bwd": (bwd_ms, bwd_bytes(dd, Lb) * th)}
    dom = max(kern, key=lambda k: kern[k][0])
    dms, dbytes = kern[dom]
    achieved = dbytes / (dms * 1e-3) / 1e9
    flops = (fwd_flops(dd, L, w.R) + (0 if fwd_only else bwd_flops(dd, L, w.R))) * th * ws
    tensor_frac = flops / (ms * 1e-3) / (peaks["bf16"] * 1e12 * ws)
    kflops = {"carve_fwd": fwd_flops(dd, L, w.R) * th}
    if not fwd_only:
        kflops["carve_bwd"] = bwd_flops(dd, L, w.R) * th
    traffic = None if (opt or packed) else load_traffic(w.name, dom)

    e2e = None
    if not args.no_e2e:
        e2e = measure_e2e(args, host, dv_, step, stream, ws, w, {"o": fwd_out["o"]} if fwd_only else bwd_out)
    cpu = None
    if not args.no_cpu_baseline and rank == 0 and ws == 1 and not packed:
        v, cores, sample = cpu_oracle_sample(w, d, dO, target_s=getattr(args, "cpu_target_s", 12.0),
                                             fwd_only=fwd_only)
        cpu = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample}
    line = {
        "metric": "fwd tokens/s per layer (B200, 16 heads, d=128)" if fwd_only else METRIC, "value": value,
        "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if w.io == "bf16" else "f32", "data": "synthetic",
        "config": {"workload": w.name, "global_batch": w.B * ws, "seq_len": w.T, "heads": w.H, "d": w.K,
                   "chunk": L, "rank": w.R, "mc_mode": mode, "parallelism": f"dp{ws}",
                   "write_gate_term": bool(args.write_gate), "decay_parameters": bool(args.decay),
                   "packed_sequences": None if lens is None else {
                       "count": len(lens), "lengths": f"U{{{VARLEN_LO}..{VARLEN_HI}}} filling {w.T} tokens",
                       "max_len": int(lens.max()), "min_len": int(lens.min())},
                   "l2": "no flush: step working set ~3 GB >> 126 MB L2"},
        "tensor_frac": tensor_frac,
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peaks["hbm"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm"], "traffic": traffic, "peak_source": peaks["source"]},
        "kernels_ms": {"carve_fwd": fwd_ms, "carve_bwd": bwd_ms},
        "per_kernel": kernel_rooflines(kern, kflops, peaks),
        "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches_per_step(w, fwd_only, args.decay) * args.steps,
        "clocks": clk.summary(),
    }
    return line


# Decode: per (b,h) and step, the fp32 state read and written (8 d^2 = 131,072 B at d = 128),
# q, k, v (768 B), g_logit and bx (1,024 B), w_logit (4 B) and o (256 B).
def step_bytes(d):
    return 8 * d * d + 3 * 2 * d + 2 * 4 * d + 4 + 2 * d


def run_decode(args, w):
    """One bench step = one carve_step (one token for every (b,h)) of the decode workload,
    reading token set j % 64 of a seeded pool held on the device; the state stays resident."""
    import torch
    import chunk_gated_delta_b200 as carve
    ws, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    seed = w.seed + 7919 * rank
    P = 64
    pool = I.make_decode_pool(w, pool=P, seed=seed)
    S_host = I.make_state(w, 0.05, seed=seed)
    host = {}
    for k, v in pool.items():
        t = torch.from_numpy(v)
        host[k] = (t.to(torch.bfloat16) if k in ("q", "k", "v") else t).pin_memory()
    dp = {k: v.to(dev) for k, v in host.items()}
    S = torch.from_numpy(S_host).to(dev)
    o = torch.empty((w.B, w.H, w.V), dtype=torch.bfloat16, device=dev)
    keys = ("q", "k", "v", "g_logit", "bx", "w_logit")
    stream = torch.cuda.current_stream()

    dec = {k: torch.from_numpy(v).to(dev) for k, v in I.make_decay(w).items()} if args.decay else {}

    def step(x):
        carve.carve_step(x["q"], x["k"], x["v"], x["g_logit"], x["bx"], x["w_logit"], dp["A"], dp["B"], S,
                         mc_mode=w.mc_mode, chunk=1, o=o, **dec)

    # One step is one short kernel, so the loop is launch-bound from Python: each pool slot's
    # step is captured once in a CUDA graph and the timed loop replays them in order.
    for j in range(2):
        step({k: dp[k][j % P] for k in keys})
    torch.cuda.synchronize()
    graphs = []
    for j in range(P):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step({k: dp[k][j] for k in keys})
        graphs.append(g)
    for j in range(args.warmup):
        graphs[j % P].replay()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier_sync(ws)
        start.record(stream)
        for j in range(args.steps):
            graphs[j % P].replay()
        end.record(stream)
        barrier_sync(ws)
    ms = max_over_ranks(start.elapsed_time(end), ws) / args.steps
    value = ws / (ms * 1e-3)            # steps/s of the whole job (each rank: its own batch shard)
    units = w.B * w.H
    achieved = step_bytes(w.K) * units / (ms * 1e-3) / 1e9

    e2e = None
    if not args.no_e2e:   # the step's token set from pinned host memory, o back to the host
        stages = [{k: torch.empty_like(dp[k][0]) for k in keys} for _ in range(2)]
        o_host = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
        h2d = sum(host[k][0].numel() * host[k][0].element_size() for k in keys)
        d2h = o.numel() * o.element_size()

        def h2d_fn(j, si):
            for k in keys:
                stages[si][k].copy_(host[k][j % P], non_blocking=True)

        def d2h_fn(j):
            o_host.copy_(o, non_blocking=True)

        pipelined_e2e(2, stream, h2d_fn, lambda si: step(stages[si]), d2h_fn)
        n = max(2, args.steps)
        barrier_sync(ws)
        e_start, e_end = pipelined_e2e(n, stream, h2d_fn, lambda si: step(stages[si]), d2h_fn)
        barrier_sync(ws)
        ems = max_over_ranks(e_start.elapsed_time(e_end), ws) / n
        e2e = {"value": ws / (ems * 1e-3), "unit": "steps/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "steps": n, "pipeline": "H2D of step j+1 and D2H of step j overlap the kernel (two input sets)"}
    cpu = None
    if not args.no_cpu_baseline and rank == 0 and ws == 1:
        import oracle
        Bs = 16
        S64 = S_host[:Bs].astype(np.float64)
        A64, B64 = pool["A"], pool["B"]
        t0, n = time.perf_counter(), 0
        while time.perf_counter() - t0 < 6.0:
            tok = {k: pool[k][n % P][:Bs] for k in keys}
            oracle.step(tok, A64, B64, S64, L=1, mc_mode=w.mc_mode)
            n += 1
        dt = time.perf_counter() - t0
        cpu = {"value": n / dt * Bs / w.B, "unit": "steps/s", "cores": oracle.threads(), "kind": "oracle",
               "sample": f"oracle decode, {n} steps on batch 0-{Bs - 1} of {w.B} (all {w.H} heads), scaled to {w.B}"}
    line = {
        "metric": "decode steps/s (B200, B=256, 16 heads, d=128)", "value": value, "unit": "steps/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": w.name, "global_batch": w.B * ws, "heads": w.H, "d": w.K, "rank": w.R,
                   "mc_mode": w.mc_mode, "parallelism": f"dp{ws}", "tokens_per_s": value * w.B,
                   "decay_parameters": bool(args.decay),
                   "launch": "one CUDA graph per token-pool slot (one kernel each), replayed in order",
                   "l2": "no flush: 256 MB state and 470 MB token pool >> 126 MB L2"},
        "roofline": {"bound": "hbm", "kernel": "carve_step", "achieved": achieved, "peak": peaks["hbm"],
                     "unit": "GB/s", "frac": achieved / peaks["hbm"],
                     "traffic": None if args.decay else load_traffic(w.name, "carve_step"),
                     "peak_source": peaks["source"]},
        "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": args.steps, "clocks": clk.summary(),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_deviation(args, w):
    """Chunk-aligned readout against the exact recurrence: the relative L2 deviation of the
    outputs o of carve_fwd at gate chunks L = 16 .. 128 (both readouts) from those of the exact
    content-aware recurrence (chunk = 1), on the same synthetic inputs, in fp32 I/O so that the
    measured deviation is not bf16 rounding; with the recipe's low-rank projections and with
    them scaled by 10 (a stronger content path).  One forward per configuration."""
    import torch
    import chunk_gated_delta_b200 as carve
    ws, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    d = I.make_inputs(w)
    x = {k: torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32)).to(dev) for k, v in d.items()}
    out = {}
    for scale in (1.0, 10.0):
        args8 = (x["q"], x["k"], x["v"], x["g_logit"], x["bx"], x["w_logit"], x["A"] * scale, x["B"] * scale)
        ref = carve.carve_fwd(*args8, chunk=1, mc_mode=0, save_for_bwd=False)["o"].double()
        row = {}
        for mode in (0, 1):
            for L in (16, 32, 64, 128):
                o = carve.carve_fwd(*args8, chunk=L, mc_mode=mode, save_for_bwd=False)["o"].double()
                row[f"mode{mode}_L{L}"] = float(torch.linalg.vector_norm(o - ref) / torch.linalg.vector_norm(ref))
        out[f"projection_scale_{scale:g}"] = row
    assert carve.carve_check() == 0
    line = {
        "metric": "chunk-aligned readout deviation (relative L2 of o against the exact recurrence)",
        "value": out["projection_scale_1"]["mode1_L64"], "unit": "relative", "n_gpus": ws, "steps": 1,
        "warmup": 0, "higher_is_better": False, "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.B, "seq_len": w.T, "heads": w.H, "d": w.K, "rank": w.R,
                   "io": "fp32"},
        "by_chunk": out,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def kernel_rooflines(kern, flops, peaks):
    """Per ABI call: its CUDA-event time, algorithmic HBM rate and bf16 tensor rate, each with its
    fraction of the peak.  kern: call -> (ms, algorithmic bytes); flops: call -> FLOPs."""
    out = {}
    for k, (kms, kbytes) in kern.items():
        sec = kms * 1e-3
        gbs = kbytes / sec / 1e9
        tfs = flops[k] / sec / 1e12
        out[k] = {"ms": kms, "hbm_gbs": gbs, "hbm_frac": gbs / peaks["hbm"], "tflops": tfs,
                  "tensor_frac": tfs / peaks["bf16"]}
    return out


def load_traffic(workload, call):
    """DRAM bytes of one `call` on `workload` from the committed ncu summary (None when that
    workload was not captured)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    return json.load(open(p)).get(f"{workload}/{call}")


def pipelined_e2e(n, stream, h2d, compute, d2h):
    """n steps of a host-buffer pipeline: the host-to-device copies of step j + 1 (on one copy
    stream) and the device-to-host copies of step j (on another) overlap the kernels, using
    both directions of the host link; inputs alternate between two device buffer sets.
    h2d(j, s) copies step j's inputs into set s, compute(s) runs one step on set s (on
    `stream`), d2h(j) copies step j's results out.  Every hand-off is ordered by events:
    a set is refilled only after the step that read it, and the results are overwritten only
    after they have left.  Returns (start, end) events on `stream` that bracket everything."""
    import torch
    sa, sb = torch.cuda.Stream(), torch.cuda.Stream()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    h_ev, k_ev, d_ev = [None] * n, [None] * n, [None] * n
    start.record(stream)
    sa.wait_event(start)
    with torch.cuda.stream(sa):
        h2d(0, 0)
        h_ev[0] = sa.record_event()
    for j in range(n):
        stream.wait_event(h_ev[j])
        if j > 0:
            stream.wait_event(d_ev[j - 1])
        with torch.cuda.stream(stream):
            compute(j % 2)
        k_ev[j] = stream.record_event()
        if j + 1 < n:
            if j >= 1:
                sa.wait_event(k_ev[j - 1])
            with torch.cuda.stream(sa):
                h2d(j + 1, (j + 1) % 2)
                h_ev[j + 1] = sa.record_event()
        sb.wait_event(k_ev[j])
        with torch.cuda.stream(sb):
            d2h(j)
            d_ev[j] = sb.record_event()
    stream.wait_event(d_ev[n - 1])
    end.record(stream)
    return start, end


def measure_e2e(args, host, dv_, step, stream, ws, w, grads):
    """Same step through the public API with host buffers: each step's inputs copied from
    pinned host memory and every result copied back, inside the timed region, pipelined
    across steps (pipelined_e2e)."""
    import torch
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    grads_host = {k: torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for k, t in grads.items()}
    d2h = sum(t.numel() * t.element_size() for t in grads.values())
    sets = [dv_, {k: torch.empty_like(v) for k, v in dv_.items()}]

    def h2d_fn(j, si):
        for k in host:
            sets[si][k].copy_(host[k], non_blocking=True)

    def d2h_fn(j):
        for k, t in grads.items():
            grads_host[k].copy_(t, non_blocking=True)

    pipelined_e2e(2, stream, h2d_fn, lambda si: step(sets[si]), d2h_fn)
    steps = max(2, min(args.steps, 8))
    barrier_sync(ws)
    start, end = pipelined_e2e(steps, stream, h2d_fn, lambda si: step(sets[si]), d2h_fn)
    barrier_sync(ws)
    ms = max_over_ranks(start.elapsed_time(end), ws) / steps
    return {"value": w.B * w.T * ws / (ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps,
            "pipeline": "H2D of step j+1 and D2H of step j overlap the kernels (two input sets)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="carve", choices=["carve", "reference"])
    ap.add_argument("--workload", default="train", choices=["train", "fwd", "decode", "exact", "deviation", "long"],
                    help="exact: the training step of the exact content-aware recurrence (chunk = 1); deviation: "
                         "the chunk-aligned readout's output deviation from the exact recurrence; long: the "
                         "long-context training step (B1 H16 T65536) at L in {32, 64, 128} x both readouts")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=None, help="override B (smaller cases for profiling)")
    ap.add_argument("--seq-len", type=int, default=None, help="override T (smaller cases for profiling)")
    ap.add_argument("--write-gate", action="store_true",
                    help="train/fwd with the write gate's content term (a seeded non-zero Aw [H, rank])")
    ap.add_argument("--clocks-csv", default=None,
                    help="also write the clock samples of the timed region to this CSV file")
    ap.add_argument("--varlen", action="store_true",
                    help="train/fwd on packed variable-length sequences: the step's tokens cut into seeded lengths "
                         "U{512..8192} (carve_fwd_varlen / carve_bwd_varlen)")
    ap.add_argument("--decay", action="store_true",
                    help="train/fwd/decode with the decay's log-amplitude A_dec [H] and bias tau [H, dk] (seeded)")
    args = ap.parse_args()
    ClockSampler.csv_path = args.clocks_csv
    w = {"fwd": I.FWD_1P3B, "decode": I.DECODE}.get(args.workload, I.TRAIN_1P3B)
    if args.workload == "exact":   # the same step with the state read at every token (L = 1)
        w = dataclasses.replace(w, L=1, name=w.name.replace("_layer_", "_layer_exact_").replace("_L64", "_L1"))
    if args.batch:
        w = dataclasses.replace(w, B=args.batch, name=w.name.replace(f"_B{w.B}_", f"_B{args.batch}_"))
    if args.seq_len:
        w = dataclasses.replace(w, T=args.seq_len, name=w.name.replace(f"_T{w.T}_", f"_T{args.seq_len}_"))
    if args.varlen:   # the same token count, packed: one row of B T tokens
        if args.workload == "decode":
            raise SystemExit("--varlen applies to the train and fwd workloads")
        w = dataclasses.replace(w, B=1, T=w.B * w.T, name=w.name.replace(f"_B{w.B}_", "_varlen_").replace(
            f"_T{w.T}_", f"_{w.B * w.T}tok_"))
    if args.workload == "long":
        if args.impl == "reference":
            run_reference(args, I.long_context(64, 0))
        else:
            run_long(args)
    elif args.workload == "deviation":
        run_deviation(args, dataclasses.replace(w, io="fp32", name=w.name.replace("train_", "deviation_")))
    elif args.impl == "reference":
        run_reference(args, w)
    elif args.workload == "decode":
        run_decode(args, w)
    else:
        run_train(args, w, fwd_only=args.workload == "fwd")


if __name__ == "__main__":
    main()
