"""Data-parallel plumbing of the CARVE layer: one process per GPU over torch.distributed.

The (batch, head) units are independent, so each rank runs the forward and backward on its
own batch shard with no exchange.  The one collective of the path is the sum over ranks of
the per-head parameter gradients, which every unit of a head adds to: the low-rank factor
gradients dA [H,K,r] and dB [H,r,V], and with the optional terms dAw [H,r], dA_dec [H] and
dtau [H,K]; all live in one flat fp32 buffer so that the sum is a single all-reduce.  The sequence axis
does not shard: the erase gate depends on the state, so a chunk cannot start before the
previous one has finished.
"""
from __future__ import annotations

import datetime
import os


def setup(backend: str = "nccl", timeout_s: float = 120.0):
    """Join the process group named by the launcher's environment (WORLD_SIZE, RANK,
    LOCAL_RANK, MASTER_ADDR/PORT) when WORLD_SIZE > 1; with "nccl" also select this rank's
    GPU.  Returns (world_size, rank, local_rank)."""
    import torch
    import torch.distributed as dist
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1 and not dist.is_initialized():
        kw = dict(backend=backend, timeout=datetime.timedelta(seconds=timeout_s))
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(**kw)
    return ws, rank, local


def shard(n: int, rank: int, world: int) -> slice:
    """Contiguous share of rank `rank` among n units (the first n % world ranks get one more)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside world of {world}")
    base, extra = divmod(n, world)
    start = rank * base + min(rank, extra)
    return slice(start, start + base + (1 if rank < extra else 0))


def grad_buffer(H: int, K: int, V: int, R: int, device):
    """One flat fp32 buffer holding dA [H,K,R] and then dB [H,R,V]; returns (flat, dA, dB),
    the last two views of the first (dB starts on a 16-byte boundary since K*R*4 does)."""
    import torch
    flat = torch.empty(H * R * (K + V), dtype=torch.float32, device=device)
    return flat, flat[:H * K * R].view(H, K, R), flat[H * K * R:].view(H, R, V)


def param_grad_buffer(H: int, K: int, V: int, R: int, device, write_term: bool = False, decay: bool = False):
    """One flat fp32 buffer for every per-head parameter gradient of a step: dA [H,K,R], dB
    [H,R,V], and (write_term) dAw [H,R], (decay) dA_dec [H] and dtau [H,K].  Returns (flat,
    views by name); each view starts on a 16-byte boundary (sections padded to 4 floats), as
    the library requires of every pointer."""
    import torch
    shapes = {"dA": (H, K, R), "dB": (H, R, V)}
    if write_term:
        shapes["dAw"] = (H, R)
    if decay:
        shapes["dA_dec"] = (H,)
        shapes["dtau"] = (H, K)
    offs, n = {}, 0
    for name, shp in shapes.items():
        size = 1
        for x in shp:
            size *= x
        offs[name] = (n, size)
        n += (size + 3) // 4 * 4
    flat = torch.zeros(n, dtype=torch.float32, device=device)
    return flat, {name: flat[o:o + size].view(shapes[name]) for name, (o, size) in offs.items()}


def allreduce_(flat, group=None):
    """Sum the factor gradients over the ranks, in place (no-op on one process)."""
    import torch.distributed as dist
    if dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
    return flat


def barrier(device=None):
    """Barrier over the ranks, then wait for this rank's GPU work (when a device is given)."""
    import torch
    import torch.distributed as dist
    if dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()
    if device is not None and device.type == "cuda":
        torch.cuda.synchronize(device)


def max_over_ranks(x: float, device=None) -> float:
    """Largest value of x over the ranks (times are reported as the slowest rank's)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_initialized() and dist.get_world_size() > 1):
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
