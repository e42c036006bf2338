"""The data-parallel path on two CPU ranks (gloo): each rank takes its batch shard, the oracle
stands in for the kernels on that shard, and the one collective (the sum of dA and dB over
ranks, through the flat buffer the bench hands to carve_bwd) must reproduce the full batch's
factor gradients; every other gradient is per unit and must equal the full batch's slice.
Also: the shard arithmetic and the slowest-rank timing reduction."""
import multiprocessing as mp
import os
import socket

import numpy as np
import pytest

from chunk_gated_delta_b200 import dist as cdist
from chunk_gated_delta_b200 import inputs as I

WORLD = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _workload():
    import dataclasses
    return dataclasses.replace(I.TINY_FP32, B=5, T=128, L=32, seed=4242)


def _rank_main(rank, port, q):
    try:
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(WORLD), RANK=str(rank),
                          LOCAL_RANK=str(rank))
        import torch
        import oracle
        ws, r, _ = cdist.setup("gloo", timeout_s=60)
        assert (ws, r) == (WORLD, rank)
        w = _workload()
        d = I.make_inputs(w)
        dO = I.make_grad_out(w)
        sl = cdist.shard(w.B, rank, ws)
        sub = {k: (v[sl] if k not in ("A", "B") else v) for k, v in d.items()}
        g = oracle.bwd(sub, w.L, dO[sl], mc_mode=1)
        flat, dA, dB = cdist.grad_buffer(w.H, w.K, w.V, w.R, "cpu")
        dA.copy_(torch.from_numpy(g["dA"]))
        dB.copy_(torch.from_numpy(g["dB"]))
        cdist.allreduce_(flat)
        cdist.barrier()
        slowest = cdist.max_over_ranks(10.0 + rank)
        q.put((rank, flat.numpy().copy(), g["dq"], g["dS0"], slowest, None))
        import torch.distributed as dist
        dist.destroy_process_group()
    except Exception as e:   # noqa: BLE001 - reported to the parent
        q.put((rank, None, None, None, None, repr(e)))


@pytest.mark.timeout(300)
def test_two_rank_factor_gradient_allreduce():
    import oracle
    oracle.build()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, port, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(WORLD):
        rank, flat, dq, dS0, slowest, err = q.get(timeout=240)
        assert err is None, f"rank {rank}: {err}"
        res[rank] = (flat, dq, dS0, slowest)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w = _workload()
    d = I.make_inputs(w)
    full = oracle.bwd(d, w.L, I.make_grad_out(w), mc_mode=1)
    want = np.concatenate([full["dA"].ravel(), full["dB"].ravel()])
    for rank in range(WORLD):
        flat, dq, dS0, slowest = res[rank]
        assert np.linalg.norm(flat - want) <= 1e-6 * np.linalg.norm(want)   # fp32 buffer of fp64 sums
        sl = cdist.shard(w.B, rank, WORLD)
        np.testing.assert_allclose(dq, full["dq"][sl], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(dS0, full["dS0"][sl], rtol=1e-12, atol=1e-14)
        assert slowest == 10.0 + WORLD - 1


def test_shard_covers_every_unit_once():
    for n in (0, 1, 5, 8, 13):
        for world in (1, 2, 3, 8):
            got = []
            for r in range(world):
                sl = cdist.shard(n, r, world)
                got.extend(range(n)[sl])
            assert got == list(range(n))
    with pytest.raises(ValueError):
        cdist.shard(4, 2, 2)


def test_grad_buffer_views_share_storage():
    flat, dA, dB = cdist.grad_buffer(3, 8, 4, 2, "cpu")
    assert dA.shape == (3, 8, 2) and dB.shape == (3, 2, 4)
    flat.zero_()
    dA.fill_(1.0)
    dB.fill_(2.0)
    assert float(flat.sum()) == 3 * 8 * 2 * 1.0 + 3 * 2 * 4 * 2.0
    assert dB.data_ptr() - flat.data_ptr() == 3 * 8 * 2 * 4 and (dB.data_ptr() - flat.data_ptr()) % 16 == 0
    assert cdist.allreduce_(flat) is flat   # one process: no-op


def _rank_main_terms(rank, port, q):
    """As _rank_main, with the write gate's content term and the decay's amplitude and bias:
    every per-head parameter gradient goes through the one flat buffer."""
    try:
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(WORLD), RANK=str(rank),
                          LOCAL_RANK=str(rank))
        import torch
        import oracle
        ws, r, _ = cdist.setup("gloo", timeout_s=60)
        w = _workload()
        d = _with_terms(w, I.make_inputs(w))
        dO = I.make_grad_out(w)
        sl = cdist.shard(w.B, rank, ws)
        sub = {k: (v[sl] if k not in ("A", "B", "Aw", "A_dec", "tau") else v) for k, v in d.items()}
        g = oracle.bwd(sub, w.L, dO[sl], mc_mode=0)
        flat, views = cdist.param_grad_buffer(w.H, w.K, w.V, w.R, "cpu", write_term=True, decay=True)
        for name, view in views.items():
            view.copy_(torch.from_numpy(g[name]))
        cdist.allreduce_(flat)
        q.put((rank, {k: v.numpy().copy() for k, v in views.items()}, None))
        import torch.distributed as dist
        dist.destroy_process_group()
    except Exception as e:   # noqa: BLE001 - reported to the parent
        q.put((rank, None, repr(e)))


def _with_terms(w, d):
    d = dict(d)
    d["Aw"] = I.normal(w.seed, 97, (w.H, w.R), 0.0, 2.0).astype(np.float32)
    d.update(I.make_decay(w))
    return d


@pytest.mark.timeout(300)
def test_two_rank_parameter_gradients_with_optional_terms():
    import oracle
    oracle.build()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main_terms, args=(r, port, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(WORLD):
        rank, views, err = q.get(timeout=240)
        assert err is None, f"rank {rank}: {err}"
        res[rank] = views
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w = _workload()
    full = oracle.bwd(_with_terms(w, I.make_inputs(w)), w.L, I.make_grad_out(w), mc_mode=0)
    for rank in range(WORLD):
        for name in ("dA", "dB", "dAw", "dA_dec", "dtau"):
            got, want = res[rank][name], full[name]
            assert np.linalg.norm(got - want) <= 1e-6 * np.linalg.norm(want), (rank, name)


def test_param_grad_buffer_sections_aligned():
    flat, views = cdist.param_grad_buffer(3, 8, 4, 3, "cpu", write_term=True, decay=True)
    assert list(views) == ["dA", "dB", "dAw", "dA_dec", "dtau"]
    for name, v in views.items():
        assert (v.data_ptr() - flat.data_ptr()) % 16 == 0, name
        v.fill_(1.0)
    assert float(flat.sum()) == 3 * 8 * 3 + 3 * 3 * 4 + 3 * 3 + 3 + 3 * 8   # padding stays zero
