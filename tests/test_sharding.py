"""Multi-rank sharding logic on CPU: plane shards cover every plane exactly once, and with
world_size-2 gloo ranks the sharded computation (per-shard float64 oracle standing in for the
per-rank library call) plus the channel-shared da all-reduce reproduces the unsharded result."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from linear_spatial_propagation_gspn_b200 import sharding


@pytest.mark.parametrize("N,C,world", [(16, 8, 2), (16, 8, 8), (1, 1152, 8), (3, 5, 2), (1, 7, 4), (5, 3, 4), (2, 2, 2)])
def test_plan_covers_every_plane_once(N, C, world):
    seen = np.zeros((N, C), dtype=int)
    for r in range(world):
        s = sharding.plan(N, C, world, r)
        if s.axis == "N":
            seen[s.start:s.stop, :] += 1
        else:
            seen[:, s.start:s.stop] += 1
    assert (seen == 1).all()


def test_plan_rejects_too_few_planes():
    with pytest.raises(ValueError):
        sharding.plan(1, 2, 4, 0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, N, C, wmode, errq):
    try:
        import oracle
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        dist.init_process_group("gloo", rank=rank, world_size=world)
        rng = np.random.default_rng(123)
        H, W, mask = 5, 6, 15
        Cw = 1 if wmode else C
        x = rng.standard_normal((N, C, H, W))
        a = rng.standard_normal((4, N, Cw, 3, H, W))
        lam = rng.uniform(0, 1, (N, C, H, W))
        u = rng.standard_normal((N, C, H, W))
        dy = rng.standard_normal((N, C, H, W))
        full_y = oracle.forward(x, a, lam, u, wmode, mask)
        full_g = oracle.backward(x, a, lam, u, dy, wmode, mask)
        sh = sharding.plan(N, C, world, rank)
        T = lambda v: torch.from_numpy(np.ascontiguousarray(v))
        xs, ls, us, dys = (sharding.take(T(v), sh).numpy() for v in (x, lam, u, dy))
        as_ = sharding.take(T(a), sh, logits=True, shared=bool(wmode)).numpy()
        ys = oracle.forward(xs, as_, ls, us, wmode, mask)
        dxs, das, dls, dus = oracle.backward(xs, as_, ls, us, dys, wmode, mask)
        da_t = torch.from_numpy(np.ascontiguousarray(das))
        sharding.allreduce_da(da_t, sh, bool(wmode))
        np.testing.assert_allclose(ys, sharding.take(T(full_y), sh).numpy(), atol=1e-12)
        np.testing.assert_allclose(dxs, sharding.take(T(full_g[0]), sh).numpy(), atol=1e-12)
        np.testing.assert_allclose(dus, sharding.take(T(full_g[3]), sh).numpy(), atol=1e-12)
        want_da = sharding.take(T(full_g[1]), sh, logits=True, shared=bool(wmode)).numpy()
        np.testing.assert_allclose(da_t.numpy(), want_da, atol=1e-11)
        dist.barrier()
        dist.destroy_process_group()
    except Exception as e:  # report to the parent
        errq.put(f"rank {rank}: {type(e).__name__}: {e}")


@pytest.mark.parametrize("N,C,wmode", [(1, 4, 1), (1, 4, 0), (4, 2, 1), (2, 3, 0)])
def test_two_gloo_ranks_match_unsharded(N, C, wmode):
    ctx = mp.get_context("spawn")
    errq = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, N, C, wmode, errq)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    errs = []
    while not errq.empty():
        errs.append(errq.get())
    assert all(p.exitcode == 0 for p in procs), errs
    assert not errs, errs
