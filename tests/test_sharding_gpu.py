"""Data-parallel sharding through libgspn on the GPU.

Every rank of a simulated world (2 and 4 ranks) runs ``sharding.forward_shard`` and
``sharding.backward_shard`` on its own plane shard, one after another on the one GPU (the shards'
kernels never wait on one another). The channel-shared logit gradient of a channel-sharded plan
is summed over the ranks on the host, standing in for the NCCL all-reduce that
``sharding.allreduce_da`` issues under torchrun. The shards' outputs, put back together, are
compared with the float64 oracle on the unsharded problem at the contract tolerances. Batch and
channel plans, both weight modes, both storage dtypes."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import gspn_inputs
import oracle
from linear_spatial_propagation_gspn_b200 import sharding

from _cases import assert_close, f64, fwd_tol, grad_tol

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("N,C,world", [(4, 3, 2), (2, 5, 4), (1, 6, 2), (1, 8, 4), (3, 2, 2)])
@pytest.mark.parametrize("wmode", [0, 1])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_simulated_world_matches_oracle(N, C, world, wmode, dtype):
    wl = gspn_inputs.small_case(N, C, 40, 48, mask=15, wmode=wmode, dtype=dtype, seed=N * 10 + C + world)
    t = gspn_inputs.make_inputs(wl, device="cuda", with_dy=True)
    x, a, lam, u, dy = t["x"], t["a"], t["lam"], t["u"], t["dy"]
    y = torch.empty_like(x)
    dx, dlam, du = torch.empty_like(x), torch.empty_like(x), torch.empty_like(x)
    da = torch.zeros(a.shape, dtype=torch.float64, device="cuda")
    for rank in range(world):
        sh = sharding.plan(N, C, world, rank)
        ys = sharding.forward_shard(x, a, lam, u, wmode, 15, sh)
        gx, ga, gl, gu = sharding.backward_shard(x, a, lam, u, dy, wmode, 15, sh)
        sharding.take(y, sh).copy_(ys)
        sharding.take(dx, sh).copy_(gx)
        sharding.take(dlam, sh).copy_(gl)
        sharding.take(du, sh).copy_(gu)
        if sharding.needs_da_allreduce(sh, bool(wmode)):
            da += ga.double()                      # host-side stand-in for the all-reduce
        else:
            sharding.take(da, sh, logits=True, shared=bool(wmode)).copy_(ga.double())
    torch.cuda.synchronize()
    ref_y = oracle.forward(f64(x), f64(a), f64(lam), f64(u), wmode, 15)
    assert_close(f64(y), ref_y, fwd_tol(dtype, ref_y), f"sharded forward world={world}")
    ref = oracle.backward(f64(x), f64(a), f64(lam), f64(u), f64(dy), wmode, 15)
    for name, got, rr in zip(("dx", "da", "dlam", "du"), (dx, da, dlam, du), ref):
        # bf16: the channel-summed da is summed from bf16-rounded shard gradients
        assert_close(f64(got), rr, grad_tol(dtype, rr), f"sharded {name} world={world}")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, N, C, wmode, errq):
    """One gloo rank on the shared GPU: libgspn on this rank's shard, the channel-shared da
    summed across ranks by sharding.allreduce_da (gloo all-reduce of a CUDA tensor)."""
    try:
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        dist.init_process_group("gloo", rank=rank, world_size=world)
        torch.cuda.set_device(0)
        wl = gspn_inputs.small_case(N, C, 24, 32, mask=15, wmode=wmode, dtype="f32", seed=11 + N + C)
        t = gspn_inputs.make_inputs(wl, device="cuda", with_dy=True)
        sh = sharding.plan(N, C, world, rank)
        ys = sharding.forward_shard(t["x"], t["a"], t["lam"], t["u"], wmode, 15, sh)
        grads = sharding.backward_shard(t["x"], t["a"], t["lam"], t["u"], t["dy"], wmode, 15, sh)
        torch.cuda.synchronize()
        cpu = {k: f64(v) for k, v in t.items()}
        ref_y = oracle.forward(cpu["x"], cpu["a"], cpu["lam"], cpu["u"], wmode, 15)
        ref_g = oracle.backward(cpu["x"], cpu["a"], cpu["lam"], cpu["u"], cpu["dy"], wmode, 15)
        T = lambda v: torch.from_numpy(np.ascontiguousarray(v))
        want_y = sharding.take(T(ref_y), sh).numpy()
        assert_close(f64(ys), want_y, fwd_tol("f32", want_y), f"rank {rank} forward")
        for i, name in enumerate(("dx", "da", "dlam", "du")):
            want = sharding.take(T(ref_g[i]), sh, logits=(name == "da"), shared=bool(wmode)).numpy()
            assert_close(f64(grads[i]), want, grad_tol("f32", want), f"rank {rank} {name}")
        dist.barrier()
        dist.destroy_process_group()
    except Exception as e:  # report to the parent
        errq.put(f"rank {rank}: {type(e).__name__}: {e}")


@pytest.mark.parametrize("N,C,wmode", [(1, 4, 1), (1, 4, 0), (4, 2, 1)])
def test_two_gloo_ranks_run_libgspn(N, C, wmode):
    ctx = mp.get_context("spawn")
    errq = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, N, C, wmode, errq)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    errs = []
    while not errq.empty():
        errs.append(errq.get())
    assert all(p.exitcode == 0 for p in procs), errs
    assert not errs, errs
