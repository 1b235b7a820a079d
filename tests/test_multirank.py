"""The N-GPU bench path's host logic with two gloo ranks on the CPU: the max
over ranks of the timed region, whole-job throughput, and per-rank batches
that share every weight (data-parallel replicas, no collective on the data
path)."""

import os
import socket

import torch
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    import workloads
    cfg = workloads.CONFIGS["qwen3_30b_a3b"].replace(T=8, H=16, E=4, k=2, I=8)
    r = workloads.router_inputs(cfg, rank=rank)
    elapsed = 10.0 + 5.0 * rank  # the slower rank sets the job time
    m = bench.dist_max(elapsed, world)
    bench.barrier(world)
    q.put((rank, m, bench.job_throughput(world, cfg.T, 4, m), r["x"].float().sum().item(),
           r["gate_w"].float().sum().item()))
    dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (_, m0, v0, x0, w0), (_, m1, v1, x1, w1) = res
    assert m0 == m1 == 15.0
    assert v0 == v1 == 2 * 8 * 4 / 0.015
    assert x0 != x1  # independent batches
    assert w0 == w1  # same weights


def _balance_worker(rank, world, port, q):
    """Each rank stashes its own routing counts; the loads are summed over the
    ranks before the sign-controller step, so every rank moves its bias
    identically (the all-reduced loads of the balancer)."""
    import numpy as np
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import oracle.balance as ob
    import sparse_top_mixture_b200 as stm
    E = 8
    local = torch.tensor([[9, 0, 3, 4, 0, 0, 0, 0], [0, 0, 3, 4, 8, 1, 0, 0]][rank], dtype=torch.int64)
    loads = stm.allreduce_loads(local.clone())
    bias, left = ob.bias_update(np.zeros(E, np.float32), loads.numpy(), 0.125)
    q.put((rank, loads.tolist(), bias.tolist(), left.tolist()))
    dist.destroy_process_group()


def test_balancer_loads_are_summed_over_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_balance_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (_, l0, b0, z0), (_, l1, b1, z1) = res
    assert l0 == l1 == [9, 0, 6, 8, 8, 1, 0, 0]  # mean 4
    assert b0 == b1 == [-0.125, 0.125, -0.125, -0.125, -0.125, 0.125, 0.125, 0.125]
    assert z0 == z1 == [0] * 8
