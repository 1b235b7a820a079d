"""Expert parallelism's host orchestration (sparse_top_mixture_b200/expert_parallel.py)
with gloo ranks on the CPU.

The exchange plan (which rows go to and come from which rank) is checked by
brute force. The whole exchange (counts; this rank's own rows through its
experts before the host read; rows, weights and local expert ids to the other
ranks, the receiver's regrouping by local expert, rows back; the combine)
runs on 1, 2 and 4 gloo ranks with the library's stage calls replaced,
inside each test process only, by CPU stand-ins with the same contracts built
from the oracle; each rank's output must equal the oracle's one-process
forward of its own tokens with all experts. A planted mistake in the local
expert ids sent with the rows must break that equality."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from sparse_top_mixture_b200 import expert_parallel as ep


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


# ---- split arithmetic ---------------------------------------------------------

def test_send_splits_sum_each_ranks_experts():
    counts = [3, 0, 5, 1, 0, 0, 7, 2]
    assert ep.send_splits(counts, 1) == [18]
    assert ep.send_splits(counts, 2) == [9, 9]
    assert ep.send_splits(counts, 4) == [3, 6, 0, 9]
    assert ep.send_splits(counts, 8) == counts
    with pytest.raises(ValueError):
        ep.send_splits(counts, 3)


def test_exchange_plan_brute_force():
    rng = np.random.default_rng(0)
    for _ in range(50):
        G, El = int(rng.integers(1, 5)), int(rng.integers(1, 5))
        rank = int(rng.integers(0, G))
        counts = rng.integers(0, 4, size=G * El)
        rc = rng.integers(0, 4, size=(G, El))
        plan = ep.exchange_plan(counts, rc, rank)
        # rank s's rows in x_perm: the rows of experts [s El, (s+1) El), after those of lower ranks
        for s in range(G):
            assert plan.send_off[s] == int(counts[:s * El].sum())
            assert plan.send_off[s + 1] - plan.send_off[s] == int(counts[s * El:(s + 1) * El].sum())
        assert plan.remote == [s for s in range(G) if s != rank]
        # receive buffers: remote sources in rank order, each source's rows contiguous
        at = 0
        for s in plan.remote:
            assert plan.recv_off[s] == at and plan.recvs[s] == int(rc[s].sum())
            at += int(rc[s].sum())
        assert plan.n_recv == at


def test_local_expert_ids():
    g = torch.tensor([8, 9, 11, 15])
    assert ep.local_expert_ids(g, 2, 4).tolist() == [0, 1, 3, 7]


CASES = {
    "softmax_plain": dict(T=13, H=16, E=8, k=2, I=8, I_shared=8, score="softmax", bias_mode="logit",
                          renormalize=False, shared="plain", bias_kind="uniform0.1"),
    "sigmoid_gated": dict(T=17, H=24, E=8, k=3, I=16, I_shared=8, score="sigmoid", bias_mode="none",
                          renormalize=True, shared="sigmoid_gated"),
    "sqrtsoftplus_select": dict(T=9, H=16, E=8, k=4, I=8, I_shared=0, score="sqrtsoftplus", bias_mode="select",
                                renormalize=True, shared="none", bias_kind="uniform0.1"),
}


def _worker(rank, world, port, case, planted, q, skew=False):
    import torch.distributed as dist

    import oracle
    import sparse_top_mixture_b200 as stm
    import stage_standins
    import workloads

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        stage_standins.install(ep)
        if planted:  # rows sent with their owner's local expert ids in reverse order
            ep.local_expert_ids = lambda g, owner, El: (owner + 1) * El - 1 - g
        cfg = workloads.CONFIGS["tiny_fp32"].replace(name="ep", **CASES[case])
        full = workloads.generate(cfg, "cpu")
        if skew:  # a selection bias that sends every pair to rank 0's experts
            full["bias"] = (torch.arange(cfg.E) < cfg.E // world).float() * 10.0
        mine = workloads.router_inputs(cfg, rank=rank)  # this rank's own batch
        El = cfg.E // world
        w = dict(full, gate_up=full["gate_up"][rank * El:(rank + 1) * El].contiguous(),
                 down=full["down"][rank * El:(rank + 1) * El].contiguous())
        p = stm.Problem.from_config(cfg)
        layer = ep.ExpertParallelMoE(p, w)
        out, rw, sel = layer(mine["x"])
        n = workloads.to_numpy64
        ref = oracle.moe_forward(n(mine["x"]), n(full["gate_w"]), n(full["gate_up"]), n(full["down"]), k=cfg.k,
                                 score=cfg.score, renormalize=cfg.renormalize, bias=n(full.get("bias")),
                                 bias_mode=cfg.bias_mode, shared=cfg.shared,
                                 shared_gate_up=n(full.get("shared_gate_up")),
                                 shared_down=n(full.get("shared_down")), shared_gate=n(full.get("shared_gate")))
        got = out.double().numpy()
        rel = float(np.linalg.norm(got - ref["out"]) / np.linalg.norm(ref["out"]))
        same = bool(np.array_equal(sel.numpy(), ref["selected_experts"]))
        q.put((rank, rel, same, None))
    except Exception as exc:  # reported to the parent, which fails the test
        q.put((rank, None, None, repr(exc)))
    finally:
        dist.destroy_process_group()


def _run(world, case, planted=False, skew=False):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, case, planted, q, skew)) for r in range(world)]
    for pr in procs:
        pr.start()
    res = sorted(q.get(timeout=180) for _ in procs)
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    for rank, rel, same, err in res:
        assert err is None, f"rank {rank}: {err}"
    return res


@pytest.mark.parametrize("world", [1, 2, 4])
@pytest.mark.parametrize("case", list(CASES))
def test_expert_parallel_matches_one_process_oracle(world, case):
    for rank, rel, same, _ in _run(world, case):
        assert same, f"rank {rank}: selection differs"
        assert rel <= 1e-6, f"rank {rank}: rel L2 {rel:.3e}"


def test_planted_local_id_mistake_is_caught():
    res = _run(2, "sigmoid_gated", planted=True)
    assert max(rel for _, rel, _, _ in res) > 1e-3


def test_ranks_that_receive_no_rows():
    """A selection bias sends every pair to rank 0's experts: the other ranks
    receive nothing, send everything, and still finish their own tokens."""
    for rank, rel, same, _ in _run(2, "sqrtsoftplus_select", skew=True):
        assert same, f"rank {rank}: selection differs"
        assert rel <= 1e-6, f"rank {rank}: rel L2 {rel:.3e}"


def _leaving_worker(rank, world, port, q):
    """Rank 1 leaves before the layer's first exchange; rank 0 must get an
    error from its collective (peer gone, or the group's short timeout), not
    wait forever."""
    import datetime

    import torch.distributed as dist

    import sparse_top_mixture_b200 as stm
    import stage_standins
    import workloads

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=10))
    def report(msg):
        q.put((rank, msg))
        q.close()
        q.join_thread()  # flushed before the process ends

    if rank == 1:
        report("left")
        os._exit(0)  # leaves between steps: nothing of its own is in flight
    try:
        stage_standins.install(ep)
        cfg = workloads.CONFIGS["tiny_fp32"].replace(name="ep", **CASES["softmax_plain"])
        full = workloads.generate(cfg, "cpu")
        El = cfg.E // world
        w = dict(full, gate_up=full["gate_up"][:El].contiguous(), down=full["down"][:El].contiguous())
        ep.ExpertParallelMoE(stm.Problem.from_config(cfg), w)(full["x"])
        msg = "no error"
    except Exception as exc:
        msg = "error: " + type(exc).__name__
    report(msg)
    os._exit(0)


def test_a_rank_that_leaves_ends_the_others_exchange_with_an_error():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_leaving_worker, args=(r, 2, port, q)) for r in range(2)]
    for pr in procs:
        pr.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for pr in procs:
        pr.join(timeout=60)
    assert res[1] == "left"
    assert res[0].startswith("error"), res[0]
