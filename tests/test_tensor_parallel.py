"""Tensor parallelism's host orchestration (sparse_top_mixture_b200/tensor_parallel.py)
with gloo ranks on the CPU.

The weight sharding is checked against the full weights directly. The whole
layer (replicated routing, each rank's slice of every expert, the fp32
all-reduce of the partial outputs, one rounding) runs on 1, 2 and 4 gloo ranks
with the library's stage calls replaced, inside each test process only, by
CPU stand-ins with the same contracts built from the oracle; every rank's
output must equal the oracle's one-process forward with unsharded experts. A
planted sharding mistake must break that equality."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from sparse_top_mixture_b200 import tensor_parallel as tp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_shards_reassemble_the_full_weights():
    E, I, H, Is, G = 3, 16, 8, 8, 4
    g = torch.Generator().manual_seed(0)
    full = {"gate_w": torch.randn(E, H, generator=g), "gate_up": torch.randn(E, 2 * I, H, generator=g),
            "down": torch.randn(E, H, I, generator=g), "shared_gate_up": torch.randn(2 * Is, H, generator=g),
            "shared_down": torch.randn(H, Is, generator=g)}
    shards = [tp.shard_expert_weights(full, r, G) for r in range(G)]
    for key, n in (("gate_up", I), ("shared_gate_up", Is)):
        s = n // G
        gate = torch.cat([sh[key][..., :s, :] for sh in shards], dim=-2)
        up = torch.cat([sh[key][..., s:, :] for sh in shards], dim=-2)
        assert torch.equal(gate, full[key][..., :n, :]) and torch.equal(up, full[key][..., n:, :])
    assert torch.equal(torch.cat([sh["down"] for sh in shards], dim=-1), full["down"])
    assert torch.equal(torch.cat([sh["shared_down"] for sh in shards], dim=-1), full["shared_down"])
    assert all(sh["gate_w"] is full["gate_w"] for sh in shards)
    with pytest.raises(ValueError):
        tp.shard_expert_weights(full, 0, 3)


CASES = {
    "softmax_plain": dict(T=11, H=16, E=6, k=2, I=32, I_shared=32, score="softmax", bias_mode="logit",
                          renormalize=False, shared="plain", bias_kind="uniform0.1"),
    "sigmoid_gated": dict(T=7, H=24, E=8, k=3, I=64, I_shared=32, score="sigmoid", bias_mode="none",
                          renormalize=True, shared="sigmoid_gated"),
    "sqrtsoftplus_select": dict(T=9, H=16, E=5, k=2, I=32, I_shared=0, score="sqrtsoftplus", bias_mode="select",
                                renormalize=True, shared="none", bias_kind="uniform0.1"),
}


def _worker(rank, world, port, case, planted, q):
    import torch.distributed as dist

    import oracle
    import sparse_top_mixture_b200 as stm
    import stage_standins
    import workloads

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        stage_standins.install(tp)
        cfg = workloads.CONFIGS["tiny_fp32"].replace(name="tp", **CASES[case])
        full = workloads.generate(cfg, "cpu")
        w = tp.shard_expert_weights(full, rank, world)
        if planted:  # up rows taken from the next rank's slice
            other = tp.shard_expert_weights(full, (rank + 1) % world, world)
            s = cfg.I // world
            w["gate_up"] = torch.cat([w["gate_up"][:, :s], other["gate_up"][:, s:]], dim=1).contiguous()
        layer = tp.TensorParallelMoE(stm.Problem.from_config(cfg), w)
        out, rw, sel = layer(full["x"])
        n = workloads.to_numpy64
        ref = oracle.moe_forward(n(full["x"]), n(full["gate_w"]), n(full["gate_up"]), n(full["down"]), k=cfg.k,
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


def _run(world, case, planted=False):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, case, planted, q)) for r in range(world)]
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
def test_tensor_parallel_matches_one_process_oracle(world, case):
    for rank, rel, same, _ in _run(world, case):
        assert same, f"rank {rank}: selection differs"
        assert rel <= 1e-6, f"rank {rank}: rel L2 {rel:.3e}"


def test_planted_sharding_mistake_is_caught():
    res = _run(2, "sigmoid_gated", planted=True)
    assert min(rel for _, rel, _, _ in res) > 1e-3
