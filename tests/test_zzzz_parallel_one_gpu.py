"""The expert- and tensor-parallel layers on one GPU, through the real CUDA
kernels and NCCL, as a one-rank process group (the all-to-alls and the
all-reduce then move data only within the GPU; nothing waits on another
rank). Outputs are checked against the fp64 oracle like the forward parity
tests. The layers' multi-rank exchange logic is covered on gloo ranks by
tests/test_expert_parallel.py and tests/test_tensor_parallel.py.

Each case runs in a child process of its own so that the process group
never outlives it; this file is collected last."""

import os
import socket

import pytest
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

CASES = ("qwen3_30b_a3b", "deepseek_v2_lite_zipf", "decode_weight_streaming")


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _child(name, port, q):
    import datetime

    import torch
    import torch.distributed as dist

    import gpu_check as gc
    import sparse_top_mixture_b200 as stm
    import workloads
    from sparse_top_mixture_b200.expert_parallel import ExpertParallelMoE
    from sparse_top_mixture_b200.tensor_parallel import TensorParallelMoE, shard_expert_weights
    from test_gpu_parity import SMALL

    try:
        torch.cuda.set_device(0)
        dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                                timeout=datetime.timedelta(seconds=60))
        cfg = SMALL[name]
        cpu = workloads.generate(cfg, "cpu")
        dev = {k: (v.cuda() if v is not None else None) for k, v in cpu.items()}
        p = stm.Problem.from_config(cfg)
        ref_out = stm.SparseMoE(p, dev)(dev["x"])[0]
        r = gc.oracle_route(cfg, cpu)
        res = {}
        ep_layer = ExpertParallelMoE(p, dev)
        # The expert-parallel layer enqueues its own rows' GEMM (and the shared
        # expert) before its one host read of the counts, on a second stream:
        # when that read is entered the local GEMM's event has been recorded,
        # on a stream other than the one the read synchronises.
        seen = {}
        host_counts = ep_layer._host_counts

        def watched(counts, recv_counts):
            seen["recorded_before_read"] = hasattr(ep_layer, "local_done") and "local_experts" in ep_layer.trace
            seen["on_second_stream"] = (ep_layer.side is not None and
                                        ep_layer.side.cuda_stream != torch.cuda.current_stream().cuda_stream)
            return host_counts(counts, recv_counts)
        ep_layer._host_counts = watched
        layers = (("ep", ep_layer), ("tp", TensorParallelMoE(p, shard_expert_weights(dev, 0, 1))))
        for label, layer in layers:
            out, rw, sel = layer(dev["x"])
            torch.cuda.synchronize()
            if label == "ep":
                want = ["local_experts"] + (["shared_expert"] if cfg.shared != "none" else []) + ["host_counts"]
                assert ep_layer.trace == want, ep_layer.trace
                assert seen == {"recorded_before_read": True, "on_second_stream": True}, seen
                assert ep_layer.local_done.query()  # joined before the combine
            gsel = sel.cpu().numpy()
            ntie = gc.check_selection(cfg, r, gsel)
            assert ntie == gc.expected_near_ties(cfg.name), f"{name} {label}: {ntie} near-tie tokens"
            o = gc.oracle_forward(cfg, cpu, selected=gsel)
            stats = gc.assert_close(out.cpu().double().numpy(), o["out"], cfg.dtype, f"{name} {label}")
            res[label] = (stats["rel_l2"], float((out.float() - ref_out.float()).abs().max()))
        dist.destroy_process_group()
        q.put((name, res, None))
    except Exception as exc:  # reported to the parent, which fails the test
        q.put((name, None, repr(exc)[:2000]))


@pytest.mark.parametrize("name", CASES)
def test_parallel_layers_on_one_gpu_match_the_oracle(name):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    proc = ctx.Process(target=_child, args=(name, _free_port(), q))
    proc.start()
    try:
        got = q.get(timeout=600)
    finally:
        proc.join(timeout=120)
        if proc.is_alive():
            proc.kill()
    assert got[2] is None, got[2]
    assert proc.exitcode == 0
    print(name, got[1])
