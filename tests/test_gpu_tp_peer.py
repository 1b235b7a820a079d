"""Tensor parallelism over peer memory (moe_tp_scatter / moe_tp_wait /
moe_tp_gather through the C ABI), on one GPU.

G ranks are emulated in this process (``PeerTensorParallelMoE.emulate``):
arenas in ordinary device memory, every expert's I sharded over the ranks,
every rank given the same tokens, and each phase (partial, reduce, finish)
run for every rank in turn on one stream, so every wait finds its flags
already published. The output must be, bit for bit, each rank's fp32
combine of its partial rows (the library's moe_combine on them) summed over
the ranks in rank order and rounded once, on every rank; with G = 1 that is
the one-GPU forward itself. Three forwards in a row, fp32 and bf16, with
plain and gated shared experts; and against the fp64 oracle within the
problem's tolerance.
"""

import dataclasses

import pytest
import torch

import gpu_check as gc
import sparse_top_mixture_b200 as stm
import workloads
from sparse_top_mixture_b200.tp_peer import PeerTensorParallelMoE
from test_gpu_parity import SMALL

pytestmark = pytest.mark.gpu

CASES = [("dsv4_flash_ablation", 1), ("dsv4_flash_ablation", 2), ("dsv4_flash_ablation", 4),
         ("decode_weight_streaming", 4), ("decode_weight_streaming", 8), ("tiny_fp32", 2), ("tiny_fp32", 4)]


@pytest.mark.parametrize("name,G", CASES)
def test_emulated_ranks_sum_the_partials_in_rank_order(name, G):
    cfg = SMALL[name]
    p = stm.Problem.from_config(cfg)
    cpu = workloads.generate(cfg, "cpu")
    dev = {k: (v.cuda() if v is not None else None) for k, v in cpu.items()}
    layers = PeerTensorParallelMoE.emulate(p, dev, G)
    one = stm.SparseMoE(p, dev)
    for step in range(3):
        x = workloads.router_inputs(cfg, rank=step)["x"].cuda()
        for layer in layers:
            layer.partial(x)
        for layer in layers:
            layer.reduce()
        got = [layer.finish() for layer in layers]
        # the reference: each rank's fp32 combine of its partial rows, summed in rank order, rounded once
        acc = None
        for layer in layers:
            d, y, shared = layer._st["keep"]
            part = stm.combine(dataclasses.replace(layer.local, dtype="f32"), y, d["pair_pos"], shared)
            acc = part.clone() if acc is None else acc + part
        ref = acc.to(p.torch_dtype)
        torch.cuda.synchronize()
        for r, (layer, (out, rw, sel)) in enumerate(zip(layers, got)):
            assert int(layer.err.item()) == 0, f"rank {r}: a wait gave up"
            assert torch.equal(out, ref), f"{name} G={G} rank {r} step {step}"
        if G == 1:
            assert torch.equal(got[0][0], one(x)[0]), f"{name}: G=1 differs from the one-GPU forward"
        if step == 0:  # and the layer against the fp64 oracle, for its own expert choice
            gsel = got[0][2].cpu().numpy()
            o = gc.oracle_forward(cfg, {**cpu, "x": x.cpu()}, selected=gsel)
            gc.assert_close(got[0][0].cpu().double().numpy(), o["out"], cfg.dtype, f"{name} G={G}")


def test_a_tp_wait_for_a_flag_nobody_publishes_gives_up_and_flags_it():
    cfg = SMALL["dsv4_flash_ablation"]
    p = stm.Problem.from_config(cfg)
    cpu = workloads.generate(cfg, "cpu")
    dev = {k: (v.cuda() if v is not None else None) for k, v in cpu.items()}
    layer = PeerTensorParallelMoE.emulate(p, dev, 2)[0]
    layer.epoch.fill_(3)
    stm.lib().moe_tp_wait(stm.ctypes.byref(p.c()), 2, layer.arena.data_ptr(), 1, 500, layer.err.data_ptr(),
                          stm._stream(layer.arena.device))
    torch.cuda.synchronize()
    assert int(layer.err.item()) == stm.DEVERR_WAIT_TIMEOUT
