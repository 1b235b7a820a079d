"""Expert parallelism over peer memory (moe_ep_dispatch_send, or moe_dispatch
then moe_ep_send; moe_ep_wait, moe_dispatch_slots, moe_ep_return; through
the C ABI), on one GPU.

G ranks are emulated in this process (``PeerExpertParallelMoE.emulate``):
their arenas are ordinary device memory, each rank has its own tokens and
its E/G experts' weights, and each phase (send, experts, finish) is run for
every rank in turn on one stream, so every wait finds its flags already
published (the waits poll once) and no kernel waits for one that has not
run. The kernels are the ones a node runs over NVLink; only the addresses
differ. Each rank's output must equal the one-GPU forward of its tokens with
all the experts bit for bit (the same per-row arithmetic), over three
forwards in a row (epoch flags and block counters re-armed), including a
skewed problem with experts that get no rows and ranks that receive few.
"""

import pytest
import torch

import sparse_top_mixture_b200 as stm
import workloads
from sparse_top_mixture_b200.ep_peer import PeerExpertParallelMoE, ep_arena_offsets
from test_gpu_parity import SMALL

pytestmark = pytest.mark.gpu

# (workload, ranks, send fused into the dispatch)
CASES = [("qwen3_30b_a3b", 2, True), ("qwen3_30b_a3b", 4, True), ("deepseek_v2_lite_zipf", 4, True),
         ("dsv4_flash_ablation", 2, True), ("decode_weight_streaming", 8, True), ("tiny_fp32", 2, True),
         ("qwen3_30b_a3b", 1, True), ("qwen3_30b_a3b", 4, False), ("deepseek_v2_lite_zipf", 4, False),
         ("tiny_fp32", 2, False)]


def _setup(name, G, fused=True):
    cfg = SMALL[name]
    p = stm.Problem.from_config(cfg)
    cpu = workloads.generate(cfg, "cpu")
    dev = {k: (v.cuda() if v is not None else None) for k, v in cpu.items()}
    return cfg, p, dev, PeerExpertParallelMoE.emulate(p, dev, G, fused=fused)


@pytest.mark.parametrize("name,G,fused", CASES)
def test_emulated_ranks_match_the_one_gpu_forward(name, G, fused):
    cfg, p, dev, layers = _setup(name, G, fused)
    ref_layer = stm.SparseMoE(p, dev)
    for step in range(3):
        xs = [workloads.router_inputs(cfg, rank=r + G * step)["x"].cuda() for r in range(G)]
        for layer, x in zip(layers, xs):
            layer.send(x)
        for layer in layers:
            layer.experts()
        got = [layer.finish() for layer in layers]
        torch.cuda.synchronize()
        for r, (layer, x, (out, rw, sel)) in enumerate(zip(layers, xs, got)):
            ref_out, ref_rw, ref_sel = ref_layer(x)
            torch.cuda.synchronize()
            assert int(layer.err.item()) == 0, f"rank {r}: a wait gave up"
            assert torch.equal(sel, ref_sel), f"{name} G={G} rank {r} step {step}: selection"
            assert torch.equal(rw, ref_rw), f"{name} G={G} rank {r} step {step}: routing weights"
            assert torch.equal(out, ref_out), (
                f"{name} G={G} rank {r} step {step}: max diff {(out.float() - ref_out.float()).abs().max().item()}")


def test_a_wait_for_a_flag_nobody_publishes_gives_up_and_flags_it():
    cfg, p, dev, layers = _setup("qwen3_30b_a3b", 2)
    layer = layers[0]
    # this rank's epoch moves to 5, which no source has published: the wait
    # polls 1000 times, raises the timeout bit and returns; the stream and
    # context stay usable
    layer.epoch.fill_(5)
    stm.lib().moe_ep_wait(stm.ctypes.byref(p.c()), 2, layer.arena.data_ptr(), 0, 1000, layer.err.data_ptr(),
                          stm._stream(layer.arena.device))
    torch.cuda.synchronize()
    assert int(layer.err.item()) == stm.DEVERR_WAIT_TIMEOUT
    x = torch.ones(4, device="cuda")
    assert float((x * 2).sum().item()) == 8.0


def test_arena_layout_matches_the_views():
    cfg, p, dev, layers = _setup("deepseek_v2_lite_zipf", 4)
    off = ep_arena_offsets(p, 4)
    C = p.T * p.k
    layer = layers[1]
    base = layer.arena.data_ptr()
    assert layer.recv_x.data_ptr() == base + off["x"] and layer.recv_x.shape == (4 * C, p.H)
    assert layer.recv_w.data_ptr() == base + off["w"] and layer.recv_id.data_ptr() == base + off["id"]
    assert layer.y.data_ptr() == base + off["y"] and layer.y.shape == (C, p.H)


def test_emulated_ranks_replay_as_one_cuda_graph():
    """All phases of two emulated ranks captured once (global capture mode)
    and replayed: each replay advances the epochs on the device, and each
    rank's output matches the one-GPU forward of its tokens."""
    cfg, p, dev, layers = _setup("qwen3_30b_a3b", 2)
    ref_layer = stm.SparseMoE(p, dev)
    xs = [workloads.router_inputs(cfg, rank=r)["x"].cuda() for r in range(2)]
    outs = [None, None]

    def run():
        for layer, x in zip(layers, xs):
            layer.send(x)
        for layer in layers:
            layer.experts()
        for r, layer in enumerate(layers):
            outs[r] = layer.finish()[0]

    run()  # first run outside the capture: workspaces and streams exist
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, capture_error_mode="global"):
        run()
    for step in range(3):
        for r, x in enumerate(xs):
            x.copy_(workloads.router_inputs(cfg, rank=10 + 2 * step + r)["x"].cuda())
        graph.replay()
        torch.cuda.synchronize()
        for r, layer in enumerate(layers):
            assert int(layer.err.item()) == 0
            assert int(layer.epoch.item()) == 2 + step  # the first run, then one per replay (capture runs nothing)
            assert torch.equal(outs[r], ref_layer(xs[r])[0]), f"replay {step} rank {r}"
    del graph
