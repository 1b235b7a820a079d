"""GPU parity of the bf16 backward (moe_backward on the tensor cores, through
the C ABI) against the fp64 backward oracle (oracle/backward.py), on the same
seeded bf16 inputs (converted exactly) and the oracle's own expert choice.

Tolerance. The GPU rounds four intermediates to bf16 where they become GEMM
operands: [dg du] (dx and dW_gate_up), w*dout and h (dW_down), and dlogits
(the router's dgate_w and its share of dx); each rounding
moves a value by at most 2^-9 of itself, products and sums are fp32. A
gradient element therefore carries a relative error of about one or two
bf16 roundings of the terms it sums (~1e-3 in L2 over a tensor, as for the
forward); the logit bias comes from fp32 dlogits.
The bar: relative L2 <= 5e-3 per tensor (the problem's bf16 output bar) and
no element off by more than 1e-2 of the tensor's largest magnitude.
"""

import numpy as np
import pytest
import torch

import gpu_check as gc
import oracle.backward as ob
import sparse_top_mixture_b200 as stm
import workloads
from workloads import CONFIGS, reduced

pytestmark = pytest.mark.gpu

KEYS = ("dx", "d_gate_w", "d_bias", "d_gate_up", "d_down", "d_shared_gate_up", "d_shared_down", "d_shared_gate")

NAMED = {
    "qwen3_30b_a3b": reduced(CONFIGS["qwen3_30b_a3b"], T=300, H=328, I=200),
    "deepseek_v2_lite_zipf": reduced(CONFIGS["deepseek_v2_lite_zipf"], T=512, H=256, I=136, I_shared=272),
    "dsv4_flash_ablation": reduced(CONFIGS["dsv4_flash_ablation"], T=384, H=512, I=256, I_shared=256),
    "decode_weight_streaming": reduced(CONFIGS["decode_weight_streaming"], T=16, H=1024, I=256, I_shared=256),
    # about 400 rows per expert: the data-gradient GEMMs run on CTA pairs, the
    # gate_up GEMM with the SwiGLU backward as its epilogue
    "pairs": CONFIGS["qwen3_30b_a3b"].replace(name="bw_pairs", T=1600, H=384, E=8, k=2, I=192),
    # the same for a sigmoid-gated shared expert over 1024 tokens (its dz from
    # the fused epilogue's dot partials), I and I_s not multiples of 128
    "pairs_gated": CONFIGS["decode_weight_streaming"].replace(name="bw_pairs_gated", T=1024, H=256, E=8, k=2,
                                                               I=136, I_shared=200),
}

GRID = {}
for _i, (_s, _b, _r) in enumerate([(s, b, r) for s in ("softmax", "sigmoid", "sqrtsoftplus")
                                   for b in ("none", "logit", "select") for r in (True, False)]):
    _sh = ("none", "plain", "sigmoid_gated")[_i % 3]
    GRID[f"{_s}-{_b}-{'renorm' if _r else 'raw'}-{_sh}"] = CONFIGS["tiny_fp32"].replace(
        name="grid16", T=37, H=40, E=6, k=3, I=24, I_shared=16 if _sh != "none" else 0, score=_s, bias_mode=_b,
        renormalize=_r, shared=_sh, bias_kind="none" if _b == "none" else "uniform0.1", seed=11 + _i, dtype="bf16")


def _oracle_grads(cfg, cpu, dout, sel):
    n = gc.np64
    return ob.moe_backward(n(cpu["x"]), n(cpu["gate_w"]), n(cpu["gate_up"]), n(cpu["down"]), dout, k=cfg.k,
                           score=cfg.score, renormalize=cfg.renormalize, bias=n(cpu.get("bias")),
                           bias_mode=cfg.bias_mode, shared=cfg.shared, shared_gate_up=n(cpu.get("shared_gate_up")),
                           shared_down=n(cpu.get("shared_down")), shared_gate=n(cpu.get("shared_gate")),
                           selected=sel)


def _check_grads(got, ref, what):
    worst = {}
    for key in KEYS:
        r = ref.get(key)
        g = got.get(key)
        assert (r is None) == (g is None), f"{what} {key}: presence differs"
        if r is None:
            continue
        assert g.dtype == torch.float32
        g = g.cpu().numpy().astype(np.float64)
        r = np.asarray(r, np.float64)
        assert g.shape == r.shape, (what, key, g.shape, r.shape)
        assert np.isfinite(g).all(), f"{what} {key}: non-finite"
        scale = max(np.abs(r).max(), 1e-30)
        rl = gc.rel_l2(g, r)
        ma = np.abs(g - r).max() / scale
        worst[key] = (rl, ma)
        assert rl <= 5e-3, f"{what} {key}: rel L2 {rl:.3e}"
        assert ma <= 1e-2, f"{what} {key}: max abs {ma:.3e} of the largest magnitude"
    return worst


def _run(cfg, sel=None, dout_seed=5):
    cpu = workloads.generate(cfg, "cpu")
    dev = {k: (v.cuda() if v is not None else None) for k, v in cpu.items()}
    if sel is None:
        sel = gc.oracle_route(cfg, cpu)["selected_experts"]
    dout = torch.randn(cfg.T, cfg.H, generator=torch.Generator().manual_seed(dout_seed)).to(torch.bfloat16)
    p = stm.Problem.from_config(cfg)
    ws = torch.zeros(stm.backward_workspace_size(p), dtype=torch.uint8, device="cuda")
    got = stm.backward(p, dev, dev["x"], dout.cuda(), torch.from_numpy(sel).cuda(), ws=ws)
    torch.cuda.synchronize()
    assert stm.read_device_error(ws) == 0
    ref = _oracle_grads(cfg, cpu, gc.np64(dout), sel)
    return got, ref


@pytest.mark.parametrize("name", list(NAMED))
def test_bf16_backward_matches_oracle_named(name):
    got, ref = _run(NAMED[name])
    print(name, _check_grads(got, ref, name))


@pytest.mark.parametrize("name", list(GRID))
def test_bf16_backward_matches_oracle_grid(name):
    got, ref = _run(GRID[name])
    _check_grads(got, ref, name)


def test_bf16_backward_experts_without_rows_get_zero_gradients():
    cfg = GRID["softmax-none-renorm-none"].replace(name="skew16", T=70, H=48, E=8, k=2, I=40)
    sel = np.tile(np.array([[3, 5]], dtype=np.int64), (cfg.T, 1))
    got, ref = _run(cfg, sel=sel)
    _check_grads(got, ref, "skew16")
    dgu, dd = got["d_gate_up"].cpu().numpy(), got["d_down"].cpu().numpy()
    for e in (0, 1, 2, 4, 6, 7):
        assert not dgu[e].any() and not dd[e].any()


def test_bf16_backward_is_deterministic():
    cfg = NAMED["dsv4_flash_ablation"]
    a, _ = _run(cfg)
    b, _ = _run(cfg)
    for key in KEYS:
        if a[key] is not None:
            assert torch.equal(a[key], b[key]), key


@pytest.mark.parametrize("name", ["dsv4_flash_ablation", "decode_weight_streaming"])
def test_bf16_backward_in_a_cuda_graph_matches_eager(name):
    """The whole backward captured as one CUDA graph (global capture mode:
    nothing in it may allocate or synchronise) replays to the eager call's
    gradients bit for bit."""
    cfg = NAMED[name]
    cpu = workloads.generate(cfg, "cpu")
    dev = {k: (v.cuda() if v is not None else None) for k, v in cpu.items()}
    sel = torch.from_numpy(gc.oracle_route(cfg, cpu)["selected_experts"]).cuda()
    dout = torch.randn(cfg.T, cfg.H, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16).cuda()
    p = stm.Problem.from_config(cfg)
    ws = torch.zeros(stm.backward_workspace_size(p), dtype=torch.uint8, device="cuda")
    eager = stm.backward(p, dev, dev["x"], dout, sel, ws=ws)
    eager = {k: (v.clone() if v is not None else None) for k, v in eager.items()}
    out = {k: torch.full_like(v, float("nan")) for k, v in eager.items() if v is not None}
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, capture_error_mode="global"):
        stm.backward(p, dev, dev["x"], dout, sel, ws=ws, out=out)
    for _ in range(2):
        graph.replay()
        torch.cuda.synchronize()
        for key, v in out.items():
            assert torch.equal(v, eager[key]), key
    del graph
    assert stm.read_device_error(ws) == 0


def test_bf16_backward_flags_bad_expert_id():
    """A pair with an expert id outside [0, E) contributes nothing (its
    routing-weight gradient is zero) and raises the workspace flag; every
    other token's dx is unchanged."""
    cfg = GRID["softmax-none-renorm-none"].replace(name="bad16", T=60, H=48, E=6, k=2, I=32, renormalize=False)
    cpu = workloads.generate(cfg, "cpu")
    dev = {k: (v.cuda() if v is not None else None) for k, v in cpu.items()}
    sel = gc.oracle_route(cfg, cpu)["selected_experts"].copy()
    sel[9, 1] = cfg.E + 2
    sel[30, 0] = -1
    p = stm.Problem.from_config(cfg)
    ws = torch.zeros(stm.backward_workspace_size(p), dtype=torch.uint8, device="cuda")
    dout = torch.randn(cfg.T, cfg.H, generator=torch.Generator().manual_seed(4)).to(torch.bfloat16)
    got = stm.backward(p, dev, dev["x"], dout.cuda(), torch.from_numpy(sel).cuda(), ws=ws)
    torch.cuda.synchronize()
    assert stm.read_device_error(ws) == stm.DEVERR_BAD_EXPERT_ID
    # without renormalisation a slot's weight is its own score: every token
    # but the two with a dropped pair matches the oracle of the valid choice
    ref = _oracle_grads(cfg, cpu, gc.np64(dout), np.where((sel < 0) | (sel >= cfg.E), 0, sel))
    dx = got["dx"].cpu().numpy().astype(np.float64)
    assert np.isfinite(dx).all()
    keep = ~np.isin(np.arange(cfg.T), [9, 30])
    assert gc.rel_l2(dx[keep], ref["dx"][keep]) <= 5e-3
