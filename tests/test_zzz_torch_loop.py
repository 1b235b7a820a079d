"""fp32 parity of the forward and the backward against a plain PyTorch
per-expert loop on the GPU ("Sparse MoE FFN for DFlash-family drafters",
Tests: grouped-GEMM outputs and gradients against a sorted per-expert loop).

The loop (tests/torch_loop.py) is written with torch.nn.functional, here on
CUDA tensors in fp32 (TF32 off): router logits, scores and the routing
weights of the given choice, then for every expert the SwiGLU MLP of its
tokens, weighted and added back, plus the shared expert; its gradients come
from torch autograd. Both sides use the kernel's expert choice (the choice
itself is checked against the fp64 oracle by the parity tests). Tolerance:
relative L2 <= 1e-5 per tensor and every element within 1e-4 of the
tensor's largest magnitude, as for the backward oracle (two fp32
evaluations with different summation orders)."""

import pytest
import torch

import sparse_top_mixture_b200 as stm
import torch_loop
import workloads
from workloads import CONFIGS

pytestmark = pytest.mark.gpu

CASES = {
    "tiny_fp32": CONFIGS["tiny_fp32"],
    "sqrtsoftplus_select_gated": CONFIGS["tiny_fp32"].replace(
        name="loop_a", T=64, H=48, E=6, k=3, I=32, I_shared=16, score="sqrtsoftplus", bias_mode="select",
        bias_kind="uniform0.1", renormalize=True, shared="sigmoid_gated"),
    "sigmoid_logit_plain": CONFIGS["tiny_fp32"].replace(
        name="loop_b", T=50, H=40, E=5, k=2, I=24, I_shared=8, score="sigmoid", bias_mode="logit",
        bias_kind="uniform0.1", renormalize=False, shared="plain"),
}


def _close(got, ref, what):
    got, ref = got.double(), ref.double()
    rel = float(torch.linalg.norm(got - ref) / torch.linalg.norm(ref))
    assert rel <= 1e-5, f"{what}: rel L2 {rel:.3e}"
    assert float((got - ref).abs().max()) <= 1e-4 * float(ref.abs().max()), f"{what}: max abs"


@pytest.fixture(autouse=True)
def _no_tf32():
    old = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = False
    yield
    torch.backends.cuda.matmul.allow_tf32 = old


@pytest.mark.parametrize("name", list(CASES))
def test_forward_and_backward_match_a_torch_per_expert_loop(name):
    cfg = CASES[name]
    dev = {k: (v.cuda() if v is not None else None) for k, v in workloads.generate(cfg, "cpu").items()}
    p = stm.Problem.from_config(cfg)
    out, rw, sel = stm.SparseMoE(p, dev)(dev["x"])
    dout = torch.randn(p.T, p.H, generator=torch.Generator().manual_seed(9)).cuda()
    grads = stm.backward(p, dev, dev["x"], dout, sel)
    torch.cuda.synchronize()

    leaves = {k: v.detach().clone().requires_grad_(True) for k, v in dev.items() if v is not None}
    ref = torch_loop.forward(cfg, leaves, sel)
    _close(out, ref.detach(), f"{name} out")
    (ref * dout).sum().backward()
    for name_w, key in torch_loop.GRAD_OF.items():
        if grads.get(key) is None:
            continue
        _close(grads[key], leaves[name_w].grad, f"{name} {key}")
    if cfg.bias_mode == "select":
        assert grads["d_bias"] is None  # a selection bias gets no gradient
