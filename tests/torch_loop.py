"""A plain PyTorch per-expert loop of the MoE FFN forward, for a given
expert choice ("Sparse MoE FFN for DFlash-family drafters", Tests: grouped-
GEMM outputs and gradients against a sorted per-expert loop). Written with
torch.nn.functional only; its gradients come from torch autograd. Used as an
independent reference on the GPU (fp32) and as a pin of the backward oracle
on the CPU (fp64)."""

import torch
import torch.nn.functional as F

GRAD_OF = {"x": "dx", "gate_w": "d_gate_w", "bias": "d_bias", "gate_up": "d_gate_up", "down": "d_down",
           "shared_gate_up": "d_shared_gate_up", "shared_down": "d_shared_down", "shared_gate": "d_shared_gate"}


def swiglu(X, gu, dn):
    I = gu.shape[0] // 2
    return F.linear(F.silu(F.linear(X, gu[:I])) * F.linear(X, gu[I:]), dn)


def forward(cfg, t, sel):
    """out [T,H] of the per-expert loop for the choice ``sel`` [T,k] (int64),
    from tensors ``t`` (x, gate_w, bias, gate_up, down, shared weights)."""
    L = F.linear(t["x"], t["gate_w"])
    if cfg.bias_mode == "logit":
        L = L + t["bias"]
    if cfg.score == "softmax":
        S = torch.softmax(L, dim=1)
    elif cfg.score == "sigmoid":
        S = torch.sigmoid(L)
    else:
        S = torch.sqrt(F.softplus(L))
    w = S.gather(1, sel)
    if cfg.renormalize:
        w = w / w.sum(dim=1, keepdim=True)
    out = torch.zeros_like(t["x"])
    for e in range(cfg.E):
        tok, slot = (sel == e).nonzero(as_tuple=True)
        if tok.numel() == 0:
            continue
        y = swiglu(t["x"][tok], t["gate_up"][e], t["down"][e]) * w[tok, slot][:, None]
        out = out.index_add(0, tok, y)
    if cfg.shared != "none":
        s = swiglu(t["x"], t["shared_gate_up"], t["shared_down"])
        if cfg.shared == "sigmoid_gated":
            s = s * torch.sigmoid(t["x"] @ t["shared_gate"])[:, None]
        out = out + s
    return out
