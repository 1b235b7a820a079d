"""Seeded synthetic workloads for the sparse top-k MoE FFN forward.

This module only draws random inputs. It holds none of the method's arithmetic
(no routing, no scores, no expert MLP): both the fp64 oracle and the CUDA path
consume what it returns, and neither is imported here.

The five named problem shapes follow the expert layouts the pages describe:

* ``tiny_fp32``: 8 experts, top-2 softmax with renormalisation, fp32.
* ``qwen3_30b_a3b``: 128 experts, top-8 (the Qwen3-30B-A3B routing shape in
  "MoE: shared experts, parameterized V_TOPK routing, explicit stage
  attribution", section 1 "C_SET_TOPK_REG").
* ``deepseek_v2_lite_zipf``: 64 experts, top-6 (DeepSeek-V2-Lite shape, same
  section) with two fused shared experts ("n_shared=2 fused", section 3
  "Tests" and section 4 "Route-trace schema v2") and a router logit bias that
  skews expert loads towards Zipf(1.2) with four dead experts.
* ``dsv4_flash_ablation``: 64 routed + 1 shared, top-6, intermediate 2048
  ("Sparse MoE FFN for DFlash-family drafters", "What's here", the DSV4-Flash
  ablation pair) with sqrtsoftplus scores and an fp32 selection-only bias.
* ``decode_weight_streaming``: 256 experts, top-8 (DeepSeek-V3 / Kimi K2
  shape) at 16 tokens, with a sigmoid-gated shared expert
  ("mstar.model.components.moe", SparseMoeBlockWithSharedExpert).

Draw recipe (every tensor has its own generator, seeded ``seed*1000 + id``):

* hidden states ``x ~ N(0, 1)``;
* router ``gate_w [E,H] ~ N(0, 1/H)``; shared gate vector ``[H] ~ N(0, 1/H)``;
* ``gate_up [E,2I,H] ~ N(0, 1/H)``; ``down [E,H,I] ~ N(0, 1/I)``;
* shared ``gate_up [2I_s,H] ~ N(0, 1/H)``, ``down [H,I_s] ~ N(0, 1/I_s)``;
* selection bias ``U(-0.1, 0.1)`` in fp32 (``dsv4_flash_ablation``);
* the Zipf logit bias of ``deepseek_v2_lite_zipf`` is a stored fp32 vector
  (``tests/golden/zipf_logit_bias_E64.json``), written offline by a script
  beside it.

Values are drawn in fp32 and rounded to bf16 round-to-nearest-even for the
bf16 problems. The router-side tensors (x, gate_w, biases, shared gate) are
always drawn on the CPU generator so that routing decisions do not depend on
the device. The large expert weights are drawn on the device the caller asks
for (CPU or CUDA Philox), one expert slab at a time.
"""

from __future__ import annotations

import dataclasses
import json
import os
from typing import Dict, Optional

import torch

SCORES = ("softmax", "sigmoid", "sqrtsoftplus")
BIAS_MODES = ("none", "logit", "select")
SHARED_KINDS = ("none", "plain", "sigmoid_gated")

_GOLDEN = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "tests", "golden")
ZIPF_BIAS_FILE = os.path.join(_GOLDEN, "zipf_logit_bias_E64.json")


@dataclasses.dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int
    H: int
    E: int
    k: int
    I: int
    I_shared: int
    dtype: str  # "f32" or "bf16"
    score: str  # one of SCORES
    bias_mode: str  # one of BIAS_MODES
    renormalize: bool
    shared: str  # one of SHARED_KINDS
    bias_kind: str = "none"  # "none", "uniform0.1", "zipf"
    seed: int = 0

    @property
    def P(self) -> int:
        return self.T * self.k

    def replace(self, **kw) -> "MoEConfig":
        return dataclasses.replace(self, **kw)

    def as_dict(self) -> dict:
        return dataclasses.asdict(self)


CONFIGS: Dict[str, MoEConfig] = {
    "tiny_fp32": MoEConfig("tiny_fp32", 256, 256, 8, 2, 512, 0, "f32", "softmax", "none", True, "none"),
    "qwen3_30b_a3b": MoEConfig("qwen3_30b_a3b", 4096, 2048, 128, 8, 768, 0, "bf16", "softmax", "none", True, "none"),
    "deepseek_v2_lite_zipf": MoEConfig(
        "deepseek_v2_lite_zipf", 8192, 2048, 64, 6, 1408, 2816, "bf16", "softmax", "logit", False, "plain",
        bias_kind="zipf"),
    "dsv4_flash_ablation": MoEConfig(
        "dsv4_flash_ablation", 8192, 4096, 64, 6, 2048, 2048, "bf16", "sqrtsoftplus", "select", True, "plain",
        bias_kind="uniform0.1"),
    "decode_weight_streaming": MoEConfig(
        "decode_weight_streaming", 16, 7168, 256, 8, 2048, 2048, "bf16", "sigmoid", "none", True, "sigmoid_gated"),
}

# Order of the named problems (the tiny one first).
CONFIG_ORDER = ["tiny_fp32", "qwen3_30b_a3b", "deepseek_v2_lite_zipf", "dsv4_flash_ablation",
                "decode_weight_streaming"]

# Tensor ids used to derive per-tensor seeds.
_TID = {"x": 1, "gate_w": 2, "bias": 3, "gate_up": 4, "down": 5, "shared_gate_up": 6, "shared_down": 7,
        "shared_gate": 8}


def _torch_dtype(cfg: MoEConfig) -> torch.dtype:
    return torch.float32 if cfg.dtype == "f32" else torch.bfloat16


def _gen(cfg: MoEConfig, name: str, device: str) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(cfg.seed * 1000 + _TID[name])
    return g


def _normal(shape, std: float, gen: torch.Generator, device: str, dtype: torch.dtype) -> torch.Tensor:
    a = torch.randn(*shape, generator=gen, device=device, dtype=torch.float32)
    a.mul_(std)
    return a.to(dtype)


def _stacked_normal(E: int, shape, std: float, gen: torch.Generator, device: str,
                    dtype: torch.dtype) -> torch.Tensor:
    """[E, *shape] drawn one expert slab at a time, bounding fp32 scratch."""
    out = torch.empty((E,) + tuple(shape), device=device, dtype=dtype)
    for e in range(E):
        out[e].copy_(_normal(shape, std, gen, device, dtype))
    return out


def load_zipf_bias(E: int) -> torch.Tensor:
    with open(ZIPF_BIAS_FILE) as f:
        d = json.load(f)
    if int(d["E"]) != E:
        raise ValueError(f"stored Zipf bias is for E={d['E']}, asked for E={E}")
    return torch.tensor(d["bias_fp32"], dtype=torch.float32)


def router_inputs(cfg: MoEConfig, rank: int = 0) -> Dict[str, Optional[torch.Tensor]]:
    """x, gate_w, bias and shared gate vector, always drawn on the CPU.

    ``rank`` selects an independent batch of hidden states (data-parallel
    replicas share every weight); rank 0 is the problem's own batch."""
    dt = _torch_dtype(cfg)
    out: Dict[str, Optional[torch.Tensor]] = {}
    gx = _gen(cfg, "x", "cpu")
    if rank:
        gx.manual_seed(cfg.seed * 1000 + _TID["x"] + 100003 * rank)
    out["x"] = _normal((cfg.T, cfg.H), 1.0, gx, "cpu", dt)
    out["gate_w"] = _normal((cfg.E, cfg.H), cfg.H ** -0.5, _gen(cfg, "gate_w", "cpu"), "cpu", dt)
    if cfg.bias_kind == "none":
        out["bias"] = None
    elif cfg.bias_kind == "uniform0.1":
        g = _gen(cfg, "bias", "cpu")
        out["bias"] = (torch.rand(cfg.E, generator=g, dtype=torch.float32) * 0.2 - 0.1).contiguous()
    elif cfg.bias_kind == "zipf":
        out["bias"] = load_zipf_bias(cfg.E)
    else:
        raise ValueError(cfg.bias_kind)
    if cfg.shared == "sigmoid_gated":
        out["shared_gate"] = _normal((cfg.H,), cfg.H ** -0.5, _gen(cfg, "shared_gate", "cpu"), "cpu", dt)
    else:
        out["shared_gate"] = None
    return out


def expert_weights(cfg: MoEConfig, device: str = "cpu") -> Dict[str, Optional[torch.Tensor]]:
    """Stacked routed weights and the shared expert, drawn on ``device``."""
    dt = _torch_dtype(cfg)
    out: Dict[str, Optional[torch.Tensor]] = {}
    out["gate_up"] = _stacked_normal(cfg.E, (2 * cfg.I, cfg.H), cfg.H ** -0.5, _gen(cfg, "gate_up", device),
                                     device, dt)
    out["down"] = _stacked_normal(cfg.E, (cfg.H, cfg.I), cfg.I ** -0.5, _gen(cfg, "down", device), device, dt)
    if cfg.shared != "none":
        out["shared_gate_up"] = _normal((2 * cfg.I_shared, cfg.H), cfg.H ** -0.5,
                                        _gen(cfg, "shared_gate_up", device), device, dt)
        out["shared_down"] = _normal((cfg.H, cfg.I_shared), cfg.I_shared ** -0.5,
                                     _gen(cfg, "shared_down", device), device, dt)
    else:
        out["shared_gate_up"] = None
        out["shared_down"] = None
    return out


def generate(cfg: MoEConfig, device: str = "cpu") -> Dict[str, Optional[torch.Tensor]]:
    """All inputs of one problem. Router-side tensors are moved to ``device``."""
    r = router_inputs(cfg)
    w = expert_weights(cfg, device)
    out = {k: (v.to(device) if v is not None else None) for k, v in r.items()}
    out.update(w)
    return out


def reduced(cfg: MoEConfig, T: int, H: Optional[int] = None, I: Optional[int] = None,
            I_shared: Optional[int] = None, name_suffix: str = "_small") -> MoEConfig:
    """Same routing structure (E, k, score, bias, shared kind) at smaller sizes."""
    return cfg.replace(name=cfg.name + name_suffix, T=T, H=H or cfg.H, I=I or cfg.I,
                       I_shared=(I_shared if I_shared is not None else cfg.I_shared) if cfg.shared != "none" else 0)


def to_numpy64(t: Optional[torch.Tensor]):
    """Exact conversion of a (possibly bf16, possibly CUDA) tensor to an fp64 numpy array."""
    if t is None:
        return None
    return t.detach().to("cpu", torch.float64).numpy()
