"""Tensor parallelism: every expert's intermediate dimension split over the
ranks of a process group, partial outputs summed across ranks.

"mstar.model.components.moe" (the tensor-parallel MoE block) shards the
experts along I and all-reduces the partial results between the down
projection and the top-k sum. The SwiGLU is elementwise in I and the down
projection sums over I, so each rank's slice of I yields a partial y_perm
whose sum over ranks is the whole one; the routing weights, the top-k sum and
the shared expert's gate are linear in y, so the sum can equally be taken
after the combine. It is taken there: the all-reduce then moves T x H fp32
values instead of T k x H. Readings taken where the page is silent:

* rank r of G holds gate rows [r I/G, (r+1) I/G) and the matching up rows
  of every expert's gate_up, the same columns of its down, and likewise for
  the shared expert (I/G and I_shared/G multiples of 8);
* the router is replicated: every rank routes the same tokens identically;
* each rank's partial output is its fp32 combine (weighted rows plus its
  shared-expert slice); the fp32 sum over ranks is rounded once to the
  problem dtype, by a one-slot combine.

The collective is a torch.distributed all_reduce (NCCL over NVLink on GPUs).
Every step of the layer's arithmetic runs in the library's CUDA kernels.
"""

from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import torch

from . import Problem, combine, dispatch, grouped_swiglu, new_workspace, route, shared_expert


def shard_expert_weights(weights: Dict[str, Optional[torch.Tensor]], rank: int, world: int
                         ) -> Dict[str, Optional[torch.Tensor]]:
    """This rank's slice of I of the routed and shared expert weights (new
    contiguous tensors); the router's weights are returned unchanged."""
    out = dict(weights)

    def rows(gu: torch.Tensor) -> torch.Tensor:  # [..., 2I, H]: gate rows, then up rows
        I = gu.shape[-2] // 2
        if I % world:
            raise ValueError(f"I={I} does not split over {world} ranks")
        s = I // world
        return torch.cat([gu[..., rank * s:(rank + 1) * s, :], gu[..., I + rank * s:I + (rank + 1) * s, :]],
                         dim=-2).contiguous()

    def cols(dn: torch.Tensor) -> torch.Tensor:  # [..., H, I]
        s = dn.shape[-1] // world
        return dn[..., rank * s:(rank + 1) * s].contiguous()

    out["gate_up"], out["down"] = rows(weights["gate_up"]), cols(weights["down"])
    if weights.get("shared_gate_up") is not None:
        out["shared_gate_up"], out["shared_down"] = rows(weights["shared_gate_up"]), cols(weights["shared_down"])
    return out


class TensorParallelMoE:
    """One MoE layer with every expert's I split over ``group``.

    ``p``: the whole layer's problem (full I and I_shared). ``weights``: the
    router's (replicated) and this rank's slice of the experts, as
    ``shard_expert_weights`` returns them. Every rank passes the same x."""

    def __init__(self, p: Problem, weights: Dict[str, Optional[torch.Tensor]], group=None):
        import torch.distributed as dist

        self.p = p
        self.w = weights
        self.group = group
        self.world = dist.get_world_size(group)
        if p.I % self.world or (p.shared != "none" and p.I_shared % self.world):
            raise ValueError(f"I={p.I} / I_shared={p.I_shared} do not split over {self.world} ranks")
        self.local = dataclasses.replace(p, I=p.I // self.world,
                                         I_shared=p.I_shared // self.world if p.shared != "none" else 0)
        self.ws = new_workspace(p, weights["gate_up"].device)  # the full problem's: the largest of the calls

    def forward(self, x: torch.Tensor):
        """out [T,H] (problem dtype), routing_weights [T,k] fp32, selected_experts [T,k] int64."""
        import torch.distributed as dist

        p, pl, w = self.p, self.local, self.w
        gate = w.get("shared_gate") if p.shared == "sigmoid_gated" else None
        ws = self.ws
        rw, sel, gamma = route(p, x, w["gate_w"], w.get("bias"), gate, ws=ws)
        d = dispatch(p, sel, x, ws=ws)
        y = grouped_swiglu(pl, d["x_perm"], d["offsets"], w["gate_up"], w["down"], rw, d["sorted_pairs"], ws=ws)
        shared = None
        if p.shared != "none":
            shared = shared_expert(pl, x, w["shared_gate_up"], w["shared_down"], gamma, ws=ws)
        part = combine(dataclasses.replace(pl, dtype="f32"), y, d["pair_pos"], shared)  # fp32 [T, H]
        dist.all_reduce(part, group=self.group)
        # round the fp32 sum once: a one-slot combine of the rows in order
        one = dataclasses.replace(p, k=1, I_shared=0, shared="none")
        ident = torch.arange(p.T, dtype=torch.int32, device=x.device)
        return combine(one, part, ident, None), rw, sel

    __call__ = forward
