"""Expert parallelism: the routed experts split over the ranks of a process
group, token rows exchanged with all-to-all.

The pages describe the experts of one MoE layer as segments of one fused
weight ("mstar.model.components.moe", SparseMoeBlock fused gate_up/down
layout) and load statistics all-reduced over data-parallel ranks ("Sparse MoE
FFN for DFlash-family drafters", What's here, MoEGate); they give no
expert-parallel layout. The plainest one that keeps every rank's arithmetic
identical to the one-GPU forward is taken here:

* rank r of G holds routed experts [r E/G, (r+1) E/G) (E divisible by G),
  the router and the shared expert replicated;
* each rank routes and dispatches its own T tokens over all E experts with
  the library's kernels; because the dispatch sorts rows by expert, the rows
  bound for each rank form one contiguous run of x_perm, in rank order;
* the per-expert counts go to their owners (all-to-all of E/G counts per
  peer; one device-to-host read of the counts sizes the row exchange), then
  the rows and their routing weights (all-to-all with those split sizes);
* the receiver's rows arrive grouped by source rank, each source's rows
  sorted by expert. A k = 1 dispatch keyed by the local expert id regroups
  them into one segment per local expert (stable, so arrival order is kept
  inside a segment), the grouped SwiGLU scales each row by its weight, and a
  k = 1 fp32 combine puts the rows back in arrival order;
* the reverse all-to-all returns every row to its sender, in the sender's
  x_perm order: exactly the y_perm of the one-GPU forward (fp32 rows), so
  the shared expert and the combine on the sender finish the layer as there.

Every per-row result is the same arithmetic as on one GPU; only where a row
sits in a GEMM tile changes. The collectives are torch.distributed
all_to_all_single calls (NCCL over NVLink on GPUs). This module holds the
host orchestration only: every step of the layer's arithmetic runs in the
library's CUDA kernels.
"""

from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np
import torch

from . import Problem, combine, dispatch, grouped_swiglu, new_workspace, route, shared_expert, workspace_size


def send_splits(counts: Sequence[int], world: int) -> List[int]:
    """Rows this rank sends to each rank: the counts of that rank's experts,
    summed (experts split into ``world`` equal contiguous groups)."""
    c = np.asarray(counts, dtype=np.int64)
    if c.size % world:
        raise ValueError(f"{c.size} experts do not split over {world} ranks")
    return [int(v) for v in c.reshape(world, -1).sum(axis=1)]


def receive_layout(recv_counts: np.ndarray) -> Tuple[List[int], np.ndarray]:
    """From the counts received [G, E/G] (row s: source rank s's rows per
    local expert), the rows received from each source and the local expert
    id of every received row in arrival order (source-major, then expert)."""
    rc = np.asarray(recv_counts, dtype=np.int64)
    splits = [int(v) for v in rc.sum(axis=1)]
    local = np.arange(rc.shape[1], dtype=np.int64)
    ids = np.concatenate([np.repeat(local, row) for row in rc]) if rc.size else np.zeros(0, np.int64)
    return splits, ids.astype(np.int64)


class WorkspacePool:
    """Library workspaces kept across calls: one per problem kind (the
    problem with T set aside), replaced by a larger one only when a call
    needs more bytes than the kept one has."""

    def __init__(self, device):
        self.device = device
        self._kept: Dict[Problem, Tuple[int, torch.Tensor]] = {}

    def get(self, p: Problem) -> torch.Tensor:
        key = dataclasses.replace(p, T=0)
        need = workspace_size(p)
        kept = self._kept.get(key)
        if kept is None or kept[0] < need:
            kept = (need, new_workspace(p, self.device))
            self._kept[key] = kept
        return kept[1]


class ExpertParallelMoE:
    """One MoE layer with its routed experts split over ``group``.

    ``p``: the whole layer's problem (global E; T = this rank's tokens).
    ``weights``: gate_w [E,H] (replicated), optional bias [E] fp32, gate_up
    [E/G, 2I, H] and down [E/G, H, I] (this rank's experts), and the
    replicated shared expert weights when ``p.shared`` is not "none".
    """

    def __init__(self, p: Problem, weights: Dict[str, Optional[torch.Tensor]], group=None):
        import torch.distributed as dist

        self.p = p
        self.w = weights
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if p.E % self.world:
            raise ValueError(f"E={p.E} is not divisible by the {self.world} ranks")
        self.E_local = p.E // self.world
        gu, dn = weights["gate_up"], weights["down"]
        if tuple(gu.shape) != (self.E_local, 2 * p.I, p.H) or tuple(dn.shape) != (self.E_local, p.H, p.I):
            raise ValueError(f"local expert weights must be [{self.E_local}, 2I, H] and [{self.E_local}, H, I]")
        self.pool = WorkspacePool(gu.device)

    def _a2a(self, out: torch.Tensor, inp: torch.Tensor, out_splits, in_splits) -> None:
        import torch.distributed as dist

        dist.all_to_all_single(out, inp, out_splits, in_splits, group=self.group)

    def forward(self, x: torch.Tensor):
        """out [T,H], routing_weights [T,k] fp32, selected_experts [T,k] int64."""
        p, w = self.p, self.w
        dev = x.device
        gate = w.get("shared_gate") if p.shared == "sigmoid_gated" else None
        ws = self.pool.get(p)
        rw, sel, gamma = route(p, x, w["gate_w"], w.get("bias"), gate, ws=ws)
        d = dispatch(p, sel, x, ws=ws)

        # counts to the experts' owners; one host read sizes the row exchange
        counts = d["counts"].to(torch.int64)
        recv_counts = torch.empty_like(counts)
        self._a2a(recv_counts, counts, None, None)
        sends = send_splits(counts.cpu().numpy(), self.world)
        recvs, local_ids = receive_layout(recv_counts.cpu().numpy().reshape(self.world, self.E_local))
        n_send, n_recv = sum(sends), sum(recvs)

        # rows (x_perm order) and their routing weights to the owners
        x_recv = torch.empty(n_recv, p.H, dtype=x.dtype, device=dev)
        self._a2a(x_recv, d["x_perm"][:n_send], recvs, sends)
        w_sorted = rw.reshape(-1)[d["sorted_pairs"][:n_send].long()]
        w_recv = torch.empty(n_recv, dtype=torch.float32, device=dev)
        self._a2a(w_recv, w_sorted, recvs, sends)

        y_recv = self._local_experts(x_recv, w_recv, local_ids)

        # weighted fp32 rows back to their senders, in x_perm order
        y_perm = torch.zeros(p.T * p.k, p.H, dtype=torch.float32, device=dev)
        self._a2a(y_perm[:n_send], y_recv, sends, recvs)
        shared = None
        if p.shared != "none":
            shared = shared_expert(p, x, w["shared_gate_up"], w["shared_down"], gamma, ws=ws)
        return combine(p, y_perm, d["pair_pos"], shared), rw, sel

    __call__ = forward

    def _local_experts(self, x_recv: torch.Tensor, w_recv: torch.Tensor, local_ids: np.ndarray) -> torch.Tensor:
        """The received rows through this rank's experts, weighted, fp32 [n, H]
        in arrival order."""
        p = self.p
        n = x_recv.shape[0]
        if n == 0:
            return torch.zeros(0, p.H, dtype=torch.float32, device=x_recv.device)
        pr = dataclasses.replace(p, T=n, E=self.E_local, k=1, I_shared=0, bias_mode="none", shared="none")
        ids = torch.from_numpy(local_ids).to(x_recv.device).view(n, 1)
        ws = self.pool.get(pr)
        d = dispatch(pr, ids, x_recv, ws=ws)
        y = grouped_swiglu(pr, d["x_perm"], d["offsets"], self.w["gate_up"], self.w["down"], w_recv.view(n, 1),
                           d["sorted_pairs"], ws=ws)
        return combine(dataclasses.replace(pr, dtype="f32"), y, d["pair_pos"], None)
