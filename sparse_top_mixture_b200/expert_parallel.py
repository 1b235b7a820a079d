"""Expert parallelism: the routed experts split over the ranks of a process
group, token rows exchanged between the ranks.

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
* the per-expert counts go to their owners (an all-to-all of E/G counts per
  peer). Everything that needs no remote count -- this rank's own run of
  x_perm through its own experts (the grouped SwiGLU over the local experts'
  segments of the one-GPU segment table, writing those rows of y_perm in
  place) and the shared expert -- is enqueued first, on a second stream that
  starts after the dispatch: the host read below waits only for the dispatch
  and the count exchange, and the row exchanges overlap the local GEMMs;
* one device-to-host read of the counts then sizes the remote exchange:
  point-to-point sends and receives, one group per exchange (rows, their
  routing weights and their local expert ids to each other rank; the
  weighted fp32 rows back);
* a receiver's remote rows arrive grouped by source rank, each source's rows
  sorted by expert, each with its local expert id. A k = 1 dispatch keyed by
  that id regroups them into one segment per local expert (stable, so
  arrival order is kept inside a segment), the grouped SwiGLU scales each row
  by its weight, and a k = 1 fp32 combine puts the rows back in arrival
  order;
* the rows come back to their senders in the sender's x_perm order: with the
  local rows, exactly the y_perm of the one-GPU forward (fp32 rows), so the
  combine finishes the layer as there, once the second stream has joined.

Every per-row result is the same arithmetic as on one GPU; only where a row
sits in a GEMM tile changes. The collectives are torch.distributed calls
(NCCL over NVLink on GPUs). This module holds the host orchestration only:
every step of the layer's arithmetic runs in the library's CUDA kernels.
"""

from __future__ import annotations

import contextlib
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


def local_expert_ids(global_ids: torch.Tensor, owner: int, experts_per_rank: int) -> torch.Tensor:
    """The owner's local expert id of each row sent to it (int64)."""
    return global_ids - owner * experts_per_rank


@dataclasses.dataclass
class ExchangePlan:
    """Where each peer's rows sit: send_off[s] .. send_off[s+1] in this rank's
    x_perm (and y_perm) go to rank s; recv_off[s] .. recv_off[s] + recvs[s] of
    the receive buffers come from rank s (remote peers only, in rank order)."""
    send_off: List[int]
    recvs: List[int]
    recv_off: Dict[int, int]
    remote: List[int]
    n_recv: int


def exchange_plan(counts: Sequence[int], recv_counts: np.ndarray, rank: int) -> ExchangePlan:
    """From this rank's per-expert counts [E] and the counts its peers send it
    [G, E/G] (row s: rank s's rows per local expert)."""
    rc = np.asarray(recv_counts, dtype=np.int64)
    G = rc.shape[0]
    sends = send_splits(counts, G)
    send_off = [0]
    for v in sends:
        send_off.append(send_off[-1] + v)
    recvs = [int(v) for v in rc.sum(axis=1)]
    remote = [s for s in range(G) if s != rank]
    recv_off, acc = {}, 0
    for s in remote:
        recv_off[s] = acc
        acc += recvs[s]
    return ExchangePlan(send_off, recvs, recv_off, remote, acc)


class WorkspacePool:
    """Library workspaces kept across calls: one per problem kind (the
    problem with T set aside) and user (`slot`: work that may run at the same
    time on two streams takes two slots), replaced by a larger one only when
    a call needs more bytes than the kept one has."""

    def __init__(self, device):
        self.device = device
        self._kept: Dict[Tuple[Problem, str], Tuple[int, torch.Tensor]] = {}

    def get(self, p: Problem, slot: str = "") -> torch.Tensor:
        key = (dataclasses.replace(p, T=0), slot)
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
        self.side = torch.cuda.Stream(gu.device) if gu.is_cuda else None  # the local GEMMs' stream

    def _a2a(self, out: torch.Tensor, inp: torch.Tensor, out_splits, in_splits) -> None:
        import torch.distributed as dist

        dist.all_to_all_single(out, inp, out_splits, in_splits, group=self.group)

    def _exchange(self, sends, recvs) -> None:
        """One group of point-to-point transfers: ``sends`` and ``recvs`` are
        lists of (peer, tensor); nothing is sent to or received from this
        rank itself."""
        import torch.distributed as dist

        ops = [dist.P2POp(dist.isend, t, dist.get_global_rank(self.group, peer) if self.group else peer, self.group)
               for peer, t in sends if t.numel()]
        ops += [dist.P2POp(dist.irecv, t, dist.get_global_rank(self.group, peer) if self.group else peer, self.group)
                for peer, t in recvs if t.numel()]
        if ops:
            for req in dist.batch_isend_irecv(ops):
                req.wait()

    def _host_counts(self, counts: torch.Tensor, recv_counts: torch.Tensor):
        """The one device-to-host read of the layer: this rank's counts and the
        counts its peers send it (synchronises the stream)."""
        self.trace.append("host_counts")
        return counts.cpu().numpy(), recv_counts.cpu().numpy().reshape(self.world, self.E_local)

    def forward(self, x: torch.Tensor):
        """out [T,H], routing_weights [T,k] fp32, selected_experts [T,k] int64."""
        p, w = self.p, self.w
        r, G, El = self.rank, self.world, self.E_local
        dev = x.device
        self.trace = []
        gate = w.get("shared_gate") if p.shared == "sigmoid_gated" else None
        ws = self.pool.get(p)
        rw, sel, gamma = route(p, x, w["gate_w"], w.get("bias"), gate, ws=ws)
        d = dispatch(p, sel, x, ws=ws)

        # Work that needs no remote count, on the second stream from the end of
        # the dispatch on: this rank's own rows through its own experts (rows
        # of y_perm in place; as a problem of T*k one-slot rows over the E/G
        # local experts: the same x_perm rows, routing weights and sorted pair
        # indices) and the shared expert.
        if self.side is not None:
            main = torch.cuda.current_stream(dev)
            self.side.wait_stream(main)
        side_ctx = torch.cuda.stream(self.side) if self.side is not None else contextlib.nullcontext()
        pl = dataclasses.replace(p, T=p.T * p.k, k=1, E=El, I_shared=0, shared="none", bias_mode="none")
        own_offsets = d["offsets"][r * El:(r + 1) * El + 1]
        shared = None
        with side_ctx:
            y_perm = grouped_swiglu(pl, d["x_perm"], own_offsets, w["gate_up"], w["down"], rw.view(-1, 1),
                                    d["sorted_pairs"], ws=self.pool.get(pl, "local"))
            self.trace.append("local_experts")
            if self.side is not None:  # marks the local GEMM's place on the second stream (tests check it)
                self.local_done = torch.cuda.Event()
                self.local_done.record(self.side)
            if p.shared != "none":
                shared = shared_expert(p, x, w["shared_gate_up"], w["shared_down"], gamma, ws=ws)
                self.trace.append("shared_expert")

        # counts to the experts' owners
        counts = d["counts"].to(torch.int64)
        recv_counts = torch.empty_like(counts)
        self._a2a(recv_counts, counts, None, None)

        # the host read sizes the remote exchange
        plan = exchange_plan(*self._host_counts(counts, recv_counts), r)
        send_off, recvs, recv_off, remote, n_recv = plan.send_off, plan.recvs, plan.recv_off, plan.remote, plan.n_recv

        # rows (x_perm order), their routing weights and local expert ids to the owners
        q_sorted = d["sorted_pairs"][:send_off[-1]].long()
        w_sorted = rw.reshape(-1)[q_sorted]
        e_sorted = sel.reshape(-1)[q_sorted]
        x_recv = torch.empty(n_recv, p.H, dtype=x.dtype, device=dev)
        w_recv = torch.empty(n_recv, dtype=torch.float32, device=dev)
        id_recv = torch.empty(n_recv, dtype=torch.int64, device=dev)
        out_rows, out_w, out_id, in_rows, in_w, in_id = [], [], [], [], [], []
        for s in remote:
            a, b = send_off[s], send_off[s + 1]
            out_rows.append((s, d["x_perm"][a:b]))
            out_w.append((s, w_sorted[a:b].contiguous()))
            out_id.append((s, local_expert_ids(e_sorted[a:b], s, El).contiguous()))
            c, n = recv_off[s], recvs[s]
            in_rows.append((s, x_recv[c:c + n]))
            in_w.append((s, w_recv[c:c + n]))
            in_id.append((s, id_recv[c:c + n]))
        self._exchange(out_rows + out_w + out_id, in_rows + in_w + in_id)

        y_recv = self._local_experts(x_recv, w_recv, id_recv)

        # weighted fp32 rows back to their senders, into y_perm in x_perm order
        self._exchange([(s, y_recv[recv_off[s]:recv_off[s] + recvs[s]]) for s in remote],
                       [(s, y_perm[send_off[s]:send_off[s + 1]]) for s in remote])
        if self.side is not None:  # join: the local rows and the shared expert are done
            main.wait_stream(self.side)
            y_perm.record_stream(main)
            if shared is not None:
                shared.record_stream(main)
        return combine(p, y_perm, d["pair_pos"], shared), rw, sel

    __call__ = forward

    def _local_experts(self, x_recv: torch.Tensor, w_recv: torch.Tensor, id_recv: torch.Tensor) -> torch.Tensor:
        """The received rows through this rank's experts, weighted, fp32 [n, H]
        in arrival order."""
        p = self.p
        n = x_recv.shape[0]
        if n == 0:
            return torch.zeros(0, p.H, dtype=torch.float32, device=x_recv.device)
        pr = dataclasses.replace(p, T=n, E=self.E_local, k=1, I_shared=0, bias_mode="none", shared="none")
        ws = self.pool.get(pr, "remote")
        d = dispatch(pr, id_recv.view(n, 1), x_recv, ws=ws)
        y = grouped_swiglu(pr, d["x_perm"], d["offsets"], self.w["gate_up"], self.w["down"], w_recv.view(n, 1),
                           d["sorted_pairs"], ws=ws)
        return combine(dataclasses.replace(pr, dtype="f32"), y, d["pair_pos"], None)
