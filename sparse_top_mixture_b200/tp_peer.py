"""Tensor parallelism with the reduction on peer memory, fused with the combine.

Same layer and sharding as ``tensor_parallel.TensorParallelMoE`` (every
expert's I, and the shared expert's, split over the ranks; router
replicated; every rank given the same tokens), but instead of a combine, an
NCCL all-reduce and a rounding pass, one library kernel (``moe_tp_scatter``)
combines each token's partial rows and stores every column slice into its
owner's arena, and the owner (``moe_tp_gather``) adds the G slices in rank
order, rounds once, and stores its columns into every rank's output. Epoch
flags with bounded waits (``moe_tp_wait``) order the two, nothing is read on
the host, and the sum over ranks has a fixed order.

``open`` maps the peers' arenas through CUDA IPC on a node; ``emulate``
builds G ranks in one process on one GPU for tests, which run each phase
(``partial``, ``reduce``, ``finish``) for every rank in turn on one stream.
"""

from __future__ import annotations

import ctypes
import dataclasses
from typing import Dict, List, Optional, Sequence

import torch

from . import Problem, _check, _stream, dispatch, grouped_swiglu, lib, new_workspace, route, shared_expert
from .tensor_parallel import shard_expert_weights

DEFAULT_MAX_POLLS = 1 << 24


def tp_arena_size(p: Problem, world: int) -> int:
    n = ctypes.c_size_t()
    _check(lib().moe_tp_arena_size(ctypes.byref(p.c()), world, ctypes.byref(n)))
    return n.value


def tp_arena_offsets(p: Problem, world: int) -> Dict[str, int]:
    v = [ctypes.c_size_t() for _ in range(5)]
    _check(lib().moe_tp_arena_offsets(ctypes.byref(p.c()), world, *[ctypes.byref(x) for x in v]))
    return dict(zip(("part_flag", "out_flag", "epoch", "part", "out"), (x.value for x in v)))


class PeerTensorParallelMoE:
    """One MoE layer with every expert's I split over `world` ranks and the
    partial outputs reduced over peer memory.

    ``p``: the whole layer's problem (full I, I_shared). ``weights``: the
    router's and this rank's slice of the experts (``shard_expert_weights``).
    ``arena`` / ``arena_ptrs`` as for ``ep_peer.PeerExpertParallelMoE``.
    """

    def __init__(self, p: Problem, weights: Dict[str, Optional[torch.Tensor]], rank: int, world: int,
                 arena: torch.Tensor, arena_ptrs: Sequence[int], max_polls: int = DEFAULT_MAX_POLLS,
                 keep: Sequence[object] = ()):
        if p.I % world or (p.shared != "none" and p.I_shared % world):
            raise ValueError(f"I={p.I} / I_shared={p.I_shared} do not split over {world} ranks")
        self.p, self.w, self.rank, self.world = p, weights, rank, world
        self.local = dataclasses.replace(p, I=p.I // world, I_shared=p.I_shared // world if p.shared != "none" else 0)
        if arena.numel() < tp_arena_size(p, world) or arena.dtype != torch.uint8:
            raise ValueError("arena too small")
        if len(arena_ptrs) != world or arena_ptrs[rank] != arena.data_ptr():
            raise ValueError("arena_ptrs must hold the G arenas, this rank's at index rank")
        dev = arena.device
        self.arena = arena
        self.ptrs = torch.tensor(list(arena_ptrs), dtype=torch.int64, device=dev)
        self.max_polls = int(max_polls)
        self._keep = list(keep)
        off = tp_arena_offsets(p, world)
        es = p.torch_dtype.itemsize
        self.out = arena[off["out"]:off["out"] + p.T * p.H * es].view(p.torch_dtype).view(p.T, p.H)
        self.epoch = arena[off["epoch"]:off["epoch"] + 8].view(torch.int64)
        self.ws = new_workspace(p, dev)
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)
        self._st: Dict[str, object] = {}

    @classmethod
    def open(cls, p: Problem, weights, group=None, max_polls: int = DEFAULT_MAX_POLLS) -> "PeerTensorParallelMoE":
        """Collective over ``group`` (one process per GPU of one node)."""
        import torch.distributed as dist

        world, rank = dist.get_world_size(group), dist.get_rank(group)
        dev = weights["gate_up"].device
        arena = torch.zeros(tp_arena_size(p, world), dtype=torch.uint8, device=dev)
        handle = arena.untyped_storage()._share_cuda_()
        handles: List[object] = [None] * world
        dist.all_gather_object(handles, handle, group=group)
        ptrs, keep = [], []
        for s, h in enumerate(handles):
            if s == rank:
                ptrs.append(arena.data_ptr())
                continue
            st = torch.UntypedStorage._new_shared_cuda(*h)
            keep.append(st)
            ptrs.append(st.data_ptr())
        torch.cuda.synchronize(dev)
        dist.barrier(group=group)
        return cls(p, weights, rank, world, arena, ptrs, max_polls, keep)

    @classmethod
    def emulate(cls, p: Problem, weights: Dict[str, Optional[torch.Tensor]], world: int
                ) -> List["PeerTensorParallelMoE"]:
        """G ranks in this process on one GPU (tests), full-model weights
        sharded along I; each wait polls once."""
        dev = weights["gate_up"].device
        arenas = [torch.zeros(tp_arena_size(p, world), dtype=torch.uint8, device=dev) for _ in range(world)]
        ptrs = [a.data_ptr() for a in arenas]
        return [cls(p, shard_expert_weights(weights, r, world), r, world, arenas[r], ptrs, max_polls=1, keep=arenas)
                for r in range(world)]

    # -- phases ---------------------------------------------------------------
    def partial(self, x: torch.Tensor) -> None:
        """Route, dispatch, this rank's slice of the experts, and the fused
        combine + scatter of its partial output."""
        p, pl, w, ws = self.p, self.local, self.w, self.ws
        gate = w.get("shared_gate") if p.shared == "sigmoid_gated" else None
        rw, sel, gamma = route(p, x, w["gate_w"], w.get("bias"), gate, ws=ws)
        d = dispatch(p, sel, x, ws=ws)
        y = grouped_swiglu(pl, d["x_perm"], d["offsets"], w["gate_up"], w["down"], rw, d["sorted_pairs"], ws=ws)
        shared = None
        if p.shared != "none":
            shared = shared_expert(pl, x, w["shared_gate_up"], w["shared_down"], gamma, ws=ws)
        _check(lib().moe_tp_scatter(ctypes.byref(p.c()), self.world, self.rank, self.ptrs.data_ptr(),
                                    self.arena.data_ptr(), y.data_ptr(), d["pair_pos"].data_ptr(),
                                    shared.data_ptr() if shared is not None else None, _stream(x.device)))
        self._st = {"rw": rw, "sel": sel, "keep": (d, y, shared)}

    def reduce(self) -> None:
        self._wait(0)
        _check(lib().moe_tp_gather(ctypes.byref(self.p.c()), self.world, self.rank, self.ptrs.data_ptr(),
                                   self.arena.data_ptr(), _stream(self.arena.device)))

    def finish(self):
        """out [T,H] (a copy: the arena's output is rewritten by the next
        forward), routing_weights [T,k] fp32, selected_experts [T,k] int64."""
        self._wait(1)
        return self.out.clone(), self._st["rw"], self._st["sel"]

    def forward(self, x: torch.Tensor):
        self.partial(x)
        self.reduce()
        return self.finish()

    __call__ = forward

    def _wait(self, which: int) -> None:
        _check(lib().moe_tp_wait(ctypes.byref(self.p.c()), self.world, self.arena.data_ptr(), which, self.max_polls,
                                 self.err.data_ptr(), _stream(self.arena.device)))
