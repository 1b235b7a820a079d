"""Expert parallelism with the row exchange on peer memory: no host read.

Same layer and layout as ``expert_parallel.ExpertParallelMoE`` (rank r of G
holds routed experts [r E/G, (r+1) E/G); router and shared expert
replicated), but the rows move by the library's peer-store kernels
(``moe_ep_send`` / ``moe_ep_return``) into arenas every rank can address,
ordered by epoch flags (``moe_ep_wait``; each arena keeps its rank's epoch,
advanced on the device), so that nothing is read on the host and the whole
forward is asynchronous and can be captured in a CUDA graph.
The per-row arithmetic is the one-GPU forward's: each rank's output equals
``SparseMoE`` on its tokens with all experts.

A forward is three phases, which ``forward`` runs back to back:

* ``send``: route this rank's tokens, then dispatch them over all E experts
  with the rows stored straight into their owners' arenas by the dispatch's
  own ranking kernel (``moe_ep_dispatch_send``: one launch instead of a
  permutation into x_perm and a copy out of it; ``fused=False`` takes the two
  steps, ``moe_dispatch`` then ``moe_ep_send``); the shared expert runs on a
  second stream meanwhile;
* ``experts``: wait for every source's rows, regroup the received slots by
  local expert, run the grouped SwiGLU, and store each weighted fp32 row back
  into its source's arena at its sorted position -- in bf16 one call
  (``moe_ep_experts``) whose down GEMM epilogue does the stores; otherwise
  (fp32, or ``fused=False``) ``moe_dispatch_slots``, ``moe_grouped_swiglu``
  and ``moe_ep_return``;
* ``finish``: wait for every owner's returns, then combine.

On a node, ``open`` allocates this rank's arena and maps the peers' through
CUDA IPC (storage handles exchanged once over the process group). ``emulate``
builds G ranks inside one process on one GPU, their arenas ordinary device
memory; a test then runs each phase for every rank in turn on one stream, so
that every wait finds its flags already published and no kernel waits for one
that has not run (its waits poll once).
"""

from __future__ import annotations

import ctypes
import dataclasses
from typing import Dict, List, Optional, Sequence

import torch

from . import (Problem, _check, _ptr, _stream, combine, dispatch, dispatch_slots, grouped_swiglu, lib,
               new_workspace, route, shared_expert)

# polls of a flag before a wait gives up (about 256 ns apart: ~4 s)
DEFAULT_MAX_POLLS = 1 << 24


def ep_arena_size(p: Problem, world: int) -> int:
    n = ctypes.c_size_t()
    _check(lib().moe_ep_arena_size(ctypes.byref(p.c()), world, ctypes.byref(n)))
    return n.value


def ep_arena_offsets(p: Problem, world: int) -> Dict[str, int]:
    v = [ctypes.c_size_t() for _ in range(7)]
    _check(lib().moe_ep_arena_offsets(ctypes.byref(p.c()), world, *[ctypes.byref(x) for x in v]))
    return dict(zip(("rows_flag", "ret_flag", "epoch", "x", "w", "id", "y"), (x.value for x in v)))


class PeerExpertParallelMoE:
    """One MoE layer with its routed experts split over `world` ranks and the
    rows exchanged over peer memory.

    ``p``: the whole layer's problem (global E; T = this rank's tokens, the
    same on every rank). ``weights``: gate_w [E,H] (replicated), optional
    bias, gate_up [E/G, 2I, H] and down [E/G, H, I] (this rank's experts),
    the shared expert's when ``p.shared`` is not "none". ``arena``: this
    rank's arena (uint8 device tensor of ``ep_arena_size`` bytes, zeroed);
    ``arena_ptrs``: the G arenas' device addresses, this one at ``rank``.
    Use ``open`` or ``emulate`` rather than this constructor.
    """

    def __init__(self, p: Problem, weights: Dict[str, Optional[torch.Tensor]], rank: int, world: int,
                 arena: torch.Tensor, arena_ptrs: Sequence[int], max_polls: int = DEFAULT_MAX_POLLS,
                 keep: Sequence[object] = (), fused: bool = True):
        if p.E % world:
            raise ValueError(f"E={p.E} is not divisible by the {world} ranks")
        self.p, self.w, self.rank, self.world = p, weights, rank, world
        self.fused = fused
        self.E_local = p.E // world
        gu, dn = weights["gate_up"], weights["down"]
        if tuple(gu.shape) != (self.E_local, 2 * p.I, p.H) or tuple(dn.shape) != (self.E_local, p.H, p.I):
            raise ValueError(f"local expert weights must be [{self.E_local}, 2I, H] and [{self.E_local}, H, I]")
        if arena.numel() < ep_arena_size(p, world) or arena.dtype != torch.uint8:
            raise ValueError("arena too small")
        if len(arena_ptrs) != world or arena_ptrs[rank] != arena.data_ptr():
            raise ValueError("arena_ptrs must hold the G arenas, this rank's at index rank")
        self.arena = arena
        self.ptrs = torch.tensor(list(arena_ptrs), dtype=torch.int64, device=arena.device)
        self.max_polls = int(max_polls)
        self._keep = list(keep)  # peer mappings stay open as long as the layer
        dev = arena.device
        self.side = torch.cuda.Stream(dev)
        C = p.T * p.k
        off = ep_arena_offsets(p, world)
        G = world
        # views of this rank's arena
        self.recv_x = arena[off["x"]:off["x"] + G * C * p.H * p.torch_dtype.itemsize].view(p.torch_dtype).view(
            G * C, p.H)
        self.recv_w = arena[off["w"]:off["w"] + G * C * 4].view(torch.float32).view(G * C, 1)
        self.recv_id = arena[off["id"]:off["id"] + G * C * 8].view(torch.int64).view(G * C, 1)
        self.y = arena[off["y"]:off["y"] + C * p.H * 4].view(torch.float32).view(C, p.H)
        self.epoch = arena[off["epoch"]:off["epoch"] + 8].view(torch.int64)  # forwards so far (device)
        self.ws = new_workspace(p, dev)
        self.ws_shared = new_workspace(p, dev) if p.shared != "none" else None  # used on the second stream
        self.pk1 = dataclasses.replace(p, T=G * C, k=1, E=self.E_local, I_shared=0, shared="none", bias_mode="none")
        self.ws1 = new_workspace(self.pk1, dev)
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)  # a wait that gave up raises its bit here
        self._st: Dict[str, object] = {}

    # -- set-up ------------------------------------------------------------------
    @classmethod
    def open(cls, p: Problem, weights, group=None, max_polls: int = DEFAULT_MAX_POLLS) -> "PeerExpertParallelMoE":
        """Collective over ``group`` (one process per GPU of one node):
        allocates this rank's arena and maps every peer's (CUDA IPC)."""
        import torch.distributed as dist

        world, rank = dist.get_world_size(group), dist.get_rank(group)
        dev = weights["gate_up"].device
        arena = torch.zeros(ep_arena_size(p, world), dtype=torch.uint8, device=dev)
        handle = arena.untyped_storage()._share_cuda_()
        handles: List[object] = [None] * world
        dist.all_gather_object(handles, (handle, arena.data_ptr() - arena.untyped_storage().data_ptr()), group=group)
        ptrs, keep = [], []
        for s, (h, off) in enumerate(handles):
            if s == rank:
                ptrs.append(arena.data_ptr())
                continue
            st = torch.UntypedStorage._new_shared_cuda(*h)
            keep.append(st)
            ptrs.append(st.data_ptr() + off)
        torch.cuda.synchronize(dev)  # every arena zeroed before any peer stores into it
        dist.barrier(group=group)
        return cls(p, weights, rank, world, arena, ptrs, max_polls, keep)

    @classmethod
    def emulate(cls, p: Problem, weights: Dict[str, Optional[torch.Tensor]], world: int, fused: bool = True
                ) -> List["PeerExpertParallelMoE"]:
        """G ranks in this process on one GPU (tests): full-model ``weights``
        split by expert ranges; each wait polls once (run the phases rank by
        rank, in order, on one stream)."""
        El = p.E // world
        dev = weights["gate_up"].device
        arenas = [torch.zeros(ep_arena_size(p, world), dtype=torch.uint8, device=dev) for _ in range(world)]
        ptrs = [a.data_ptr() for a in arenas]
        layers = []
        for r in range(world):
            w = dict(weights)
            w["gate_up"] = weights["gate_up"][r * El:(r + 1) * El].contiguous()
            w["down"] = weights["down"][r * El:(r + 1) * El].contiguous()
            layers.append(cls(p, w, r, world, arenas[r], ptrs, max_polls=1, keep=arenas, fused=fused))
        return layers

    # -- the three phases ----------------------------------------------------------
    def send(self, x: torch.Tensor) -> None:
        p, w = self.p, self.w
        dev = x.device
        gate = w.get("shared_gate") if p.shared == "sigmoid_gated" else None
        rw, sel, gamma = route(p, x, w["gate_w"], w.get("bias"), gate, ws=self.ws)
        main = torch.cuda.current_stream(dev)
        shared = None
        if p.shared != "none":  # beside the exchange, on the second stream
            self.side.wait_stream(main)
            with torch.cuda.stream(self.side):
                shared = shared_expert(p, x, w["shared_gate_up"], w["shared_down"], gamma, ws=self.ws_shared)
        if self.fused and p.T > 0:
            P = p.T * p.k
            d = {"counts": torch.empty(p.E, dtype=torch.int32, device=dev),
                 "offsets": torch.empty(p.E + 1, dtype=torch.int32, device=dev),
                 "sorted_pairs": torch.empty(P, dtype=torch.int32, device=dev),
                 "pair_pos": torch.empty(P, dtype=torch.int32, device=dev)}
            _check(lib().moe_ep_dispatch_send(ctypes.byref(p.c()), self.world, self.rank, self.ptrs.data_ptr(),
                                              self.arena.data_ptr(), _ptr(sel), _ptr(x), _ptr(rw),
                                              _ptr(d["counts"]), _ptr(d["offsets"]), _ptr(d["sorted_pairs"]),
                                              _ptr(d["pair_pos"]), self.ws.data_ptr(), self.ws.numel(),
                                              _stream(dev)))
        else:
            d = dispatch(p, sel, x, ws=self.ws)
            _check(lib().moe_ep_send(ctypes.byref(p.c()), self.world, self.rank, self.ptrs.data_ptr(),
                                     self.arena.data_ptr(), _ptr(d["x_perm"]), _ptr(d["offsets"]),
                                     _ptr(d["sorted_pairs"]), _ptr(rw), _ptr(sel), _stream(dev)))
        self._st = {"rw": rw, "sel": sel, "pair_pos": d["pair_pos"], "shared": shared, "keep": d}

    def experts(self) -> None:
        p, dev = self.p, self.arena.device
        self._wait(0)
        if self.fused and p.dtype == "bf16":
            # regroup, GEMMs, and the down epilogue storing each row into its source's arena
            _check(lib().moe_ep_experts(ctypes.byref(p.c()), self.world, self.rank, self.ptrs.data_ptr(),
                                        self.arena.data_ptr(), self.w["gate_up"].data_ptr(),
                                        self.w["down"].data_ptr(), self.ws1.data_ptr(), self.ws1.numel(),
                                        _stream(dev)))
            return
        pk = self.pk1
        d1 = dispatch_slots(pk, self.recv_id, self.recv_x, ws=self.ws1)
        y_sorted = grouped_swiglu(pk, d1["x_perm"], d1["offsets"], self.w["gate_up"], self.w["down"], self.recv_w,
                                  d1["sorted_pairs"], ws=self.ws1)
        _check(lib().moe_ep_return(ctypes.byref(p.c()), self.world, self.rank, self.ptrs.data_ptr(),
                                   self.arena.data_ptr(), _ptr(y_sorted), _ptr(d1["offsets"]),
                                   _ptr(d1["sorted_pairs"]), _stream(dev)))
        self._st["keep1"] = (d1, y_sorted)

    def finish(self):
        """out [T,H], routing_weights [T,k] fp32, selected_experts [T,k] int64."""
        p, st = self.p, self._st
        self._wait(1)
        shared = st["shared"]
        if shared is not None:
            main = torch.cuda.current_stream(self.arena.device)
            main.wait_stream(self.side)
            shared.record_stream(main)
        out = combine(p, self.y, st["pair_pos"], shared)
        return out, st["rw"], st["sel"]

    def forward(self, x: torch.Tensor):
        self.send(x)
        self.experts()
        return self.finish()

    __call__ = forward

    def _wait(self, which: int) -> None:
        _check(lib().moe_ep_wait(ctypes.byref(self.p.c()), self.world, self.arena.data_ptr(), which, self.max_polls,
                                 self.err.data_ptr(), _stream(self.arena.device)))
