"""Thin Python binding of ``libstm_moe.so``, the B200 sparse top-k MoE FFN forward.

Argument marshalling only: tensors are checked (device, dtype, shape,
contiguity) and their device pointers handed to the C ABI of
``include/moe.h`` on the current CUDA stream. Every step of the forward pass
runs in the library's CUDA kernels; PyTorch provides device memory and
streams. There is no CPU fallback: if the library is missing or cannot be
loaded, every call raises.

Build the library with ``python -m sparse_top_mixture_b200.build``.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Dict, Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libstm_moe.so")

DTYPES = {"f32": 0, "bf16": 1}
SCORES = {"softmax": 0, "sigmoid": 1, "sqrtsoftplus": 2}
BIAS_MODES = {"none": 0, "logit": 1, "select": 2}
SHARED_KINDS = {"none": 0, "plain": 1, "sigmoid_gated": 2}
TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}

STAGES = ("route", "dispatch", "gate_up", "down", "shared", "combine")
DEVERR_BAD_EXPERT_ID = 1
DEVERR_WAIT_TIMEOUT = 2
DEVERR_SMEM_LAYOUT = 4


class MoeError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"moe status {status}: {msg}")
        self.status = status


class moe_problem(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("H", ctypes.c_int64), ("E", ctypes.c_int64), ("k", ctypes.c_int64),
                ("I", ctypes.c_int64), ("I_shared", ctypes.c_int64), ("dtype", ctypes.c_int32),
                ("score", ctypes.c_int32), ("bias_mode", ctypes.c_int32), ("renormalize", ctypes.c_int32),
                ("shared", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class moe_weights(ctypes.Structure):
    _fields_ = [("gate_w", ctypes.c_void_p), ("bias", ctypes.c_void_p), ("gate_up", ctypes.c_void_p),
                ("down", ctypes.c_void_p), ("shared_gate_up", ctypes.c_void_p), ("shared_down", ctypes.c_void_p),
                ("shared_gate", ctypes.c_void_p)]


class moe_grads(ctypes.Structure):
    _fields_ = [("dx", ctypes.c_void_p), ("d_gate_w", ctypes.c_void_p), ("d_bias", ctypes.c_void_p),
                ("d_gate_up", ctypes.c_void_p), ("d_down", ctypes.c_void_p), ("d_shared_gate_up", ctypes.c_void_p),
                ("d_shared_down", ctypes.c_void_p), ("d_shared_gate", ctypes.c_void_p)]


# name -> (restype, argtypes)
_VP, _I32P, _SZ = ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32), ctypes.c_size_t
_PP = ctypes.POINTER(moe_problem)
SIGNATURES = {
    "moe_workspace_size": (ctypes.c_int, [_PP, ctypes.POINTER(ctypes.c_size_t)]),
    "moe_workspace_init": (ctypes.c_int, [_VP, _SZ, _VP]),
    "moe_route": (ctypes.c_int, [_PP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "moe_topk_from_logits": (ctypes.c_int, [_PP, _VP, _VP, _VP, _VP, _VP]),
    "moe_dispatch": (ctypes.c_int, [_PP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "moe_dispatch_noalloc": (ctypes.c_int, [_PP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP]),
    "moe_grouped_swiglu": (ctypes.c_int, [_PP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "moe_shared_expert": (ctypes.c_int, [_PP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "moe_combine": (ctypes.c_int, [_PP, _VP, _VP, _VP, _VP, _VP]),
    "moe_forward": (ctypes.c_int, [_PP, ctypes.POINTER(moe_weights), _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "moe_forward_ex": (ctypes.c_int, [_PP, ctypes.POINTER(moe_weights), _VP, _VP, _VP, _VP, _VP, _SZ, _VP, _VP,
                                      ctypes.POINTER(ctypes.c_void_p)]),
    "moe_gemm_path": (ctypes.c_int, [_PP, _I32P]),
    "moe_launches_per_forward": (ctypes.c_int, [_PP, ctypes.c_int32, _I32P]),
    "moe_read_device_error": (ctypes.c_int, [_VP, _I32P, _VP]),
    "moe_check_device_error": (ctypes.c_int, [_VP, _VP, _I32P]),
    "moe_selftest_wait_timeout": (ctypes.c_int, [_VP, _SZ, _VP]),
    "moe_bias_stash": (ctypes.c_int, [_PP, _VP, _VP, _VP]),
    "moe_bias_update": (ctypes.c_int, [_PP, _VP, _VP, ctypes.c_float, _VP]),
    "moe_forward_counts": (ctypes.c_int, [_PP, _VP, _SZ, ctypes.POINTER(ctypes.c_void_p)]),
    "moe_backward_workspace_size": (ctypes.c_int, [_PP, ctypes.POINTER(ctypes.c_size_t)]),
    "moe_backward": (ctypes.c_int, [_PP, ctypes.POINTER(moe_weights), _VP, _VP, _VP, ctypes.POINTER(moe_grads), _VP,
                                    _SZ, _VP]),
    "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "moe_dispatch_slots": (ctypes.c_int, [_PP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "moe_ep_arena_size": (ctypes.c_int, [_PP, ctypes.c_int32, ctypes.POINTER(ctypes.c_size_t)]),
    "moe_ep_arena_offsets": (ctypes.c_int, [_PP, ctypes.c_int32] + [ctypes.POINTER(ctypes.c_size_t)] * 7),
    "moe_ep_send": (ctypes.c_int, [_PP, ctypes.c_int32, ctypes.c_int32, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP]),
    "moe_ep_wait": (ctypes.c_int, [_PP, ctypes.c_int32, _VP, ctypes.c_int32, ctypes.c_int64, _VP, _VP]),
    "moe_ep_return": (ctypes.c_int, [_PP, ctypes.c_int32, ctypes.c_int32, _VP, _VP, _VP, _VP, _VP, _VP]),
    "moe_ep_experts": (ctypes.c_int, [_PP, ctypes.c_int32, ctypes.c_int32, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "moe_ep_dispatch_send": (ctypes.c_int, [_PP, ctypes.c_int32, ctypes.c_int32, _VP, _VP, _VP, _VP, _VP, _VP, _VP,
                                            _VP, _VP, _VP, _SZ, _VP]),
    "moe_tp_arena_size": (ctypes.c_int, [_PP, ctypes.c_int32, ctypes.POINTER(ctypes.c_size_t)]),
    "moe_tp_arena_offsets": (ctypes.c_int, [_PP, ctypes.c_int32] + [ctypes.POINTER(ctypes.c_size_t)] * 5),
    "moe_tp_scatter": (ctypes.c_int, [_PP, ctypes.c_int32, ctypes.c_int32, _VP, _VP, _VP, _VP, _VP, _VP]),
    "moe_tp_gather": (ctypes.c_int, [_PP, ctypes.c_int32, ctypes.c_int32, _VP, _VP, _VP]),
    "moe_tp_wait": (ctypes.c_int, [_PP, ctypes.c_int32, _VP, ctypes.c_int32, ctypes.c_int64, _VP, _VP]),
}

_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """Load the CUDA library (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; build it with `python -m sparse_top_mixture_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(status: int) -> None:
    if status != 0:
        raise MoeError(status, lib().moe_status_string(status).decode())


@dataclass(frozen=True)
class Problem:
    T: int
    H: int
    E: int
    k: int
    I: int
    I_shared: int = 0
    dtype: str = "bf16"
    score: str = "softmax"
    bias_mode: str = "none"
    renormalize: bool = True
    shared: str = "none"

    @classmethod
    def from_config(cls, cfg, T: Optional[int] = None) -> "Problem":
        return cls(T=cfg.T if T is None else T, H=cfg.H, E=cfg.E, k=cfg.k, I=cfg.I, I_shared=cfg.I_shared,
                   dtype=cfg.dtype, score=cfg.score, bias_mode=cfg.bias_mode, renormalize=cfg.renormalize,
                   shared=cfg.shared)

    def c(self) -> moe_problem:
        return moe_problem(self.T, self.H, self.E, self.k, self.I, self.I_shared, DTYPES[self.dtype],
                           SCORES[self.score], BIAS_MODES[self.bias_mode], int(bool(self.renormalize)),
                           SHARED_KINDS[self.shared], 0)

    @property
    def torch_dtype(self) -> torch.dtype:
        return TORCH_DTYPE[self.dtype]


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(device=None) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _req(t: torch.Tensor, name: str, shape: Sequence[int], dtype: torch.dtype) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def workspace_size(p: Problem) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().moe_workspace_size(ctypes.byref(p.c()), ctypes.byref(n)))
    return int(n.value)


def new_workspace(p: Problem, device="cuda") -> torch.Tensor:
    ws = torch.empty(max(workspace_size(p), 256), dtype=torch.uint8, device=device)
    _check(lib().moe_workspace_init(ws.data_ptr(), ws.numel(), _stream(ws.device)))
    return ws


def gemm_path(p: Problem) -> int:
    out = ctypes.c_int32(-1)
    _check(lib().moe_gemm_path(ctypes.byref(p.c()), ctypes.byref(out)))
    return int(out.value)


def launches_per_forward(p: Problem, two_streams: bool = False) -> int:
    out = ctypes.c_int32(-1)
    _check(lib().moe_launches_per_forward(ctypes.byref(p.c()), int(bool(two_streams)), ctypes.byref(out)))
    return int(out.value)


def read_device_error(ws: torch.Tensor) -> int:
    """Synchronises the current stream; returns and clears the error bits."""
    code = ctypes.c_int32(0)
    st = lib().moe_read_device_error(ws.data_ptr(), ctypes.byref(code), _stream(ws.device))
    if st not in (0, 5):
        _check(st)
    return int(code.value)


def selftest_wait_timeout(ws: torch.Tensor) -> int:
    """Run the bounded-wait self-test on ws's device; returns the error bits
    it left (MOE_DEVERR_WAIT_TIMEOUT expected). Synchronises."""
    _check(lib().moe_selftest_wait_timeout(ws.data_ptr(), ws.numel(), _stream(ws.device)))
    return read_device_error(ws)


def route(p: Problem, x, gate_w, bias=None, shared_gate=None, ws=None):
    """(routing_weights [T,k] fp32, selected_experts [T,k] int64, gamma [T] fp32 or None)."""
    dt = p.torch_dtype
    _req(x, "x", (p.T, p.H), dt)
    _req(gate_w, "gate_w", (p.E, p.H), dt)
    if bias is not None:
        _req(bias, "bias", (p.E,), torch.float32)
    if shared_gate is not None:
        _req(shared_gate, "shared_gate", (p.H,), dt)
    ws = new_workspace(p, x.device) if ws is None else ws
    w = torch.empty(p.T, p.k, dtype=torch.float32, device=x.device)
    sel = torch.empty(p.T, p.k, dtype=torch.int64, device=x.device)
    gam = torch.empty(p.T, dtype=torch.float32, device=x.device) if shared_gate is not None else None
    _check(lib().moe_route(ctypes.byref(p.c()), _ptr(x), _ptr(gate_w), _ptr(bias), _ptr(shared_gate), _ptr(w),
                           _ptr(sel), _ptr(gam), ws.data_ptr(), ws.numel(), _stream(x.device)))
    return w, sel, gam


def topk_from_logits(p: Problem, logits, bias=None):
    _req(logits, "logits", (p.T, p.E), torch.float32)
    if bias is not None:
        _req(bias, "bias", (p.E,), torch.float32)
    w = torch.empty(p.T, p.k, dtype=torch.float32, device=logits.device)
    sel = torch.empty(p.T, p.k, dtype=torch.int64, device=logits.device)
    _check(lib().moe_topk_from_logits(ctypes.byref(p.c()), _ptr(logits), _ptr(bias), _ptr(w), _ptr(sel),
                                      _stream(logits.device)))
    return w, sel


def dispatch(p: Problem, selected, x=None, ws=None) -> Dict[str, torch.Tensor]:
    _req(selected, "selected_experts", (p.T, p.k), torch.int64)
    dev = selected.device
    P = p.T * p.k
    if x is not None:
        _req(x, "x", (p.T, p.H), p.torch_dtype)
    ws = new_workspace(p, dev) if ws is None else ws
    r = {"counts": torch.empty(p.E, dtype=torch.int32, device=dev),
         "offsets": torch.empty(p.E + 1, dtype=torch.int32, device=dev),
         "sorted_pairs": torch.empty(P, dtype=torch.int32, device=dev),
         "pair_pos": torch.empty(P, dtype=torch.int32, device=dev),
         "x_perm": torch.empty(P, p.H, dtype=p.torch_dtype, device=dev) if x is not None else None}
    _check(lib().moe_dispatch(ctypes.byref(p.c()), _ptr(selected), _ptr(x), _ptr(r["counts"]), _ptr(r["offsets"]),
                              _ptr(r["sorted_pairs"]), _ptr(r["pair_pos"]), _ptr(r["x_perm"]), ws.data_ptr(),
                              ws.numel(), _stream(dev)))
    return r


def dispatch_slots(p: Problem, selected, x=None, ws=None) -> Dict[str, torch.Tensor]:
    """moe_dispatch over slots some of which are empty (ids outside [0, E),
    e.g. -1): those are skipped (pair_pos -1) without an error flag."""
    _req(selected, "selected", (p.T, p.k), torch.int64)
    dev = selected.device
    P = p.T * p.k
    ws = new_workspace(p, dev) if ws is None else ws
    r = {"counts": torch.empty(p.E, dtype=torch.int32, device=dev),
         "offsets": torch.empty(p.E + 1, dtype=torch.int32, device=dev),
         "sorted_pairs": torch.empty(P, dtype=torch.int32, device=dev),
         "pair_pos": torch.empty(P, dtype=torch.int32, device=dev),
         "x_perm": torch.empty(P, p.H, dtype=p.torch_dtype, device=dev) if x is not None else None}
    _check(lib().moe_dispatch_slots(ctypes.byref(p.c()), _ptr(selected), _ptr(x), _ptr(r["counts"]),
                                    _ptr(r["offsets"]), _ptr(r["sorted_pairs"]), _ptr(r["pair_pos"]),
                                    _ptr(r["x_perm"]), ws.data_ptr(), ws.numel(), _stream(dev)))
    return r


def dispatch_noalloc(p: Problem, selected, x=None, out: Optional[Dict[str, torch.Tensor]] = None
                     ) -> Dict[str, torch.Tensor]:
    """moe_dispatch without a workspace, for callers that may not allocate
    device memory (the library keeps the dispatch's scratch in fixed device
    arrays; concurrent calls must be serialised). ``out``: optional dict of
    preallocated results (counts, offsets, sorted_pairs, pair_pos and, with
    ``x``, x_perm), so that the call itself allocates nothing; missing ones
    are allocated by PyTorch here. Runs with selected's device current."""
    _req(selected, "selected_experts", (p.T, p.k), torch.int64)
    dev = selected.device
    P = p.T * p.k
    if x is not None:
        _req(x, "x", (p.T, p.H), p.torch_dtype)
    shapes = {"counts": ((p.E,), torch.int32), "offsets": ((p.E + 1,), torch.int32),
              "sorted_pairs": ((P,), torch.int32), "pair_pos": ((P,), torch.int32),
              "x_perm": ((P, p.H), p.torch_dtype)}
    r: Dict[str, Optional[torch.Tensor]] = {}
    for key, (shape, dt) in shapes.items():
        t = None if out is None else out.get(key)
        if key == "x_perm" and x is None:
            r[key] = None
        elif t is None:
            r[key] = torch.empty(*shape, dtype=dt, device=dev)
        else:
            _req(t, key, shape, dt)
            r[key] = t
    with torch.cuda.device(dev):
        _check(lib().moe_dispatch_noalloc(ctypes.byref(p.c()), _ptr(selected), _ptr(x), _ptr(r["counts"]),
                                          _ptr(r["offsets"]), _ptr(r["sorted_pairs"]), _ptr(r["pair_pos"]),
                                          _ptr(r["x_perm"]), _stream(dev)))
    return r


def grouped_swiglu(p: Problem, x_perm, offsets, gate_up, down, routing_weights=None, sorted_pairs=None, ws=None):
    dt = p.torch_dtype
    P = p.T * p.k
    _req(x_perm, "x_perm", (P, p.H), dt)
    _req(offsets, "offsets", (p.E + 1,), torch.int32)
    _req(gate_up, "gate_up", (p.E, 2 * p.I, p.H), dt)
    _req(down, "down", (p.E, p.H, p.I), dt)
    if routing_weights is not None:
        _req(routing_weights, "routing_weights", (p.T, p.k), torch.float32)
        _req(sorted_pairs, "sorted_pairs", (P,), torch.int32)
    ws = new_workspace(p, x_perm.device) if ws is None else ws
    y = torch.empty(P, p.H, dtype=torch.float32, device=x_perm.device)
    _check(lib().moe_grouped_swiglu(ctypes.byref(p.c()), _ptr(x_perm), _ptr(offsets), _ptr(gate_up), _ptr(down),
                                    _ptr(routing_weights), _ptr(sorted_pairs), _ptr(y), ws.data_ptr(), ws.numel(),
                                    _stream(x_perm.device)))
    return y


def shared_expert(p: Problem, x, shared_gate_up, shared_down, gamma=None, ws=None):
    dt = p.torch_dtype
    _req(x, "x", (p.T, p.H), dt)
    _req(shared_gate_up, "shared_gate_up", (2 * p.I_shared, p.H), dt)
    _req(shared_down, "shared_down", (p.H, p.I_shared), dt)
    if gamma is not None:
        _req(gamma, "gamma", (p.T,), torch.float32)
    ws = new_workspace(p, x.device) if ws is None else ws
    out = torch.empty(p.T, p.H, dtype=torch.float32, device=x.device)
    _check(lib().moe_shared_expert(ctypes.byref(p.c()), _ptr(x), _ptr(shared_gate_up), _ptr(shared_down),
                                   _ptr(gamma), _ptr(out), ws.data_ptr(), ws.numel(), _stream(x.device)))
    return out


def combine(p: Problem, y_perm, pair_pos, shared_out=None):
    dt = p.torch_dtype
    _req(y_perm, "y_perm", (p.T * p.k, p.H), torch.float32)
    _req(pair_pos, "pair_pos", (p.T * p.k,), torch.int32)
    if shared_out is not None:
        _req(shared_out, "shared_out", (p.T, p.H), torch.float32)
    out = torch.empty(p.T, p.H, dtype=dt, device=y_perm.device)
    _check(lib().moe_combine(ctypes.byref(p.c()), _ptr(y_perm), _ptr(pair_pos), _ptr(shared_out), _ptr(out),
                             _stream(y_perm.device)))
    return out


def _weights_struct(p: Problem, w: Dict[str, Optional[torch.Tensor]]) -> moe_weights:
    dt = p.torch_dtype
    _req(w["gate_w"], "gate_w", (p.E, p.H), dt)
    _req(w["gate_up"], "gate_up", (p.E, 2 * p.I, p.H), dt)
    _req(w["down"], "down", (p.E, p.H, p.I), dt)
    if w.get("bias") is not None:
        _req(w["bias"], "bias", (p.E,), torch.float32)
    if p.shared != "none":
        _req(w["shared_gate_up"], "shared_gate_up", (2 * p.I_shared, p.H), dt)
        _req(w["shared_down"], "shared_down", (p.H, p.I_shared), dt)
    if w.get("shared_gate") is not None:
        _req(w["shared_gate"], "shared_gate", (p.H,), dt)
    g = lambda n: _ptr(w.get(n))  # noqa: E731
    return moe_weights(g("gate_w"), g("bias"), g("gate_up"), g("down"),
                       g("shared_gate_up") if p.shared != "none" else None,
                       g("shared_down") if p.shared != "none" else None,
                       g("shared_gate") if p.shared == "sigmoid_gated" else None)


def backward_workspace_size(p: Problem) -> int:
    n = ctypes.c_size_t()
    _check(lib().moe_backward_workspace_size(ctypes.byref(p.c()), ctypes.byref(n)))
    return n.value


def backward(p: Problem, weights: Dict[str, Optional[torch.Tensor]], x, dout, selected, ws=None, out=None
             ) -> Dict[str, Optional[torch.Tensor]]:
    """Gradients of sum(dout * out) for the forward with the expert choice
    held at ``selected`` [T,k] int64: dx, d_gate_w, d_bias (logit bias only),
    d_gate_up, d_down and, with a shared expert, d_shared_gate_up,
    d_shared_down and d_shared_gate (gated only). x and dout are in the
    problem's dtype (fp32: SIMT kernels; bf16: tensor-core GEMMs); every
    gradient is fp32. ``out``: optional dict of preallocated fp32 tensors for
    any of them (written, never accumulated into). Async on the current
    stream."""
    cw = _weights_struct(p, weights)
    _req(x, "x", (p.T, p.H), p.torch_dtype)
    _req(dout, "dout", (p.T, p.H), p.torch_dtype)
    _req(selected, "selected", (p.T, p.k), torch.int64)
    dev = x.device
    sh, gated = p.shared != "none", p.shared == "sigmoid_gated"
    shapes = {"dx": (p.T, p.H), "d_gate_w": (p.E, p.H), "d_bias": (p.E,) if p.bias_mode == "logit" else None,
              "d_gate_up": (p.E, 2 * p.I, p.H), "d_down": (p.E, p.H, p.I),
              "d_shared_gate_up": (2 * p.I_shared, p.H) if sh else None,
              "d_shared_down": (p.H, p.I_shared) if sh else None, "d_shared_gate": (p.H,) if gated else None}
    g: Dict[str, Optional[torch.Tensor]] = {}
    for key, shape in shapes.items():
        t = None if (out is None or shape is None) else out.get(key)
        if shape is None:
            g[key] = None
        elif t is None:
            g[key] = torch.empty(*shape, dtype=torch.float32, device=dev)
        else:
            _req(t, key, shape, torch.float32)
            g[key] = t
    if ws is None:
        ws = torch.zeros(backward_workspace_size(p), dtype=torch.uint8, device=dev)
    cg = moe_grads(*[_ptr(g[f]) for f, _ in moe_grads._fields_])
    _check(lib().moe_backward(ctypes.byref(p.c()), ctypes.byref(cw), _ptr(x), _ptr(dout), _ptr(selected),
                              ctypes.byref(cg), ws.data_ptr(), ws.numel(), _stream(dev)))
    return g


class SparseMoE:
    """A sparse top-k MoE FFN with device-resident weights and workspace.

    ``weights``: gate_w [E,H], gate_up [E,2I,H], down [E,H,I], optional bias
    [E] fp32, shared_gate_up [2I_s,H], shared_down [H,I_s], shared_gate [H].
    ``overlap_shared``: run the shared expert on a second stream concurrently
    with the routed path (the call still completes on the current stream).
    """

    def __init__(self, p: Problem, weights: Dict[str, Optional[torch.Tensor]], device="cuda",
                 overlap_shared: bool = True):
        self.p = p
        self.w = weights
        self._cw = _weights_struct(p, weights)
        self.device = torch.device(device)
        self.ws = new_workspace(p, self.device)
        self.aux = torch.cuda.Stream(self.device) if (overlap_shared and p.shared != "none") else None

    def _outputs(self, x, out, routing_weights, selected_experts):
        p = self.p
        _req(x, "x", (p.T, p.H), p.torch_dtype)
        out = torch.empty(p.T, p.H, dtype=p.torch_dtype, device=x.device) if out is None else out
        rw = torch.empty(p.T, p.k, dtype=torch.float32, device=x.device) if routing_weights is None \
            else routing_weights
        sel = torch.empty(p.T, p.k, dtype=torch.int64, device=x.device) if selected_experts is None \
            else selected_experts
        return out, rw, sel

    def forward(self, x, out=None, routing_weights=None, selected_experts=None, events=None):
        """out, routing_weights, selected_experts = moe(x). ``events``: optional
        len(STAGES)+1 torch.cuda.Event recorded before each stage and after the
        combine."""
        p = self.p
        out, rw, sel = self._outputs(x, out, routing_weights, selected_experts)
        arr = None
        if events is not None:
            if len(events) != len(STAGES) + 1:
                raise ValueError("need one event per stage plus one")
            arr = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
        aux = self.aux.cuda_stream if self.aux is not None else None
        _check(lib().moe_forward_ex(ctypes.byref(p.c()), ctypes.byref(self._cw), _ptr(x), _ptr(out), _ptr(rw),
                                    _ptr(sel), self.ws.data_ptr(), self.ws.numel(), _stream(x.device), aux, arr))
        return out, rw, sel

    __call__ = forward

    def forward_from_host(self, x_host: torch.Tensor, out_host: torch.Tensor, x_dev=None, out_dev=None,
                          rw=None, sel=None):
        """End-to-end call from pinned host memory: copy x in, run the forward,
        copy out back, all on the current stream (the caller synchronises)."""
        p = self.p
        x_dev = torch.empty(p.T, p.H, dtype=p.torch_dtype, device=self.device) if x_dev is None else x_dev
        x_dev.copy_(x_host, non_blocking=True)
        out_dev, rw, sel = self.forward(x_dev, out_dev, rw, sel)
        out_host.copy_(out_dev, non_blocking=True)
        return out_host

    def read_device_error(self) -> int:
        return read_device_error(self.ws)

    def forward_counts(self) -> torch.Tensor:
        """Per-expert counts [E] int32 of the last forward (a view into the
        workspace, overwritten by the next forward)."""
        ptr = ctypes.c_void_p()
        _check(lib().moe_forward_counts(ctypes.byref(self.p.c()), self.ws.data_ptr(), self.ws.numel(),
                                        ctypes.byref(ptr)))
        off = ptr.value - self.ws.data_ptr()
        return self.ws[off:off + 4 * self.p.E].view(torch.int32)


def bias_stash(p: Problem, counts: torch.Tensor, load_stash: torch.Tensor) -> None:
    """load_stash [E] int64 += counts [E] int32 (async on the current stream)."""
    _req(counts, "counts", (p.E,), torch.int32)
    _req(load_stash, "load_stash", (p.E,), torch.int64)
    _check(lib().moe_bias_stash(ctypes.byref(p.c()), _ptr(counts), _ptr(load_stash), _stream(counts.device)))


def bias_update(p: Problem, load_stash: torch.Tensor, bias: torch.Tensor, rate: float) -> None:
    """Sign-controller step on bias [E] fp32 in place from load_stash [E]
    int64 (then zeroed); async on the current stream."""
    _req(load_stash, "load_stash", (p.E,), torch.int64)
    _req(bias, "bias", (p.E,), torch.float32)
    _check(lib().moe_bias_update(ctypes.byref(p.c()), _ptr(load_stash), _ptr(bias), float(rate),
                                 _stream(bias.device)))


def allreduce_loads(load_stash: torch.Tensor, group=None) -> torch.Tensor:
    """Sum the stashed loads over the ranks of `group` in place (no-op
    without torch.distributed or with one rank)."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(load_stash, op=dist.ReduceOp.SUM, group=group)
    return load_stash


class BiasBalancer:
    """Deferred aux-loss-free balancing of a SparseMoE's selection bias
    ("Sparse MoE FFN for DFlash-family drafters", MoEGate and the deferred
    balance updates): ``stash()`` after a forward adds that forward's
    per-expert counts; ``update()`` before the next forward sums the stash
    over the data-parallel ``group`` and moves the fp32 bias (the SparseMoE's
    own ``bias`` tensor, in place) by ``rate`` toward balance, then clears the
    stash, so a second ``update()`` changes nothing."""

    def __init__(self, moe: "SparseMoE", rate: float, group=None):
        if moe.p.bias_mode == "none" or moe.w.get("bias") is None:
            raise ValueError("the problem has no selection / logit bias to balance")
        self.moe = moe
        self.rate = float(rate)
        self.group = group
        self.bias = moe.w["bias"]
        self.load_stash = torch.zeros(moe.p.E, dtype=torch.int64, device=moe.device)

    def forward_counts(self) -> torch.Tensor:
        """View of the per-expert counts the last forward wrote (int32 [E])."""
        return self.moe.forward_counts()

    def stash(self, counts: Optional[torch.Tensor] = None) -> None:
        bias_stash(self.moe.p, self.forward_counts() if counts is None else counts, self.load_stash)

    def update(self) -> None:
        allreduce_loads(self.load_stash, self.group)
        bias_update(self.moe.p, self.load_stash, self.bias, self.rate)


class GraphedForward:
    """One forward recorded as a CUDA graph on fixed device buffers.

    Replaying it runs the same kernels on the same buffers as
    ``moe.forward(x, out, routing_weights, selected_experts)``, with one graph
    launch in place of one launch per kernel. Write the next batch into ``x``
    (on the stream the replay is issued on) and call ``replay()``; results
    land in ``out``, ``routing_weights`` and ``selected_experts``.
    """

    def __init__(self, moe: "SparseMoE", x, out=None, routing_weights=None, selected_experts=None, events=None):
        """``events``: optional len(STAGES)+1 timing events recorded between
        the stages at every replay (as in ``SparseMoE.forward``)."""
        self.moe = moe
        self.x = x
        self.out, self.rw, self.sel = moe._outputs(x, out, routing_weights, selected_experts)
        # one eager call first: the library's one-time host setup (kernel
        # attributes, driver entry points) then happens outside the capture
        moe.forward(self.x, self.out, self.rw, self.sel, events=events)
        torch.cuda.synchronize(moe.device)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph, capture_error_mode="thread_local"):
            moe.forward(self.x, self.out, self.rw, self.sel, events=events)
        torch.cuda.synchronize(moe.device)

    def replay(self):
        self.graph.replay()
        return self.out, self.rw, self.sel

    __call__ = replay


class HostPipeline:
    """Forward passes over batches that live in pinned host memory, with the
    copies of one batch overlapping the compute of its neighbours.

    Slot i % depth owns a stream, a workspace and device buffers; batch i is
    copied in, run and copied back on its slot's stream, so batch i+1's
    host->device copy and batch i-1's device->host copy proceed while batch i
    computes (the GPU's copy engines run beside the SMs). Each batch's own
    three steps stay ordered on its stream. With depth 3 a slot's next input
    copy never waits on its previous output copy while the compute engine is
    busy, so the copies stay off the forward's critical path.
    """

    def __init__(self, moe: SparseMoE, depth: int = 3, graphs: bool = True):
        p = moe.p
        self.moe = moe
        self.slots = []
        for i in range(depth):
            m = moe if i == 0 else SparseMoE(p, moe.w, moe.device, overlap_shared=moe.aux is not None)
            slot = {
                "moe": m,
                "stream": torch.cuda.Stream(moe.device),
                "x": torch.empty(p.T, p.H, dtype=p.torch_dtype, device=moe.device),
                "out": torch.empty(p.T, p.H, dtype=p.torch_dtype, device=moe.device),
                "rw": torch.empty(p.T, p.k, dtype=torch.float32, device=moe.device),
                "sel": torch.empty(p.T, p.k, dtype=torch.int64, device=moe.device),
            }
            # each slot's forward as one graph launch on the slot's buffers
            slot["graph"] = GraphedForward(m, slot["x"], slot["out"], slot["rw"], slot["sel"]) if graphs else None
            self.slots.append(slot)
        self.i = 0

    def submit(self, x_host: torch.Tensor, out_host: torch.Tensor) -> torch.cuda.Stream:
        """Enqueue one batch (pinned host tensors [T,H]); returns its stream.
        out_host is complete once that stream has passed this call."""
        slot = self.slots[self.i % len(self.slots)]
        self.i += 1
        s = slot["stream"]
        s.wait_stream(torch.cuda.current_stream(self.moe.device))
        with torch.cuda.stream(s):
            slot["x"].copy_(x_host, non_blocking=True)
            if slot["graph"] is not None:
                slot["graph"].replay()
            else:
                slot["moe"].forward(slot["x"], slot["out"], slot["rw"], slot["sel"])
            out_host.copy_(slot["out"], non_blocking=True)
        return s

    def synchronize(self) -> None:
        for slot in self.slots:
            slot["stream"].synchronize()
