"""fp64 CPU oracle of the sparse top-k MoE FFN forward (dense-masked form).

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import or run anything under
``oracle/``. The CUDA library and its Python binding never import it, and the
product path has no CPU fallback.

What it computes, and where each step is defined:

* Dense-masked dispatch is the correctness reference: every routed expert runs
  on every token and the per-expert result is masked by the routing decision;
  a sparse dispatch must be numerically equivalent to it ("feat: Phase 43 --
  Sparse/Grouped MoE Dispatch (v4.0.0-alpha.3)", Summary and Core /
  DispatchKind).
* Router contract: hidden_states [T,H] in; routing_weights [T,k] and int64
  selected_experts [T,k] out ("mstar.model.components.moe", Router contract;
  TopKRouter).
* Scores: softmax over all E experts, then top-k, optionally renormalised so
  the k weights sum to 1 (TopKRouter, ``norm_topk_prob``); sigmoid scores
  (the decode problem); sqrtsoftplus scores with an fp32 aux-loss-free bias
  that enters selection only ("Sparse MoE FFN for DFlash-family drafters",
  What's here, MoEGate).
* Stacked expert weights in the fused layout: gate_up [E, 2I, H] (rows 0..I-1
  gate, rows I..2I-1 up) and down [E, H, I] ("mstar.model.components.moe",
  SparseMoeBlock; "Sparse MoE FFN for DFlash-family drafters", GroupedExperts).
* SwiGLU expert: (silu(x W_g^T) * (x W_u^T)) W_d^T with silu(a) = a sigmoid(a)
  (dispatch_experts_fused "runs SwiGLU per expert"; the Phase 43 page's
  "SwiGLU matmul").
* Sorted-segment dispatch: a stable argsort of routed expert ids into
  contiguous per-expert segments ("Sparse MoE FFN for DFlash-family
  drafters", What's here, SparseMoE; Phase 43, Neural Network,
  sparse_grouped_dispatch).
* Shared expert: plain (DeepSeek, summed) or gated, out = routed(x) +
  sigmoid(shared_gate(x)) * shared_expert(x) ("mstar.model.components.moe",
  SparseMoeBlockWithSharedExpert; "MoE: shared experts, parameterized V_TOPK
  routing, explicit stage attribution", 3. Tests, the three variants).

Readings taken where the pages are silent:
softmax is over all E experts before top-k; equal keys go to the lower expert
index; the gate half of gate_up comes first; the shared gate is a bias-free
vector [H]; the routed scaling factor is 1; a zero renormalisation sum gives
zero weights; sqrtsoftplus(l) = sqrt(log(1 + e^l)).

Parity status: every function here is pinned by tests under ``tests/``
(brute force, closed forms, library reductions, invariants), except that the
definition of sqrtsoftplus is pinned only up to the reading above (the pages
name the function without a formula): "parity unpinned" beyond that reading.
"""

from __future__ import annotations

from typing import Dict, Optional, Sequence

import numpy as np

SOFTMAX, SIGMOID, SQRTSOFTPLUS = "softmax", "sigmoid", "sqrtsoftplus"
BIAS_NONE, BIAS_LOGIT, BIAS_SELECT = "none", "logit", "select"
SHARED_NONE, SHARED_PLAIN, SHARED_GATED = "none", "plain", "sigmoid_gated"


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


# ----------------------------------------------------------------------------
# Router
# ----------------------------------------------------------------------------

def router_logits(x, gate_w, bias=None, bias_mode: str = BIAS_NONE) -> np.ndarray:
    """l[t,e] = sum_h x[t,h] gate_w[e,h] (+ b[e] when the bias is a logit bias).

    TopKRouter is a linear map hidden -> num_experts ("mstar.model.components.moe").
    """
    L = _f64(x) @ _f64(gate_w).T
    if bias_mode == BIAS_LOGIT:
        L = L + _f64(bias)[None, :]
    return L


def sigmoid(a) -> np.ndarray:
    a = _f64(a)
    out = np.empty_like(a)
    pos = a >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-a[pos]))
    ea = np.exp(a[~pos])
    out[~pos] = ea / (1.0 + ea)
    return out


def softplus(a) -> np.ndarray:
    a = _f64(a)
    return np.maximum(a, 0.0) + np.log1p(np.exp(-np.abs(a)))


def softmax_rows(L) -> np.ndarray:
    L = _f64(L)
    m = L.max(axis=1, keepdims=True)
    z = np.exp(L - m)
    return z / z.sum(axis=1, keepdims=True)


def scores(L, kind: str) -> np.ndarray:
    """Score function applied to router logits."""
    if kind == SOFTMAX:
        return softmax_rows(L)
    if kind == SIGMOID:
        return sigmoid(L)
    if kind == SQRTSOFTPLUS:
        return np.sqrt(softplus(L))
    raise ValueError(kind)


def selection_keys(S, bias=None, bias_mode: str = BIAS_NONE) -> np.ndarray:
    """The aux-loss-free bias is added for selection only ("Sparse MoE FFN for
    DFlash-family drafters", MoEGate)."""
    if bias_mode == BIAS_SELECT:
        return _f64(S) + _f64(bias)[None, :]
    return _f64(S)


def select_topk(K, k: int) -> np.ndarray:
    """Indices of the k largest keys per row, in descending key order; equal
    keys keep ascending expert index (a stable sort on -key)."""
    order = np.argsort(-_f64(K), axis=1, kind="stable")
    return order[:, :k].astype(np.int64)


def topk_weights(S, selected, renormalize: bool) -> np.ndarray:
    """w = score of each selected expert, divided by their sum when renormalised
    (TopKRouter ``norm_topk_prob``)."""
    w = np.take_along_axis(_f64(S), selected, axis=1)
    if renormalize:
        tot = w.sum(axis=1, keepdims=True)
        safe = np.where(tot > 0, tot, 1.0)
        w = np.where(tot > 0, w / safe, 0.0)
    return w


def route(x, gate_w, k: int, score: str, bias=None, bias_mode: str = BIAS_NONE,
          renormalize: bool = True) -> Dict[str, np.ndarray]:
    """Router forward: (routing_weights [T,k] fp64, selected_experts [T,k] int64)
    plus the logits, scores and selection keys for tie analysis."""
    L = router_logits(x, gate_w, bias, bias_mode)
    S = scores(L, score)
    K = selection_keys(S, bias, bias_mode)
    sel = select_topk(K, k)
    w = topk_weights(S, sel, renormalize)
    return {"routing_weights": w, "selected_experts": sel, "logits": L, "scores": S, "keys": K}


# ----------------------------------------------------------------------------
# Dispatch
# ----------------------------------------------------------------------------

def dispatch(selected, E: int) -> Dict[str, np.ndarray]:
    """Sorted-segment dispatch of the T*k (token, slot) pairs.

    counts[e]: pairs routed to e; offsets: exclusive prefix sum (E+1 entries);
    sorted_pairs[p]: the flat pair index q = t*k + j at segment position p,
    pairs of one expert in ascending q; pair_pos: the inverse permutation.
    """
    flat = np.asarray(selected, dtype=np.int64).reshape(-1)
    counts = np.bincount(flat, minlength=E).astype(np.int64)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    sorted_pairs = np.argsort(flat, kind="stable").astype(np.int64)
    pair_pos = np.empty_like(sorted_pairs)
    pair_pos[sorted_pairs] = np.arange(flat.size, dtype=np.int64)
    return {"counts": counts, "offsets": offsets, "sorted_pairs": sorted_pairs, "pair_pos": pair_pos}


# ----------------------------------------------------------------------------
# Expert MLP
# ----------------------------------------------------------------------------

def silu(a) -> np.ndarray:
    """silu(a) = a * sigmoid(a)."""
    a = _f64(a)
    return a * sigmoid(a)


def gate_half(w_gate_up, I: int) -> np.ndarray:
    return _f64(w_gate_up)[:I]


def up_half(w_gate_up, I: int) -> np.ndarray:
    return _f64(w_gate_up)[I:2 * I]


def swiglu_mlp(X, w_gate_up, w_down) -> np.ndarray:
    """SwiGLU MLP with fused gate_up [2I, H] and down [H, I] weights."""
    w_gate_up = _f64(w_gate_up)
    I = w_gate_up.shape[0] // 2
    X = _f64(X)
    g = X @ gate_half(w_gate_up, I).T
    u = X @ up_half(w_gate_up, I).T
    return (silu(g) * u) @ _f64(w_down).T


def routing_matrix(weights, selected, E: int):
    """Dense [T,E] routing matrix M and selection mask."""
    T, k = selected.shape
    M = np.zeros((T, E), dtype=np.float64)
    mask = np.zeros((T, E), dtype=bool)
    rows = np.repeat(np.arange(T), k)
    M[rows, selected.reshape(-1)] = _f64(weights).reshape(-1)
    mask[rows, selected.reshape(-1)] = True
    return M, mask


def shared_gate_values(x, shared_gate, shared: str) -> np.ndarray:
    """gamma[t] = 1 for a plain shared expert, sigmoid(x[t] . g) when gated."""
    T = _f64(x).shape[0]
    if shared == SHARED_GATED:
        return sigmoid(_f64(x) @ _f64(shared_gate))
    return np.ones(T, dtype=np.float64)


def moe_forward(x, gate_w, gate_up: Sequence, down: Sequence, *, k: int, score: str,
                renormalize: bool, bias=None, bias_mode: str = BIAS_NONE,
                shared: str = SHARED_NONE, shared_gate_up=None, shared_down=None, shared_gate=None,
                selected: Optional[np.ndarray] = None, skip_unrouted: bool = False) -> Dict[str, np.ndarray]:
    """Dense-masked MoE FFN forward in fp64.

    ``gate_up[e]`` / ``down[e]`` may be arrays or any indexable that yields one
    expert's [2I,H] / [H,I] weights (so very large stacks can be streamed).

    ``selected``: when given, routing uses these indices instead of the top-k
    (weights are still the scores at those indices); used to recompute the
    reference from another, equally valid, choice among near-tied experts.

    ``skip_unrouted``: do not evaluate experts that no token selected. Their
    masked contribution is exactly zero either way, so the result is identical
    (a test pins this); it only saves time at large sizes.
    """
    x = _f64(x)
    T = x.shape[0]
    E = len(gate_up)
    r = route(x, gate_w, k, score, bias, bias_mode, renormalize)
    if selected is not None:
        sel = np.asarray(selected, dtype=np.int64)
        w = topk_weights(r["scores"], sel, renormalize)
        r["selected_experts"], r["routing_weights"] = sel, w
    sel, w = r["selected_experts"], r["routing_weights"]
    M, mask = routing_matrix(w, sel, E)
    H = x.shape[1]
    out = np.zeros((T, H), dtype=np.float64)
    for e in range(E):
        if skip_unrouted and not mask[:, e].any():
            continue
        Y = swiglu_mlp(x, gate_up[e], down[e])
        out += np.where(mask[:, e:e + 1], M[:, e:e + 1] * Y, 0.0)
    routed = out.copy()
    gamma = None
    if shared != SHARED_NONE:
        gamma = shared_gate_values(x, shared_gate, shared)
        out = out + gamma[:, None] * swiglu_mlp(x, shared_gate_up, shared_down)
    res = dict(r)
    res.update(dispatch(sel, E))
    res["out"] = out
    res["routed_out"] = routed
    res["shared_gamma"] = gamma
    return res


def decision_margins(keys, k: int) -> np.ndarray:
    """Per token, the gap between the k-th and (k+1)-th largest selection key
    (inf when k == E). Tokens with a tiny gap have several valid top-k sets
    once keys carry fp32 rounding."""
    K = np.sort(_f64(keys), axis=1)[:, ::-1]
    if k >= K.shape[1]:
        return np.full(K.shape[0], np.inf)
    return K[:, k - 1] - K[:, k]
