"""Brute-force per-token MoE forward on tiny inputs (pure Python, math.fsum).

TEST INFRASTRUCTURE ONLY (same import rule as ``oracle.moe``). It restates the
method a second, independent way -- explicit index loops, exactly rounded sums,
a full ``sorted`` of every token's keys, scalar transcendental forms different
from the vectorised oracle's -- so that a dropped term, a wrong sign or index
or a transposed operand in ``oracle.moe`` shows up as a mismatch.

Definitions followed: "mstar.model.components.moe" (Router contract,
TopKRouter, SparseMoeBlock fused layout, SparseMoeBlockWithSharedExpert);
"Sparse MoE FFN for DFlash-family drafters" (MoEGate: sqrtsoftplus scores, fp32
bias for selection only); "feat: Phase 43 -- Sparse/Grouped MoE Dispatch"
(only the assigned top-k experts contribute).
"""

from __future__ import annotations

import math
from typing import Dict, List, Optional


def _sigmoid(v: float) -> float:
    if v >= 0:
        return 1.0 / (1.0 + math.exp(-v))
    e = math.exp(v)
    return e / (1.0 + e)


def _sqrtsoftplus(v: float) -> float:
    # log(1 + e^v), written without the max/abs split used by the oracle.
    if v > 30.0:
        sp = v + math.log1p(math.exp(-v))
    else:
        sp = math.log1p(math.exp(v))
    return math.sqrt(sp)


def _dot(a: List[float], b: List[float]) -> float:
    return math.fsum(ai * bi for ai, bi in zip(a, b))


def _expert(xt: List[float], gu: List[List[float]], dn: List[List[float]]) -> List[float]:
    """One token through one SwiGLU expert: gu is [2I][H], dn is [H][I]."""
    I = len(gu) // 2
    act = []
    for i in range(I):
        g = _dot(xt, gu[i])
        u = _dot(xt, gu[I + i])
        act.append(g * _sigmoid(g) * u)
    return [_dot(act, dn[o]) for o in range(len(dn))]


def brute_forward(x, gate_w, gate_up, down, *, k: int, score: str, renormalize: bool,
                  bias=None, bias_mode: str = "none", shared: str = "none",
                  shared_gate_up=None, shared_down=None, shared_gate=None) -> Dict[str, list]:
    """Token-by-token loop. Inputs are nested lists (or anything indexable)."""
    T = len(x)
    E = len(gate_w)
    H = len(x[0])
    out_all, sel_all, w_all = [], [], []
    for t in range(T):
        xt = [float(v) for v in x[t]]
        logits = []
        for e in range(E):
            l = _dot(xt, [float(v) for v in gate_w[e]])
            if bias_mode == "logit":
                l += float(bias[e])
            logits.append(l)
        if score == "softmax":
            mx = max(logits)
            z = [math.exp(l - mx) for l in logits]
            zs = math.fsum(z)
            s = [zi / zs for zi in z]
        elif score == "sigmoid":
            s = [_sigmoid(l) for l in logits]
        elif score == "sqrtsoftplus":
            s = [_sqrtsoftplus(l) for l in logits]
        else:
            raise ValueError(score)
        key = [s[e] + (float(bias[e]) if bias_mode == "select" else 0.0) for e in range(E)]
        chosen = sorted(range(E), key=lambda e: (-key[e], e))[:k]
        w = [s[e] for e in chosen]
        if renormalize:
            tot = math.fsum(w)
            w = [wi / tot for wi in w] if tot > 0 else [0.0] * k
        terms: List[List[float]] = [[] for _ in range(H)]
        for j, e in enumerate(chosen):
            y = _expert(xt, gate_up[e], down[e])
            for o in range(H):
                terms[o].append(w[j] * y[o])
        if shared != "none":
            gam = 1.0
            if shared == "sigmoid_gated":
                gam = _sigmoid(_dot(xt, [float(v) for v in shared_gate]))
            ys = _expert(xt, shared_gate_up, shared_down)
            for o in range(H):
                terms[o].append(gam * ys[o])
        out_all.append([math.fsum(tm) for tm in terms])
        sel_all.append(chosen)
        w_all.append(w)
    return {"out": out_all, "selected_experts": sel_all, "routing_weights": w_all}


def brute_dispatch(selected, E: int) -> Dict[str, list]:
    """Bucket the flat pairs expert by expert, visiting pairs in order."""
    flat = [int(e) for row in selected for e in row]
    buckets: List[List[int]] = [[] for _ in range(E)]
    for q, e in enumerate(flat):
        buckets[e].append(q)
    counts = [len(b) for b in buckets]
    offsets = [0]
    for c in counts:
        offsets.append(offsets[-1] + c)
    sorted_pairs = [q for b in buckets for q in b]
    pair_pos: List[Optional[int]] = [None] * len(flat)
    for p, q in enumerate(sorted_pairs):
        pair_pos[q] = p
    return {"counts": counts, "offsets": offsets, "sorted_pairs": sorted_pairs, "pair_pos": pair_pos}
