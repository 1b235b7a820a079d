"""fp64 CPU oracle of the sparse top-k MoE FFN backward pass (gradients).

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import or run anything under
``oracle/``. The CUDA library and its Python binding never import it.

What it differentiates is the forward of ``oracle.moe.moe_forward`` with the
expert choice held fixed: top-k selection is piecewise constant in its keys,
so no gradient flows through the choice itself (nor through an aux-loss-free
selection bias, which only ranks experts: "Sparse MoE FFN for DFlash-family
drafters", What's here, MoEGate, whose bias is moved by a sign controller and
never by gradients). The pages name a backward pass and grad parity of the
grouped GEMM against a sorted per-expert loop (same page, Tests) without
formulas; the derivatives below are the chain rule of that forward, written
out without any automatic differentiation:

* expert e on token t: g = x Wg_e^T, u = x Wu_e^T, h = silu(g) * u,
  y = h Wd_e^T, out_t += w_t,e * y;
* dy = w dout, dWd_e += dy^T h, dh = dy Wd_e, du = dh * silu(g),
  dg = dh * u * silu'(g) with silu'(g) = sig(g) (1 + g (1 - sig(g))),
  dWg_e += dg^T x, dWu_e += du^T x, dx += dg Wg_e + du Wu_e;
* routing weight of slot j: dw_j = dout_t . y_e; with renormalisation
  w_j = s_j / sum_m s_m, so ds_i = (dw_i - sum_j dw_j w_j) / sum_m s_m;
* scores to logits: softmax dL = S * (dS - sum_e dS_e S_e); sigmoid
  dL = dS S (1 - S); sqrtsoftplus S = sqrt(softplus(L)): dL = dS sig(L) / (2 S);
* logits: dgate_w = dL^T x, dx += dL gate_w, and a logit bias gets sum_t dL;
* shared expert: out += gamma * Y_s(x); the SwiGLU part as above with
  dy = gamma dout; gated: gamma = sig(x . g), dgamma = dout . Y_s,
  dz = dgamma gamma (1 - gamma), dg_vec = sum_t dz x_t, dx += dz g.

Parity status: pinned by central finite differences of the forward oracle on
small problems (every parameter and input, every score function, bias mode,
renormalisation and shared kind) and by planted mistakes that those pins
catch (tests/test_backward_oracle.py).
"""

from __future__ import annotations

from typing import Dict, Optional, Sequence

import numpy as np

from oracle import moe as om


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def silu_grad(g) -> np.ndarray:
    """d silu(g) / dg = sig(g) (1 + g (1 - sig(g)))."""
    g = _f64(g)
    s = om.sigmoid(g)
    return s * (1.0 + g * (1.0 - s))


def swiglu_backward(X, w_gate_up, w_down, dY) -> Dict[str, np.ndarray]:
    """Gradients of Y = (silu(X Wg^T) * (X Wu^T)) Wd^T for rows X [n,H] given
    dY [n,H]: dX [n,H], d_gate_up [2I,H], d_down [H,I], and Y itself."""
    X, w_gate_up, w_down, dY = _f64(X), _f64(w_gate_up), _f64(w_down), _f64(dY)
    I = w_gate_up.shape[0] // 2
    Wg, Wu = w_gate_up[:I], w_gate_up[I:]
    g = X @ Wg.T
    u = X @ Wu.T
    a = om.silu(g)
    h = a * u
    Y = h @ w_down.T
    d_down = dY.T @ h
    dh = dY @ w_down
    du = dh * a
    dg = dh * u * silu_grad(g)
    d_gate_up = np.concatenate([dg.T @ X, du.T @ X], axis=0)
    dX = dg @ Wg + du @ Wu
    return {"dX": dX, "d_gate_up": d_gate_up, "d_down": d_down, "Y": Y}


def scores_backward(L, S, dS, kind: str) -> np.ndarray:
    """dL from dS for the score function S = f(L) applied row-wise."""
    L, S, dS = _f64(L), _f64(S), _f64(dS)
    if kind == om.SOFTMAX:
        return S * (dS - (dS * S).sum(axis=1, keepdims=True))
    if kind == om.SIGMOID:
        return dS * S * (1.0 - S)
    if kind == om.SQRTSOFTPLUS:
        return dS * om.sigmoid(L) / (2.0 * S)
    raise ValueError(kind)


def weights_backward(S, selected, dw, renormalize: bool) -> np.ndarray:
    """dS [T,E] from the gradient dw [T,k] of the routing weights."""
    S, dw = _f64(S), _f64(dw)
    sel = np.asarray(selected, dtype=np.int64)
    s = np.take_along_axis(S, sel, axis=1)
    if renormalize:
        tot = s.sum(axis=1, keepdims=True)
        safe = np.where(tot > 0, tot, 1.0)
        w = np.where(tot > 0, s / safe, 0.0)
        ds = np.where(tot > 0, (dw - (dw * w).sum(axis=1, keepdims=True)) / safe, 0.0)
    else:
        ds = dw
    dS = np.zeros_like(S)
    np.put_along_axis(dS, sel, ds, axis=1)
    return dS


def moe_backward(x, gate_w, gate_up: Sequence, down: Sequence, dout, *, k: int, score: str, renormalize: bool,
                 bias=None, bias_mode: str = om.BIAS_NONE, shared: str = om.SHARED_NONE, shared_gate_up=None,
                 shared_down=None, shared_gate=None, selected: Optional[np.ndarray] = None) -> Dict[str, np.ndarray]:
    """Gradients of sum(dout * out) for the forward of oracle.moe.moe_forward
    (same arguments; ``selected`` fixes the expert choice, else the top-k of
    the forward is used). Returns dx [T,H], d_gate_w [E,H], d_bias [E] (logit
    bias only, else None), d_gate_up [E,2I,H], d_down [E,H,I], d_routing
    weights [T,k], and d_shared_gate_up / d_shared_down / d_shared_gate when
    there is a shared expert (the gate only when gated)."""
    x, dout = _f64(x), _f64(dout)
    T, H = x.shape
    E = len(gate_up)
    r = om.route(x, gate_w, k, score, bias, bias_mode, renormalize)
    sel = r["selected_experts"] if selected is None else np.asarray(selected, dtype=np.int64)
    w = om.topk_weights(r["scores"], sel, renormalize)
    dx = np.zeros((T, H))
    d_gate_up = [np.zeros_like(_f64(gate_up[e])) for e in range(E)]
    d_down = [np.zeros_like(_f64(down[e])) for e in range(E)]
    dw = np.zeros_like(w)
    for e in range(E):
        t_idx, j_idx = np.nonzero(sel == e)
        if t_idx.size == 0:
            continue
        we = w[t_idx, j_idx][:, None]
        b = swiglu_backward(x[t_idx], gate_up[e], down[e], we * dout[t_idx])
        np.add.at(dx, t_idx, b["dX"])
        d_gate_up[e] += b["d_gate_up"]
        d_down[e] += b["d_down"]
        dw[t_idx, j_idx] = (dout[t_idx] * b["Y"]).sum(axis=1)
    dS = weights_backward(r["scores"], sel, dw, renormalize)
    dL = scores_backward(r["logits"], r["scores"], dS, score)
    d_gate_w = dL.T @ x
    dx += dL @ _f64(gate_w)
    res = {"dx": dx, "d_gate_w": d_gate_w, "d_bias": dL.sum(axis=0) if bias_mode == om.BIAS_LOGIT else None,
           "d_gate_up": np.stack(d_gate_up), "d_down": np.stack(d_down), "d_routing_weights": dw,
           "selected_experts": sel}
    if shared != om.SHARED_NONE:
        gamma = om.shared_gate_values(x, shared_gate, shared)
        b = swiglu_backward(x, shared_gate_up, shared_down, gamma[:, None] * dout)
        dx += b["dX"]
        res["d_shared_gate_up"], res["d_shared_down"] = b["d_gate_up"], b["d_down"]
        if shared == om.SHARED_GATED:
            dz = (dout * b["Y"]).sum(axis=1) * gamma * (1.0 - gamma)
            res["d_shared_gate"] = dz @ x
            dx += dz[:, None] * _f64(shared_gate)[None, :]
    res["dx"] = dx
    return res
