"""Pins of the backward oracle (oracle/backward.py) by central finite
differences of the forward oracle, with the expert choice held fixed, by
torch autograd of a plain per-expert loop in fp64, and planted mistakes that
those pins must catch. CPU only."""

from __future__ import annotations

import numpy as np
import pytest

import oracle.backward as ob
import torch
import torch_loop
from oracle_pins import oracle_run, tiny_problem

CASES = []
for _i, (_score, _bias, _renorm) in enumerate(
        [(s, b, r) for s in ("softmax", "sigmoid", "sqrtsoftplus") for b in ("none", "logit", "select")
         for r in (True, False)]):
    CASES.append((_score, _bias, _renorm, ("none", "plain", "sigmoid_gated")[_i % 3]))

PARAMS = ("x", "gate_w", "bias", "gate_up", "down", "shared_gate_up", "shared_down", "shared_gate")
GRAD_KEY = {"x": "dx", "gate_w": "d_gate_w", "bias": "d_bias", "gate_up": "d_gate_up", "down": "d_down",
            "shared_gate_up": "d_shared_gate_up", "shared_down": "d_shared_down", "shared_gate": "d_shared_gate"}


def _problem(score, bias_mode, renorm, shared, seed):
    cfg, a = tiny_problem(score, bias_mode, renorm, shared, T=6, H=8, E=5, k=2, I=4, I_shared=3, seed=seed)
    return cfg, {n: (np.asarray(v, np.float64) if v is not None else None) for n, v in a.items()}


def _loss(cfg, a, dout, sel):
    return float((oracle_run(cfg, a, selected=sel)["out"] * dout).sum())


def _backward(cfg, a, dout, sel):
    return ob.moe_backward(a["x"], a["gate_w"], a["gate_up"], a["down"], dout, k=cfg.k, score=cfg.score,
                           renormalize=cfg.renormalize, bias=a.get("bias"), bias_mode=cfg.bias_mode,
                           shared=cfg.shared, shared_gate_up=a.get("shared_gate_up"),
                           shared_down=a.get("shared_down"), shared_gate=a.get("shared_gate"), selected=sel)


def finite_difference_pin(case, seed=0, eps=1e-5):
    """Directional derivative of sum(dout * out) along a random direction of
    each parameter, central differences vs the oracle's gradient."""
    score, bias_mode, renorm, shared = case
    cfg, a = _problem(score, bias_mode, renorm, shared, seed)
    rng = np.random.default_rng(seed + 100)
    dout = rng.normal(size=(cfg.T, cfg.H))
    sel = oracle_run(cfg, a)["selected_experts"]
    g = _backward(cfg, a, dout, sel)
    for name in PARAMS:
        if a.get(name) is None:
            continue
        v = rng.normal(size=a[name].shape)
        plus = dict(a, **{name: a[name] + eps * v})
        minus = dict(a, **{name: a[name] - eps * v})
        fd = (_loss(cfg, plus, dout, sel) - _loss(cfg, minus, dout, sel)) / (2 * eps)
        grad = g.get(GRAD_KEY[name])
        an = 0.0 if grad is None else float((np.asarray(grad) * v).sum())  # a selection bias has no gradient
        if abs(fd - an) > 1e-6 * max(1.0, abs(an)):
            return False, f"{case} {name}: finite difference {fd:.9g} vs gradient {an:.9g}"
    return True, ""


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(str(v) for v in c))
def test_backward_matches_finite_differences(case):
    for seed in (0, 1):
        ok, detail = finite_difference_pin(case, seed)
        assert ok, detail


def test_gradient_is_linear_in_dout():
    """Doubling dout doubles every gradient exactly (power-of-two scaling)."""
    cfg, a = _problem("softmax", "logit", True, "sigmoid_gated", 3)
    dout = np.random.default_rng(3).normal(size=(cfg.T, cfg.H))
    sel = oracle_run(cfg, a)["selected_experts"]
    g1, g2 = _backward(cfg, a, dout, sel), _backward(cfg, a, 2 * dout, sel)
    for key in GRAD_KEY.values():
        if g1.get(key) is not None:
            assert np.array_equal(2 * g1[key], g2[key]), key


# ---- planted mistakes: each must make some finite-difference pin fail ------

def _mut_silu_grad(g):
    return ob.om.sigmoid(g)  # drops the g * sig'(g) term


def _mut_weights_backward(S, selected, dw, renormalize):
    S, dw = np.asarray(S, np.float64), np.asarray(dw, np.float64)
    s = np.take_along_axis(S, selected, axis=1)
    ds = dw / s.sum(axis=1, keepdims=True) if renormalize else dw  # misses the -sum(dw w) term
    dS = np.zeros_like(S)
    np.put_along_axis(dS, selected, ds, axis=1)
    return dS


def _mut_scores_backward(L, S, dS, kind):
    if kind == "softmax":
        return S * (dS + (dS * S).sum(axis=1, keepdims=True))  # sign of the normaliser term
    if kind == "sqrtsoftplus":
        return dS * ob.om.sigmoid(L) / S  # loses the 1/2 of the square root
    return dS * S * (1.0 - S)


_orig_swiglu_backward = ob.swiglu_backward


def _mut_swiglu_backward(X, w_gate_up, w_down, dY):
    b = _orig_swiglu_backward(X, w_gate_up, w_down, dY)
    I = np.asarray(w_gate_up).shape[0] // 2
    b["d_gate_up"] = np.concatenate([b["d_gate_up"][I:], b["d_gate_up"][:I]], axis=0)  # gate/up halves swapped
    return b


MUTANTS = {"silu_grad": _mut_silu_grad, "weights_backward": _mut_weights_backward,
           "scores_backward": _mut_scores_backward, "swiglu_backward": _mut_swiglu_backward}


@pytest.mark.parametrize("name", list(MUTANTS))
def test_planted_backward_mistake_is_caught(name, monkeypatch):
    monkeypatch.setattr(ob, name, MUTANTS[name])
    caught = [c for c in CASES if not finite_difference_pin(c)[0]]
    assert caught, f"no finite-difference pin caught the planted mistake in {name}"


def test_planted_shared_gate_mistake_is_caught(monkeypatch):
    """Dropping the shared gate's own gradient (and its dx term) is caught."""
    orig = ob.moe_backward

    def no_gate_grad(*args, **kw):
        r = orig(*args, **kw)
        if r.get("d_shared_gate") is not None:
            r["d_shared_gate"] = np.zeros_like(r["d_shared_gate"])
        return r

    monkeypatch.setattr(ob, "moe_backward", no_gate_grad)
    caught = [c for c in CASES if c[3] == "sigmoid_gated" and not finite_difference_pin(c)[0]]
    assert caught


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(str(v) for v in c))
def test_backward_matches_autograd_of_a_per_expert_loop(case):
    """torch autograd (fp64) of the per-expert loop, for the oracle's choice,
    gives the oracle's gradients to rounding."""
    score, bias_mode, renorm, shared = case
    cfg, a = _problem(score, bias_mode, renorm, shared, 2)
    dout = np.random.default_rng(7).normal(size=(cfg.T, cfg.H))
    sel = oracle_run(cfg, a)["selected_experts"]
    g = _backward(cfg, a, dout, sel)
    leaves = {k: torch.from_numpy(v).requires_grad_(True) for k, v in a.items() if v is not None}
    out = torch_loop.forward(cfg, leaves, torch.from_numpy(sel))
    assert np.allclose(out.detach().numpy(), oracle_run(cfg, a, selected=sel)["out"], rtol=1e-12, atol=1e-12)
    (out * torch.from_numpy(dout)).sum().backward()
    for name, key in torch_loop.GRAD_OF.items():
        if g.get(key) is None:  # no such parameter, or a selection bias: no gradient on either side
            assert leaves.get(name) is None or leaves[name].grad is None, key
            continue
        auto = leaves[name].grad.numpy()
        assert np.allclose(g[key], auto, rtol=1e-10, atol=1e-12), f"{case} {key}"
