"""Pins of the fp64 oracle against things other than itself.

Each pin returns ``(ok, detail)``. They are run one by one by
``test_oracle_pins.py`` and all together, against an oracle with a planted
mistake, by ``test_oracle_mutations.py`` (every planted mistake must make at
least one pin fail).

Kinds of pin used:

* hand-derived worked examples with closed forms (``tests/golden/worked_examples.json``);
* brute force: an independent token-by-token restatement (``oracle.brute``);
* reductions to library routines: E=1/k=1 is a dense SwiGLU MLP and k=E with
  renormalised softmax is the dense softmax mixture (torch.nn.functional in
  fp64); score functions against scipy.special and mpmath;
* invariants: renormalised weights sum to 1, the permutation is a bijection,
  offsets are the prefix sum of counts, token permutation equivariance, exact
  power-of-two scaling, NaN-poisoned unrouted experts change nothing.
"""

from __future__ import annotations

import json
import math
import os
from typing import Callable, Dict, List, Tuple

import numpy as np
import torch
import torch.nn.functional as F

import oracle
import oracle.brute as brute
import oracle.moe as om
import workloads

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

Pin = Callable[[], Tuple[bool, str]]


def _np(t):
    return workloads.to_numpy64(t)


def tiny_problem(score: str, bias_mode: str, renormalize: bool, shared: str, *, T=5, H=12, E=6, k=2, I=6,
                 I_shared=4, seed=0, dtype="f32") -> Tuple[workloads.MoEConfig, Dict[str, np.ndarray]]:
    bias_kind = "none" if bias_mode == "none" else "uniform0.1"
    cfg = workloads.MoEConfig("tiny_pin", T, H, E, k, I, I_shared if shared != "none" else 0, dtype, score,
                              bias_mode, renormalize, shared, bias_kind=bias_kind, seed=seed)
    inp = workloads.generate(cfg, "cpu")
    a = {name: _np(v) for name, v in inp.items()}
    if bias_mode == "logit":
        a["bias"] = a["bias"] * 20.0  # large enough to change selections
    if bias_mode == "select":
        a["bias"] = a["bias"] * 5.0
    return cfg, a


def oracle_run(cfg, a, **kw):
    return oracle.moe_forward(a["x"], a["gate_w"], a["gate_up"], a["down"], k=cfg.k, score=cfg.score,
                              renormalize=cfg.renormalize, bias=a.get("bias"), bias_mode=cfg.bias_mode,
                              shared=cfg.shared, shared_gate_up=a.get("shared_gate_up"),
                              shared_down=a.get("shared_down"), shared_gate=a.get("shared_gate"), **kw)


def _rel(a, b) -> float:
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    den = max(np.abs(b).max(), 1e-300)
    return float(np.abs(a - b).max() / den)


def torch_swiglu(X, gu, dn) -> np.ndarray:
    """Dense SwiGLU MLP through torch.nn.functional in fp64 (library reduction)."""
    X, gu, dn = (torch.from_numpy(np.ascontiguousarray(v, dtype=np.float64)) for v in (X, gu, dn))
    I = gu.shape[0] // 2
    h = F.silu(F.linear(X, gu[:I])) * F.linear(X, gu[I:])
    return F.linear(h, dn).numpy()


# ----------------------------------------------------------------------------

BRUTE_CASES = []
for _score in ("softmax", "sigmoid", "sqrtsoftplus"):
    for _bias in ("none", "logit", "select"):
        for _renorm in (True, False):
            _shared = {"softmax": "plain", "sigmoid": "sigmoid_gated", "sqrtsoftplus": "none"}[_score]
            if _bias == "logit" and _score != "softmax":
                _shared = "none"
            BRUTE_CASES.append(dict(score=_score, bias_mode=_bias, renormalize=_renorm, shared=_shared))
BRUTE_CASES.append(dict(score="softmax", bias_mode="none", renormalize=True, shared="sigmoid_gated", k=1))
BRUTE_CASES.append(dict(score="softmax", bias_mode="none", renormalize=True, shared="none", k=6, E=6))
BRUTE_CASES.append(dict(score="sigmoid", bias_mode="select", renormalize=True, shared="plain", k=3, H=8, I=8))


def pin_brute_force() -> Tuple[bool, str]:
    worst = 0.0
    for i, c in enumerate(BRUTE_CASES):
        c = dict(c)
        cfg, a = tiny_problem(c.pop("score"), c.pop("bias_mode"), c.pop("renormalize"), c.pop("shared"),
                              seed=10 + i, **c)
        o = oracle_run(cfg, a)
        b = brute.brute_forward(a["x"].tolist(), a["gate_w"].tolist(), a["gate_up"].tolist(), a["down"].tolist(),
                                k=cfg.k, score=cfg.score, renormalize=cfg.renormalize,
                                bias=None if a.get("bias") is None else a["bias"].tolist(),
                                bias_mode=cfg.bias_mode, shared=cfg.shared,
                                shared_gate_up=None if a.get("shared_gate_up") is None else a["shared_gate_up"].tolist(),
                                shared_down=None if a.get("shared_down") is None else a["shared_down"].tolist(),
                                shared_gate=None if a.get("shared_gate") is None else a["shared_gate"].tolist())
        if not np.array_equal(o["selected_experts"], np.array(b["selected_experts"])):
            return False, f"case {i}: selection differs"
        ew = _rel(o["routing_weights"], b["routing_weights"])
        eo = _rel(o["out"], b["out"])
        worst = max(worst, ew, eo)
        if ew > 1e-12 or eo > 1e-12:
            return False, f"case {i}: weights rel {ew:.3g}, out rel {eo:.3g}"
        bd = brute.brute_dispatch(b["selected_experts"], cfg.E)
        for key in ("counts", "offsets", "sorted_pairs", "pair_pos"):
            if not np.array_equal(o[key], np.array(bd[key])):
                return False, f"case {i}: dispatch {key} differs"
    return True, f"{len(BRUTE_CASES)} cases, worst rel {worst:.2e}"


def _ev(s, names):
    return float(eval(str(s), {"__builtins__": {}}, names))


def pin_worked_examples() -> Tuple[bool, str]:
    names = {"ln2": math.log(2), "ln3": math.log(3), "ln4": math.log(4), "ln8": math.log(8),
             "sqrt2": math.sqrt(2)}
    with open(os.path.join(GOLDEN, "worked_examples.json")) as f:
        doc = json.load(f)

    def arr(v):
        if v is None:
            return None
        return np.vectorize(lambda s: _ev(s, names), otypes=[np.float64])(np.array(v, dtype=object))

    for c in doc["cases"]:
        o = oracle.moe_forward(arr(c["x"]), arr(c["gate_w"]), arr(c["gate_up"]), arr(c["down"]), k=c["k"],
                               score=c["score"], renormalize=c["renormalize"], bias=arr(c.get("bias")),
                               bias_mode=c["bias_mode"], shared=c["shared"],
                               shared_gate_up=arr(c.get("shared_gate_up")), shared_down=arr(c.get("shared_down")),
                               shared_gate=arr(c.get("shared_gate")))
        if not np.array_equal(o["selected_experts"], np.array(c["expect_selected"])):
            return False, f"{c['name']}: selected {o['selected_experts'].tolist()}"
        for key, exp in (("routing_weights", c["expect_weights"]), ("out", c["expect_out"])):
            e = arr(exp)
            err = np.abs(o[key] - e).max()
            if not err <= 1e-13:
                return False, f"{c['name']}: {key} err {err:.3g}"
    return True, f"{len(doc['cases'])} hand-derived cases"


def pin_dense_swiglu_E1() -> Tuple[bool, str]:
    for renorm, score in ((True, "sigmoid"), (False, "softmax"), (True, "sqrtsoftplus")):
        cfg, a = tiny_problem(score, "none", renorm, "none", E=1, k=1, seed=3, H=10, I=7)
        o = oracle_run(cfg, a)
        ref = torch_swiglu(a["x"], a["gate_up"][0], a["down"][0])
        if _rel(o["out"], ref) > 1e-13:
            return False, f"{score}/renorm={renorm}: {_rel(o['out'], ref):.3g}"
    return True, "E=1,k=1 equals torch dense SwiGLU"


def pin_softmax_renorm_closed_form() -> Tuple[bool, str]:
    from scipy.special import softmax as sp_softmax
    cfg, a = tiny_problem("softmax", "none", True, "none", T=9, E=6, k=3, seed=4)
    r = oracle.route(a["x"], a["gate_w"], cfg.k, "softmax", renormalize=True)
    L = a["x"] @ a["gate_w"].T
    for t in range(cfg.T):
        ref = sp_softmax(L[t, r["selected_experts"][t]])
        if np.abs(ref - r["routing_weights"][t]).max() > 1e-15:
            return False, f"token {t}"
    s = r["routing_weights"].sum(axis=1)
    if np.abs(s - 1).max() > 1e-15:
        return False, "renormalised weights do not sum to 1"
    return True, "equals softmax over the selected logits; sums to 1"


def pin_dense_mixture_k_eq_E() -> Tuple[bool, str]:
    from scipy.special import softmax as sp_softmax
    cfg, a = tiny_problem("softmax", "none", True, "none", T=4, E=5, k=5, seed=5, H=9, I=5)
    o = oracle_run(cfg, a)
    P = sp_softmax(a["x"] @ a["gate_w"].T, axis=1)
    ref = sum(P[:, e:e + 1] * torch_swiglu(a["x"], a["gate_up"][e], a["down"][e]) for e in range(cfg.E))
    err = _rel(o["out"], ref)
    return err < 1e-13, f"k=E dense softmax mixture rel {err:.2e}"


def pin_score_functions() -> Tuple[bool, str]:
    import mpmath
    from scipy.special import expit
    from scipy.special import softmax as sp_softmax
    pts = np.array([-40.0, -12.5, -3.0, -0.7, 0.0, 1e-3, 0.9, 4.0, 17.0, 35.0])
    if np.abs(oracle.scores(pts[None, :], "sigmoid")[0] - expit(pts)).max() > 1e-16:
        return False, "sigmoid vs scipy expit"
    mpmath.mp.dps = 50
    for p in pts:
        ref = float(mpmath.sqrt(mpmath.log(1 + mpmath.exp(mpmath.mpf(float(p))))))
        got = float(oracle.scores(np.array([[p]]), "sqrtsoftplus")[0, 0])
        if abs(got - ref) > 4e-16 * max(1.0, abs(ref)):
            return False, f"sqrtsoftplus({p}) {got} vs {ref}"
    L = np.array([[0.3, -1.2, 4.0, 4.0, -30.0], [700.0, 699.0, -700.0, 0.0, 1.0]])
    if np.abs(oracle.scores(L, "softmax") - sp_softmax(L, axis=1)).max() > 1e-15:
        return False, "softmax vs scipy"
    x = np.linspace(-30, 30, 61)
    silu_ref = x * expit(x)
    if np.abs(oracle.silu(x) - silu_ref).max() > 1e-14:
        return False, "silu"
    return True, "sigmoid/softmax vs scipy; sqrtsoftplus vs mpmath (50 digits); silu"


def pin_shared_gate_zero() -> Tuple[bool, str]:
    cfg, a = tiny_problem("sigmoid", "none", True, "sigmoid_gated", seed=6)
    a["shared_gate"] = np.zeros_like(a["shared_gate"])
    o = oracle_run(cfg, a)
    if not np.all(o["shared_gamma"] == 0.5):
        return False, "gamma != 0.5 at g = 0"
    base = oracle_run(cfg.replace(shared="none"), a)
    ref = base["out"] + 0.5 * torch_swiglu(a["x"], a["shared_gate_up"], a["shared_down"])
    err = _rel(o["out"], ref)
    return err < 1e-14, f"g=0 gives gamma=0.5; decomposition rel {err:.2e}"


def pin_shared_decomposition() -> Tuple[bool, str]:
    from scipy.special import expit
    for shared in ("plain", "sigmoid_gated"):
        cfg, a = tiny_problem("softmax", "none", True, shared, seed=7)
        o = oracle_run(cfg, a)
        base = oracle_run(cfg.replace(shared="none"), a)
        gam = 1.0 if shared == "plain" else expit(a["x"] @ a["shared_gate"])[:, None]
        ref = base["out"] + gam * torch_swiglu(a["x"], a["shared_gate_up"], a["shared_down"])
        if _rel(o["out"], ref) > 1e-14:
            return False, shared
        if np.abs(o["routed_out"] - base["out"]).max() != 0.0:
            return False, "routed part changed by the shared expert"
    return True, "out = routed + gamma * shared (plain and gated)"


def pin_empty_expert_poison() -> Tuple[bool, str]:
    cfg, a = tiny_problem("softmax", "none", True, "none", T=6, E=6, k=2, seed=8)
    o = oracle_run(cfg, a)
    unused = [e for e in range(cfg.E) if o["counts"][e] == 0]
    if not unused:
        a["gate_w"][5] -= 50.0  # make expert 5 unattractive
        o = oracle_run(cfg, a)
        unused = [e for e in range(cfg.E) if o["counts"][e] == 0]
    if not unused:
        return False, "no empty expert to poison"
    a2 = {kk: (v.copy() if isinstance(v, np.ndarray) else v) for kk, v in a.items()}
    for e in unused:
        a2["gate_up"][e][:] = np.nan
        a2["down"][e][:] = np.nan
    o2 = oracle_run(cfg, a2)
    o3 = oracle_run(cfg, a2, skip_unrouted=True)
    ok = np.isfinite(o2["out"]).all() and np.array_equal(o2["out"], o["out"]) and np.array_equal(o3["out"], o["out"])
    return bool(ok), f"experts {unused} poisoned with NaN"


def pin_dispatch_invariants() -> Tuple[bool, str]:
    rng = np.random.RandomState(9)
    for T, E, k in ((1, 1, 1), (7, 5, 2), (33, 8, 8), (50, 16, 3), (0, 4, 2)):
        sel = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]) if T else np.zeros((0, k), np.int64)
        d = oracle.dispatch(sel, E)
        P = T * k
        if d["counts"].sum() != P or not np.array_equal(d["offsets"][1:], np.cumsum(d["counts"])) or d["offsets"][0]:
            return False, "counts/offsets"
        if not np.array_equal(np.sort(d["sorted_pairs"]), np.arange(P)):
            return False, "not a bijection"
        if not np.array_equal(d["sorted_pairs"][d["pair_pos"]], np.arange(P)):
            return False, "pair_pos is not the inverse"
        flat = sel.reshape(-1)
        for e in range(E):
            seg = d["sorted_pairs"][d["offsets"][e]:d["offsets"][e + 1]]
            if not (np.all(flat[seg] == e) and np.all(np.diff(seg) > 0)):
                return False, f"segment {e}"
        bd = brute.brute_dispatch(sel.tolist(), E)
        for key in ("counts", "offsets", "sorted_pairs", "pair_pos"):
            if not np.array_equal(d[key], np.array(bd[key], dtype=np.int64).reshape(d[key].shape)):
                return False, f"{key} vs brute bucket sort"
    return True, "bijection, inverse, prefix sums, ascending segments, brute bucket sort"


def pin_token_permutation() -> Tuple[bool, str]:
    cfg, a = tiny_problem("sqrtsoftplus", "select", True, "plain", T=7, seed=11)
    o = oracle_run(cfg, a)
    perm = np.random.RandomState(0).permutation(cfg.T)
    a2 = dict(a)
    a2["x"] = a["x"][perm]
    o2 = oracle_run(cfg, a2)
    ok = np.array_equal(o2["selected_experts"], o["selected_experts"][perm]) and \
        _rel(o2["out"], o["out"][perm]) < 1e-15
    return bool(ok), "permuting tokens permutes outputs"


def pin_down_scaling_exact() -> Tuple[bool, str]:
    cfg, a = tiny_problem("softmax", "logit", False, "plain", seed=12)
    o = oracle_run(cfg, a)
    a2 = dict(a)
    a2["down"] = a["down"] * 2.0
    a2["shared_down"] = a["shared_down"] * 2.0
    o2 = oracle_run(cfg, a2)
    return bool(np.array_equal(o2["out"], 2.0 * o["out"])), "doubling down doubles out exactly"


def pin_selected_override_identity() -> Tuple[bool, str]:
    cfg, a = tiny_problem("sigmoid", "select", True, "sigmoid_gated", seed=13)
    o = oracle_run(cfg, a)
    o2 = oracle_run(cfg, a, selected=o["selected_experts"])
    return bool(np.array_equal(o["out"], o2["out"])), "forcing the oracle's own selection changes nothing"


def pin_bias_modes() -> Tuple[bool, str]:
    """A logit bias shifts softmax probabilities; a selection bias never enters weights."""
    from scipy.special import softmax as sp_softmax
    cfg, a = tiny_problem("softmax", "logit", True, "none", T=6, seed=14)
    r = oracle.route(a["x"], a["gate_w"], cfg.k, "softmax", bias=a["bias"], bias_mode="logit", renormalize=False)
    P = sp_softmax(a["x"] @ a["gate_w"].T + a["bias"][None, :], axis=1)
    if np.abs(np.take_along_axis(P, r["selected_experts"], 1) - r["routing_weights"]).max() > 1e-15:
        return False, "logit bias"
    cfg, a = tiny_problem("sqrtsoftplus", "select", False, "none", T=6, seed=15)
    r = oracle.route(a["x"], a["gate_w"], cfg.k, "sqrtsoftplus", bias=a["bias"], bias_mode="select",
                     renormalize=False)
    S = np.sqrt(np.logaddexp(0.0, a["x"] @ a["gate_w"].T))
    if np.abs(np.take_along_axis(S, r["selected_experts"], 1) - r["routing_weights"]).max() > 1e-15:
        return False, "selection bias leaked into weights"
    Kref = S + a["bias"][None, :]
    for t in range(cfg.T):
        chosen = sorted(range(cfg.E), key=lambda e: (-Kref[t, e], e))[:cfg.k]
        if list(r["selected_experts"][t]) != chosen:
            return False, f"token {t} selection"
    return True, "logit bias enters softmax; selection bias only ranks"


PINS: Dict[str, Pin] = {
    "brute_force": pin_brute_force,
    "worked_examples": pin_worked_examples,
    "dense_swiglu_E1": pin_dense_swiglu_E1,
    "softmax_renorm_closed_form": pin_softmax_renorm_closed_form,
    "dense_mixture_k_eq_E": pin_dense_mixture_k_eq_E,
    "score_functions": pin_score_functions,
    "shared_gate_zero": pin_shared_gate_zero,
    "shared_decomposition": pin_shared_decomposition,
    "empty_expert_poison": pin_empty_expert_poison,
    "dispatch_invariants": pin_dispatch_invariants,
    "token_permutation": pin_token_permutation,
    "down_scaling_exact": pin_down_scaling_exact,
    "selected_override_identity": pin_selected_override_identity,
    "bias_modes": pin_bias_modes,
}


def run_all() -> Dict[str, Tuple[bool, str]]:
    res = {}
    for name, fn in PINS.items():
        try:
            res[name] = fn()
        except Exception as exc:  # a planted mistake may also raise
            res[name] = (False, f"raised {type(exc).__name__}: {exc}")
    return res


def failing(results: Dict[str, Tuple[bool, str]]) -> List[str]:
    return [n for n, (ok, _) in results.items() if not ok]


def first_failure():
    """Name and detail of the first pin that fails, or None."""
    for name, fn in PINS.items():
        try:
            ok, detail = fn()
        except Exception as exc:
            ok, detail = False, f"raised {type(exc).__name__}: {exc}"
        if not ok:
            return name, detail
    return None
