"""Negative tests: each mistake planted in the oracle (on the CPU, through
monkeypatch) must make at least one pin fail. This is the "each guard against
the defect it claims to catch" practice of "MoE: shared experts, parameterized
V_TOPK routing, explicit stage attribution" (3. Tests, Negative-tested),
applied to the oracle's own pins.
"""

import numpy as np
import pytest

import oracle.moe as om
import oracle_pins

_orig = {name: getattr(om, name) for name in (
    "gate_half", "up_half", "silu", "topk_weights", "select_topk", "selection_keys", "shared_gate_values",
    "dispatch", "scores", "router_logits", "sigmoid", "swiglu_mlp", "softplus", "routing_matrix")}


def _swap_gate_up_gate(w, I):
    return _orig["up_half"](w, I)


def _swap_gate_up_up(w, I):
    return _orig["gate_half"](w, I)


def _select_reverse_ties(K, k):
    K = np.asarray(K, np.float64)
    E = K.shape[1]
    rev = np.argsort(-K[:, ::-1], axis=1, kind="stable")
    return (E - 1 - rev)[:, :k].astype(np.int64)


def _dispatch_unstable(selected, E):
    d = _orig["dispatch"](selected, E)
    sp = d["sorted_pairs"].copy()
    for e in range(E):
        a, b = d["offsets"][e], d["offsets"][e + 1]
        sp[a:b] = sp[a:b][::-1]
    pos = np.empty_like(sp)
    pos[sp] = np.arange(sp.size)
    d.update(sorted_pairs=sp, pair_pos=pos)
    return d


def _dispatch_inclusive(selected, E):
    d = _orig["dispatch"](selected, E)
    d["offsets"] = np.concatenate([np.cumsum(d["counts"]), [d["counts"].sum()]])
    return d


def _dispatch_pos_not_inverse(selected, E):
    d = _orig["dispatch"](selected, E)
    d["pair_pos"] = d["sorted_pairs"].copy()
    return d


def _scores_sqrt_dropped(L, kind):
    if kind == "sqrtsoftplus":
        return om.softplus(L)
    return _orig["scores"](L, kind)


def _routing_matrix_dense(weights, selected, E):
    M, mask = _orig["routing_matrix"](weights, selected, E)
    return M, np.ones_like(mask)


def _swiglu_no_gate_act(X, w_gate_up, w_down):
    w_gate_up = np.asarray(w_gate_up, np.float64)
    I = w_gate_up.shape[0] // 2
    X = np.asarray(X, np.float64)
    return ((X @ w_gate_up[:I].T) * (X @ w_gate_up[I:].T)) @ np.asarray(w_down, np.float64).T


def _swiglu_down_transposed(X, w_gate_up, w_down):
    w_gate_up = np.asarray(w_gate_up, np.float64)
    I = w_gate_up.shape[0] // 2
    X = np.asarray(X, np.float64)
    h = om.silu(X @ w_gate_up[:I].T) * (X @ w_gate_up[I:].T)
    wd = np.asarray(w_down, np.float64)
    return h @ wd.reshape(wd.shape[1], wd.shape[0])


MUTATIONS = {
    "gate_up_halves_swapped": [("gate_half", _swap_gate_up_gate), ("up_half", _swap_gate_up_up)],
    "silu_is_identity": [("silu", lambda a: np.asarray(a, np.float64))],
    "silu_wrong_sign": [("silu", lambda a: np.asarray(a, np.float64) * _orig["sigmoid"](-np.asarray(a, np.float64)))],
    "swiglu_without_activation": [("swiglu_mlp", _swiglu_no_gate_act)],
    "down_operand_transposed": [("swiglu_mlp", _swiglu_down_transposed)],
    "renorm_dropped": [("topk_weights", lambda S, sel, r: _orig["topk_weights"](S, sel, False))],
    "renorm_always": [("topk_weights", lambda S, sel, r: _orig["topk_weights"](S, sel, True))],
    "ties_to_higher_index": [("select_topk", _select_reverse_ties)],
    "select_smallest": [("select_topk", lambda K, k: _orig["select_topk"](-np.asarray(K, np.float64), k))],
    "selection_bias_ignored": [("selection_keys", lambda S, b=None, m="none": np.asarray(S, np.float64))],
    "selection_bias_subtracted": [("selection_keys", lambda S, b=None, m="none": _orig["selection_keys"](
        S, None if b is None else -np.asarray(b, np.float64), m))],
    "logit_bias_dropped": [("router_logits", lambda x, w, b=None, m="none": _orig["router_logits"](x, w))],
    "shared_gate_dropped": [("shared_gate_values", lambda x, g, s: np.ones(np.asarray(x).shape[0]))],
    "shared_gate_sign": [("shared_gate_values", lambda x, g, s: _orig["shared_gate_values"](
        x, None if g is None else -np.asarray(g, np.float64), s))],
    "dispatch_unstable": [("dispatch", _dispatch_unstable)],
    "offsets_inclusive": [("dispatch", _dispatch_inclusive)],
    "pair_pos_not_inverse": [("dispatch", _dispatch_pos_not_inverse)],
    "sqrt_dropped": [("scores", _scores_sqrt_dropped)],
    "sigmoid_sign": [("sigmoid", lambda a: _orig["sigmoid"](-np.asarray(a, np.float64)))],
    "unmasked_experts": [("routing_matrix", _routing_matrix_dense)],
}


@pytest.mark.parametrize("name", list(MUTATIONS))
def test_planted_mistake_is_caught(name, monkeypatch):
    for attr, fn in MUTATIONS[name]:
        monkeypatch.setattr(om, attr, fn)
    caught = oracle_pins.first_failure()
    assert caught is not None, f"planted mistake '{name}' passed every pin"
