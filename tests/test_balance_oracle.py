"""Pins of the balancer oracle (oracle/balance.py) against things other than
itself, and planted mistakes that each pin set must catch. CPU only."""

from __future__ import annotations

import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle.balance as ob
import oracle.moe as om

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "bias_update_examples.json")


def brute_update(bias, loads, rate):
    """Independent restatement: exact rational mean, numpy fp32 addition."""
    E = len(loads)
    mean = Fraction(int(sum(int(v) for v in loads)), E)
    r = np.float32(rate)
    out = []
    for b, v in zip(bias, loads):
        b = np.float32(b)
        if Fraction(int(v)) < mean:
            out.append(np.float32(b + r))
        elif Fraction(int(v)) > mean:
            out.append(np.float32(b - r))
        else:
            out.append(b)
    return np.array(out, dtype=np.float32)


def pin_worked_examples(update=ob.bias_update):
    """Hand-worked cases in tests/golden/bias_update_examples.json."""
    for case in json.load(open(GOLDEN))["cases"]:
        got, cleared = update(np.array(case["bias"], np.float32), np.array(case["loads"]), case["rate"])
        want = np.array(case["expect"], np.float32)
        if not np.array_equal(got, want) or np.any(cleared != 0):
            return False, f"{case['name']}: {got.tolist()} != {want.tolist()}"
    return True, ""


def pin_brute_force(update=ob.bias_update):
    rng = np.random.default_rng(11)
    for E in (1, 2, 5, 8, 64, 256):
        for _ in range(20):
            if rng.random() < 0.5:
                loads = rng.integers(0, 50, size=E)
            else:  # pairs c - d, c + d around c = 20 (d = 0 sits exactly at the mean)
                d = rng.integers(0, 3, size=E // 2) * rng.integers(0, 15, size=E // 2)
                loads = np.concatenate([20 - d, 20 + d, [20] * (E % 2)]).astype(np.int64)
            bias = rng.normal(0, 0.3, size=E).astype(np.float32)
            rate = float(rng.choice([1e-3, 0.05, 0.5]))
            got, _ = update(bias, loads, rate)
            want = brute_update(bias, loads, rate)
            if not np.array_equal(got, want):
                return False, f"E={E}: {got[:4]} vs {want[:4]}"
    return True, ""


def pin_balanced_loads_keep_bias(update=ob.bias_update):
    bias = np.linspace(-1, 1, 16).astype(np.float32)
    got, _ = update(bias, np.full(16, 123), 0.01)
    return bool(np.array_equal(got, bias)), "balanced loads moved the bias"


def pin_second_apply_is_noop(update=ob.bias_update):
    """The page's balance-update semantics: apply, then apply again with
    what is left in the stash: the bias changes once."""
    bias = np.zeros(6, np.float32)
    loads = np.array([9, 1, 3, 3, 2, 0])
    b1, left = update(bias, loads, 0.25)
    b2, _ = update(b1, left, 0.25)
    return bool(np.array_equal(b1, b2) and not np.array_equal(b1, bias)), f"{b1} / {b2}"


def pin_controller_balances_routing(update=ob.bias_update):
    """Closed-loop property: with fixed router logits skewed toward a few
    experts, repeated (route with the selection bias, stash counts, update)
    steps shrink the max/mean load ratio, as a balancing controller must."""
    rng = np.random.default_rng(5)
    T, E, k = 512, 16, 2
    logits = rng.normal(size=(T, E)) + np.linspace(2.0, 0.0, E)[None, :]
    scores = 1.0 / (1.0 + np.exp(-logits))
    bias = np.zeros(E, np.float32)

    def ratio(b):
        sel = om.select_topk(scores + b.astype(np.float64)[None, :], k)
        load = np.bincount(sel.ravel(), minlength=E)
        return load.max() / load.mean(), load

    r0, _ = ratio(bias)
    stash = np.zeros(E, np.int64)
    for _ in range(300):
        _, load = ratio(bias)
        stash = ob.stash_counts(stash, load)
        bias, stash = update(bias, stash, 0.01)
    r1, _ = ratio(bias)
    return bool(r0 > 2.0 and r1 < 1.5), f"max/mean load {r0:.2f} -> {r1:.2f}"


def pin_stash_sums_counts(stash_fn=ob.stash_counts):
    s = np.zeros(4, np.int64)
    for c in ([1, 2, 3, 4], [0, 0, 5, 1], [2, 2, 2, 2]):
        s = stash_fn(s, np.array(c, np.int32))
    return bool(np.array_equal(s, [3, 4, 10, 7])), f"{s}"


UPDATE_PINS = [pin_worked_examples, pin_brute_force, pin_balanced_loads_keep_bias, pin_second_apply_is_noop,
               pin_controller_balances_routing]


@pytest.mark.parametrize("pin", UPDATE_PINS + [pin_stash_sums_counts], ids=lambda f: f.__name__)
def test_balance_pin(pin):
    ok, detail = pin()
    assert ok, detail


# ---- planted mistakes: each must fail at least one pin -------------------

def _flipped_sign(bias, loads, rate):
    b, z = ob.bias_update(bias, loads, rate)
    return (2 * np.asarray(bias, np.float32) - b).astype(np.float32), z


def _moves_at_mean(bias, loads, rate):
    L = np.asarray(loads, np.int64)
    b = np.asarray(bias, np.float32).astype(np.float64)
    up = L.sum() >= len(L) * L
    return np.where(up, b + np.float32(rate), b - np.float32(rate)).astype(np.float32), np.zeros_like(L)


def _keeps_stash(bias, loads, rate):
    b, _ = ob.bias_update(bias, loads, rate)
    return b, np.asarray(loads, np.int64)


def _step_proportional(bias, loads, rate):
    L = np.asarray(loads, np.int64)
    b = np.asarray(bias, np.float32).astype(np.float64)
    return (b + np.float32(rate) * (L.mean() - L)).astype(np.float32), np.zeros_like(L)


def _mean_of_nonzero(bias, loads, rate):
    L = np.asarray(loads, np.int64)
    live = L > 0
    m = L[live].mean() if live.any() else 0.0
    b = np.asarray(bias, np.float32).astype(np.float64)
    return (b + np.float32(rate) * np.sign(m - L)).astype(np.float32), np.zeros_like(L)


@pytest.mark.parametrize("mutant", [_flipped_sign, _moves_at_mean, _keeps_stash, _step_proportional, _mean_of_nonzero],
                         ids=lambda f: f.__name__)
def test_planted_update_mistake_is_caught(mutant):
    failures = [p.__name__ for p in UPDATE_PINS if not p(update=mutant)[0]]
    assert failures, f"no pin caught {mutant.__name__}"


def test_planted_stash_mistake_is_caught():
    assert not pin_stash_sums_counts(stash_fn=lambda s, c: np.asarray(c, np.int64))[0]
