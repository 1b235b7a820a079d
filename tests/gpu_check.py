"""Comparison helpers for the GPU parity tests (CUDA path vs fp64 oracle).

Tolerances:
* bf16 problems: relative L2 <= 5e-3 and max-abs <= 3e-2 * rms(reference);
* fp32 problems: relative L2 <= 1e-5 and max-abs <= 1e-5 * max|reference|;
* routing weights and shared gate values (fp32): max-abs <= 1e-5;
* indices, counts, offsets and permutations: bit-exact.

Near ties. The CUDA router accumulates logits in fp32 while the oracle works
in fp64. Each bf16 x bf16 product is exact in fp32, so the logit error is the
rounding of an H-term fp32 sum (plus at most 16 split partials added in
order): every addition rounds by at most u = 2^-24 of the running sum, and
those roundings are independent in sign, so the error behaves like a random
walk of sqrt(H) steps of size u * |running sum|. With H <= 7168 and running
sums of a few units (the logits here are ~N(0,1), |l| <= ~5), that is about
85 * 6e-8 * 2 ~ 1e-5 at the very worst token of a batch and ~1e-6 typically;
scores and keys add a few fp32 ulps, and adding a logit bias rounds once more
at the key's own magnitude. Hence the tie margin of the survey's reading,
TAU * max(1, |key|) with TAU = 1e-5, where |key| is the larger magnitude of
the token's k-th and (k+1)-th oracle keys (the keys at the decision, not the
token's largest key: a dead expert's -1e4 logit bias must not widen the
margin). On a token whose oracle margin between those two keys is below it,
more than one top-k set is correct: the CUDA choice passes if it is one of
them (every chosen key >= every unchosen key - tau, slot order descending
within tau), and the reference output is recomputed from the CUDA choice.
Every test asserts how many tokens took this escape (EXPECTED_NEAR_TIES; 0
unless listed), so a router that mis-ordered keys inside the margin would
change the count and fail.
"""

from __future__ import annotations

from typing import Dict

import numpy as np
import torch

import oracle
import workloads

TAU = 1e-5

# Tokens whose CUDA top-k differs from the oracle's inside the tie margin, at
# the fixed seeds (problem name -> count). Every other problem: 0.
# The Zipf-skewed problem at full size has 26 tokens whose oracle margin is
# below 1e-5 (the smallest 1.1e-7); the CUDA router's fp32 logits order four
# of them the other way.
EXPECTED_NEAR_TIES = {"deepseek_v2_lite_zipf": 4}


def expected_near_ties(name: str) -> int:
    return EXPECTED_NEAR_TIES.get(name, 0)


class LazyExperts:
    """Indexable view of a stacked [E, ...] device tensor for the oracle: each
    expert slab is copied to the host and widened to fp64 when asked for."""

    def __init__(self, t: torch.Tensor):
        self.t = t

    def __len__(self) -> int:
        return self.t.shape[0]

    def __getitem__(self, e: int) -> np.ndarray:
        return self.t[e].to("cpu").to(torch.float64).numpy()


def np64(t):
    return workloads.to_numpy64(t)


def oracle_kwargs(cfg, inp, lazy: bool = False) -> Dict:
    conv = (lambda t: None if t is None else LazyExperts(t)) if lazy else np64
    return dict(k=cfg.k, score=cfg.score, renormalize=cfg.renormalize, bias=np64(inp.get("bias")),
                bias_mode=cfg.bias_mode, shared=cfg.shared,
                shared_gate_up=np64(inp.get("shared_gate_up")), shared_down=np64(inp.get("shared_down")),
                shared_gate=np64(inp.get("shared_gate")),
                _gate_up=conv(inp["gate_up"]), _down=conv(inp["down"]))


def oracle_forward(cfg, inp, x_rows=None, selected=None, lazy=False, skip_unrouted=False):
    kw = oracle_kwargs(cfg, inp, lazy)
    gu, dn = kw.pop("_gate_up"), kw.pop("_down")
    x = np64(inp["x"]) if x_rows is None else x_rows
    return oracle.moe_forward(x, np64(inp["gate_w"]), gu, dn, selected=selected, skip_unrouted=skip_unrouted, **kw)


def oracle_route(cfg, inp):
    return oracle.route(np64(inp["x"]), np64(inp["gate_w"]), cfg.k, cfg.score, bias=np64(inp.get("bias")),
                        bias_mode=cfg.bias_mode, renormalize=cfg.renormalize)


def ranking_keys(cfg, r) -> np.ndarray:
    """The keys the CUDA router ranks by: the logits (every score function is
    increasing) unless a selection bias is added to the scores."""
    return r["keys"] if cfg.bias_mode == "select" else r["logits"]


def tie_margin(K_t: np.ndarray, k: int) -> float:
    """TAU * max(1, |k-th key|, |(k+1)-th key|) for one token's oracle keys."""
    s = np.sort(K_t)[::-1]
    mag = abs(float(s[k - 1])) if k >= len(s) else max(abs(float(s[k - 1])), abs(float(s[k])))
    return TAU * max(1.0, mag)


def check_selection(cfg, r, gpu_sel: np.ndarray) -> int:
    """Assert the CUDA top-k is exact except at near ties, where it must be a
    correct alternative. Returns the number of tokens that differ."""
    ref = r["selected_experts"]
    assert gpu_sel.shape == ref.shape
    K = ranking_keys(cfg, r)
    diff = np.nonzero((gpu_sel != ref).any(axis=1))[0]
    for t in diff:
        g = gpu_sel[t]
        assert len(set(g.tolist())) == cfg.k, f"token {t}: repeated expert {g}"
        assert g.min() >= 0 and g.max() < cfg.E
        tau = tie_margin(K[t], cfg.k)
        chosen = K[t, g]
        mask = np.ones(cfg.E, bool)
        mask[g] = False
        if mask.any():
            assert chosen.min() >= K[t, mask].max() - tau, \
                f"token {t}: gpu {g} vs oracle {ref[t]} beyond the tie margin"
        assert np.all(np.diff(chosen) <= tau), f"token {t}: slot order {g}"
    return int(diff.size)


def rel_l2(got, ref) -> float:
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


def assert_close(got, ref, dtype: str, what: str = "") -> Dict[str, float]:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - ref)
    rl = rel_l2(got, ref)
    if dtype == "bf16":
        rms = float(np.sqrt(np.mean(ref ** 2)))
        assert rl <= 5e-3, f"{what}: rel L2 {rl:.3e} > 5e-3"
        assert err.max() <= 3e-2 * rms, f"{what}: max abs {err.max():.3e} > 3e-2 * rms {rms:.3e}"
    else:
        assert rl <= 1e-5, f"{what}: rel L2 {rl:.3e} > 1e-5"
        assert err.max() <= 1e-5 * np.abs(ref).max(), f"{what}: max abs {err.max():.3e}"
    return {"rel_l2": rl, "max_abs": float(err.max())}


def assert_within_bound(got, ref, bound, what: str = "") -> float:
    """Elementwise |got - ref| <= bound (a bound derived from the arithmetic),
    plus relative L2 <= 5e-3. Returns max(err / bound)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(got - ref)
    assert np.isfinite(got).all(), f"{what}: non-finite"
    ratio = float((err / np.maximum(bound, 1e-300)).max())
    assert ratio <= 1.0, f"{what}: error exceeds its rounding bound by x{ratio:.3f}"
    assert rel_l2(got, ref) <= 5e-3, f"{what}: rel L2 {rel_l2(got, ref):.3e}"
    return ratio


def swiglu_with_bound(X, gu, dn, scale, dtype: str):
    """Oracle SwiGLU rows times ``scale`` and a bound on the CUDA result's error.

    On the bf16 path h is rounded to bf16 once (relative error <= 2^-9) before
    the down GEMM; the fp32 accumulations add far less than another 2^-9. So
    |y_cuda - y| <= 2^-8 * scale * (|h| . |W_d|^T). On the fp32 path the bound
    is 1e-5 * scale * (|h| . |W_d|^T)."""
    I = gu.shape[0] // 2
    h = oracle.silu(X @ gu[:I].T) * (X @ gu[I:].T)
    y = scale[:, None] * (h @ dn.T)
    mag = np.abs(scale)[:, None] * (np.abs(h) @ np.abs(dn).T)
    return y, mag * (2.0 ** -8 if dtype == "bf16" else 1e-5)


def assert_dispatch_exact(gpu: Dict[str, torch.Tensor], sel: np.ndarray, E: int) -> Dict[str, np.ndarray]:
    d = oracle.dispatch(sel, E)
    for key in ("counts", "offsets", "sorted_pairs", "pair_pos"):
        got = gpu[key].cpu().numpy().astype(np.int64)
        assert np.array_equal(got, d[key]), f"dispatch {key} differs"
    return d
