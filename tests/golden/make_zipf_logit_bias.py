"""Write ``zipf_logit_bias_E64.json``: the router logit bias of the skewed
DeepSeek-V2-Lite-shaped problem (T=8192, H=2048, E=64, top-6 softmax).

The bias is calibrated with the sign controller of the aux-loss-free balancer
("Sparse MoE FFN for DFlash-family drafters", What's here, MoEGate: the bias is
moved by a sign controller from expert loads, never by gradients), steered
here towards Zipf(s=1.2) target loads instead of uniform ones:

* 60 live experts get target loads proportional to rank**-1.2, water-filled
  under the cap T (an expert is picked at most once per token), summing to
  T*k; 4 dead experts get bias -1e4 and so receive no tokens;
* expert ids are a seeded permutation of the ranks;
* b <- b + step * sign(target - load), with a step decaying from 0.05 to 1e-3.

Router logits come from the fp64 oracle on the seeded inputs. The stored bias
is rounded to fp32 (the dtype the router takes). The realised loads, recomputed
by the oracle with the fp32 bias, are stored beside it. Run from the repo root:

    python tests/golden/make_zipf_logit_bias.py
"""

from __future__ import annotations

import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import workloads  # noqa: E402

N_DEAD = 4
ZIPF_S = 1.2
DEAD_BIAS = -1.0e4


def water_filled_targets(n_live: int, total: int, cap: int, s: float) -> np.ndarray:
    w = np.arange(1, n_live + 1, dtype=np.float64) ** -s
    tgt = np.zeros(n_live)
    capped = np.zeros(n_live, dtype=bool)
    while True:
        rem = total - cap * capped.sum()
        free = ~capped
        tgt[free] = rem * w[free] / w[free].sum()
        tgt[capped] = cap
        newly = free & (tgt > cap)
        if not newly.any():
            return tgt
        capped |= newly


def main() -> None:
    cfg = workloads.CONFIGS["deepseek_v2_lite_zipf"].replace(bias_kind="none")
    r = workloads.router_inputs(cfg)
    x = workloads.to_numpy64(r["x"])
    gw = workloads.to_numpy64(r["gate_w"])
    L = oracle.router_logits(x, gw)
    T, E, k = cfg.T, cfg.E, cfg.k

    rng = np.random.RandomState(1234 + cfg.seed)
    perm = rng.permutation(E)
    live, dead = perm[:E - N_DEAD], perm[E - N_DEAD:]
    tgt_rank = water_filled_targets(E - N_DEAD, T * k, T, ZIPF_S)
    target = np.zeros(E)
    target[live] = tgt_rank

    b = np.zeros(E)
    b[dead] = DEAD_BIAS
    steps = 3000
    for i in range(steps):
        step = max(1e-3, 0.05 * (0.998 ** i))
        Z = L + b[None, :]
        sel = np.argpartition(-Z, k - 1, axis=1)[:, :k]
        load = np.bincount(sel.reshape(-1), minlength=E)
        b[live] += step * np.sign(target[live] - load[live])

    b32 = b.astype(np.float32)
    res = oracle.route(x, gw, k, oracle.SOFTMAX, bias=b32.astype(np.float64), bias_mode=oracle.BIAS_LOGIT,
                       renormalize=False)
    counts = np.bincount(res["selected_experts"].reshape(-1), minlength=E)
    margins = oracle.decision_margins(res["logits"], k)
    out = {
        "what": "router logit bias, DeepSeek-V2-Lite-shaped skewed problem (T=8192, H=2048, E=64, top-6 softmax)",
        "E": E, "T": T, "k": k, "seed": cfg.seed, "zipf_s": ZIPF_S, "dead_experts": sorted(int(d) for d in dead),
        "bias_fp32": [float(v) for v in b32],
        "target_loads": [float(v) for v in target],
        "realised_loads_fp64_oracle": [int(c) for c in counts],
        "min_logit_decision_margin": float(margins.min()),
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "zipf_logit_bias_E64.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    order = np.argsort(-counts)
    print("loads (sorted):", counts[order][:12], "...", counts[order][-8:])
    print("targets (sorted):", np.round(np.sort(target)[::-1][:12]))
    print("min margin", margins.min(), "sum", counts.sum())


if __name__ == "__main__":
    main()
