"""Seeded inputs: determinism, shapes, and the stored Zipf logit bias."""

import json

import numpy as np
import torch
import pytest

import oracle
import workloads


def test_configs_shapes():
    c = workloads.CONFIGS
    assert [c[n].T for n in workloads.CONFIG_ORDER] == [256, 4096, 8192, 8192, 16]
    assert c["deepseek_v2_lite_zipf"].I_shared == 2816 and c["dsv4_flash_ablation"].I_shared == 2048
    assert c["decode_weight_streaming"].shared == "sigmoid_gated"


def test_generation_is_deterministic():
    cfg = workloads.CONFIGS["tiny_fp32"].replace(T=16, H=32, I=16)
    a = workloads.generate(cfg, "cpu")
    b = workloads.generate(cfg, "cpu")
    for key in a:
        if a[key] is None:
            assert b[key] is None
        else:
            assert a[key].dtype == b[key].dtype and bool((a[key] == b[key]).all())
    assert a["x"].shape == (16, 32) and a["gate_up"].shape == (8, 32, 32) and a["down"].shape == (8, 32, 16)


def test_bf16_rounding_and_std():
    cfg = workloads.CONFIGS["qwen3_30b_a3b"].replace(T=64, E=4)
    a = workloads.generate(cfg, "cpu")
    import torch
    assert a["x"].dtype == torch.bfloat16
    g = a["gate_w"].float()
    assert abs(g.std().item() * cfg.H ** 0.5 - 1.0) < 0.05


@pytest.mark.slow
def test_stored_zipf_bias_reproduces_loads():
    """The stored fp32 bias, pushed through the oracle's router on the seeded
    inputs, gives the stored loads (4 dead experts, one saturated expert)."""
    cfg = workloads.CONFIGS["deepseek_v2_lite_zipf"]
    with open(workloads.ZIPF_BIAS_FILE) as f:
        d = json.load(f)
    r = workloads.router_inputs(cfg)
    res = oracle.route(workloads.to_numpy64(r["x"]), workloads.to_numpy64(r["gate_w"]), cfg.k, "softmax",
                       bias=workloads.to_numpy64(r["bias"]), bias_mode="logit", renormalize=False)
    counts = np.bincount(res["selected_experts"].reshape(-1), minlength=cfg.E)
    assert counts.tolist() == d["realised_loads_fp64_oracle"]
    assert sorted(np.nonzero(counts == 0)[0].tolist()) == d["dead_experts"]
    assert counts.max() == cfg.T and counts.sum() == cfg.T * cfg.k


def test_oracle_rows_are_independent():
    """Sampled full-size parity evaluates the oracle on a subset of tokens; a
    token's result must not depend on which other tokens are present."""
    cfg = workloads.CONFIGS["dsv4_flash_ablation"].replace(T=12, H=24, E=8, I=16, I_shared=8)
    a = {k: workloads.to_numpy64(v) for k, v in workloads.generate(cfg, "cpu").items()}
    kw = dict(k=cfg.k, score=cfg.score, renormalize=cfg.renormalize, bias=a["bias"], bias_mode=cfg.bias_mode,
              shared=cfg.shared, shared_gate_up=a["shared_gate_up"], shared_down=a["shared_down"])
    full = oracle.moe_forward(a["x"], a["gate_w"], a["gate_up"], a["down"], **kw)
    rows = [0, 5, 11]
    part = oracle.moe_forward(a["x"][rows], a["gate_w"], a["gate_up"], a["down"], skip_unrouted=True, **kw)
    assert np.array_equal(part["selected_experts"], full["selected_experts"][rows])
    assert np.abs(part["out"] - full["out"][rows]).max() <= 1e-13 * np.abs(full["out"]).max()


def test_decode_shared_gate_is_not_saturated():
    """The sigmoid shared-expert gate of the decode problem must stay away from
    saturation (|x . g| < 15 on every token, and spread out), so that a gate
    that is dropped or applied twice changes the output visibly."""
    cfg = workloads.CONFIGS["decode_weight_streaming"]
    r = workloads.router_inputs(cfg)
    z = r["x"].double() @ r["shared_gate"].double()
    assert z.abs().max().item() < 15
    gamma = torch.sigmoid(z)
    assert gamma.std().item() > 0.05 and (gamma - 0.5).abs().max().item() > 0.1
