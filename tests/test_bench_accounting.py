"""The bench's work accounting (CPU): the algorithmic FLOPs and bytes that
the roofline figures divide by, recounted here contraction by contraction
from the shapes, for every named problem."""

import pytest

import bench
import workloads
from workloads import CONFIGS


def _gemm(m, n, k):
    return 2.0 * m * n * k


@pytest.mark.parametrize("name", list(CONFIGS))
def test_backward_flops_count_every_contraction(name):
    c = CONFIGS[name]
    P = c.T * c.k
    routed = (_gemm(P, 2 * c.I, c.H)     # recompute [g | u] = x W_gu^T
              + _gemm(P, c.I, c.H)       # dhu = dout W_d
              + _gemm(P, c.H, 2 * c.I)   # dx rows = [dg du] W_gu
              + _gemm(c.H, c.I, P)       # dW_d = (w dout)^T h, summed over the experts' rows
              + _gemm(2 * c.I, c.H, P))  # dW_gu = [dg du]^T x
    router = _gemm(c.T, c.E, c.H) * 3    # logits, dgate_w = dL^T x, dx += dL gate_w
    Is = c.I_shared
    shared = (_gemm(c.T, 2 * Is, c.H) + _gemm(c.T, Is, c.H) + _gemm(c.T, c.H, 2 * Is) + _gemm(c.H, Is, c.T)
              + _gemm(2 * Is, c.H, c.T))
    assert bench.backward_flops(c) == pytest.approx(routed + router + shared, rel=1e-12)


@pytest.mark.parametrize("name", list(CONFIGS))
def test_backward_bytes_count_every_tensor(name):
    c = CONFIGS[name]
    es = 4 if c.dtype == "f32" else 2
    active = min(c.E, c.T * c.k) // 2 or 1
    gu, dn, gw = 2 * c.I * c.H, c.H * c.I, c.E * c.H  # elements of one expert's gate_up, down; the router
    sh = 3 * c.I_shared * c.H + (c.H if c.shared == "sigmoid_gated" else 0)
    reads = es * (active * (gu + dn) + gw + sh + 2 * c.T * c.H)              # weights in use, x, dout
    writes = 4 * (c.E * (gu + dn) + gw + sh + c.T * c.H                      # every gradient, dx
                  + (c.E if c.bias_mode == "logit" else 0))                  # d_bias
    assert bench.backward_bytes(c, active, es) == pytest.approx(reads + writes, rel=1e-12)


@pytest.mark.parametrize("name", list(CONFIGS))
def test_forward_accounting(name):
    c = CONFIGS[name]
    P = c.T * c.k
    es = 4 if c.dtype == "f32" else 2
    active = min(c.E, P)
    fb = bench.flops_and_bytes(c, active)
    assert fb["gate_up_flops"] == _gemm(P, 2 * c.I, c.H)
    assert fb["active_flops"] == pytest.approx(
        _gemm(P, 2 * c.I, c.H) + _gemm(P, c.H, c.I) + (_gemm(c.T, 2 * c.I_shared, c.H) + _gemm(c.T, c.H, c.I_shared)),
        rel=1e-12)
    assert fb["router_flops"] == _gemm(c.T, c.E, c.H)
    # gate_up kernel: the active experts' gate_up weights once and x read once (x_perm and h are the
    # implementation's intermediates, not algorithmic traffic); down: its weights once and out written once
    assert fb["gate_up_bytes"] == (active * 2 * c.I * c.H + c.T * c.H) * es
    assert fb["down_flops"] == _gemm(P, c.H, c.I)
    assert fb["down_bytes"] == (active * c.H * c.I + c.T * c.H) * es
    # whole forward: every active weight once, the router and shared weights, x in and out back
    shared_w = 3 * c.I_shared * c.H if c.shared != "none" else 0
    assert fb["min_bytes"] == (active * 3 * c.I * c.H + c.E * c.H + shared_w + 2 * c.T * c.H) * es


def test_host_memory_probe_is_positive():
    assert bench.host_memory_available() > 0


def test_job_throughput_is_whole_job():
    # two ranks of 4096 tokens, 10 steps in 20 ms (the slower rank's time)
    assert bench.job_throughput(2, 4096, 10, 20.0) == pytest.approx(2 * 4096 * 10 / 0.020)
    assert workloads.CONFIGS["qwen3_30b_a3b"].P == 4096 * 8


def test_reference_arm_prints_one_contract_line():
    """`bench.py --impl reference` (the oracle on the host cores) prints one
    JSON line with the contract's keys; it needs no GPU."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--config",
                        "tiny_fp32", "--steps", "2", "--warmup", "3"], capture_output=True, text=True, timeout=300,
                       cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["steps"] == 2 and line["warmup"] == 3
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["config"]["workload"] == "tiny_fp32"


def test_roofline_entry_by_hand():
    """The fraction is algorithmic work / time / peak, bounded by the larger of
    the tensor and HBM times; a reader can redo it from the printed numbers."""
    pk = {"hbm_gbs": 6500.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0, "source": "measured"}
    e = bench.roofline_entry(206.16e9, 822e6, 0.2171, pk, "bf16")
    assert e["bound"] == "tensor"
    assert e["achieved"] == pytest.approx(206.16e9 / 0.2171e-3 / 1e12)
    assert e["frac"] == pytest.approx(206.16e9 / 0.2171e-3 / 1e12 / 1600.0)
    assert e["t_roof_ms"] == pytest.approx(206.16e9 / 1600e12 * 1e3)
    h = bench.roofline_entry(12.7e9, 9.08e9, 1.45, pk, "bf16")
    assert h["bound"] == "hbm" and h["frac"] == pytest.approx(9.08e9 / 1.45e-3 / 1e9 / 6500.0)
    f = bench.roofline_entry(1e12, 1e6, 100.0, pk, "f32", mhz=1965.0)
    assert f["bound"] == "alu" and f["peak"] == pytest.approx(148 * 128 * 2 * 1965e6 / 1e12)


def test_config_is_the_same_for_both_arms():
    """The workload dict carries no arm-specific key: the reference arm's
    config equals ours for every named problem."""
    for c in CONFIGS.values():
        d = bench.config_dict(c)
        assert d == bench.config_dict(c) and "parallelism" not in d
        assert d["workload"] == c.name and "l2" in d
