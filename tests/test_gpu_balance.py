"""GPU parity of the aux-loss-free balancer's bias update (moe_bias_stash /
moe_bias_update) against oracle/balance.py: bit-exact fp32 biases and int64
stashes, through the C ABI."""

import numpy as np
import pytest
import torch

import oracle.balance as ob
import sparse_top_mixture_b200 as stm
import workloads
from workloads import CONFIGS, reduced

pytestmark = pytest.mark.gpu


def _problem(E):
    return stm.Problem(T=1, H=64, E=E, k=1, I=64, dtype="bf16", bias_mode="select")


@pytest.mark.parametrize("E", [1, 5, 8, 64, 128, 256])
def test_bias_update_bit_exact(E):
    rng = np.random.default_rng(E)
    p = _problem(E)
    for trial in range(6):
        if trial % 2:
            loads = rng.integers(0, 1 << 20, size=E)
        else:  # pairs around a common value, some exactly at the mean
            d = rng.integers(0, 2, size=E // 2) * rng.integers(0, 1000, size=E // 2)
            loads = np.concatenate([5000 - d, 5000 + d, [5000] * (E % 2)])
        bias = rng.normal(0, 0.5, size=E).astype(np.float32)
        rate = [1e-3, 0.05, 2.0 ** -12][trial % 3]
        want, cleared = ob.bias_update(bias, loads, rate)
        st = torch.tensor(loads, dtype=torch.int64, device="cuda")
        b = torch.tensor(bias, device="cuda")
        stm.bias_update(p, st, b, rate)
        torch.cuda.synchronize()
        assert np.array_equal(b.cpu().numpy(), want)
        assert np.array_equal(st.cpu().numpy(), cleared)


def test_second_update_is_noop():
    p = _problem(6)
    st = torch.tensor([9, 1, 3, 3, 2, 0], dtype=torch.int64, device="cuda")
    b = torch.zeros(6, device="cuda")
    stm.bias_update(p, st, b, 0.25)
    once = b.clone()
    stm.bias_update(p, st, b, 0.25)
    torch.cuda.synchronize()
    assert torch.equal(b, once) and not torch.equal(once, torch.zeros_like(once))


def test_invalid_rate_rejected():
    p = _problem(4)
    st = torch.zeros(4, dtype=torch.int64, device="cuda")
    b = torch.zeros(4, device="cuda")
    with pytest.raises(stm.MoeError):
        stm.bias_update(p, st, b, float("nan"))


def test_balancer_tracks_oracle_over_forwards():
    """Forward, stash the forward's counts, update, repeat: the stash equals
    the bincount of the returned selections, and the bias the GPU keeps
    equals the oracle's bias step by step (bit for bit)."""
    cfg = reduced(CONFIGS["dsv4_flash_ablation"], T=384, H=512, I=256, I_shared=256)
    cpu = workloads.generate(cfg, "cpu")
    dev = {k: (v.cuda() if v is not None else None) for k, v in cpu.items()}
    dev["bias"] = dev["bias"].clone()
    p = stm.Problem.from_config(cfg)
    moe = stm.SparseMoE(p, dev)
    bal = stm.BiasBalancer(moe, rate=1e-3)
    bias_ref = cpu["bias"].numpy().astype(np.float32)
    g = torch.Generator(device="cuda").manual_seed(9)
    for step in range(4):
        stash_ref = np.zeros(cfg.E, np.int64)
        for micro in range(2):  # two forwards stash into one update
            x = torch.randn(cfg.T, cfg.H, generator=g, device="cuda").to(torch.bfloat16)
            _, _, sel = moe(x)
            bal.stash()
            stash_ref = ob.stash_counts(stash_ref, np.bincount(sel.cpu().numpy().ravel(), minlength=cfg.E))
        torch.cuda.synchronize()
        assert np.array_equal(bal.load_stash.cpu().numpy(), stash_ref)
        bal.update()
        bias_ref, _ = ob.bias_update(bias_ref, stash_ref, 1e-3)
        torch.cuda.synchronize()
        assert np.array_equal(bal.bias.cpu().numpy(), bias_ref)
        assert torch.count_nonzero(bal.load_stash).item() == 0
    assert moe.read_device_error() == 0
