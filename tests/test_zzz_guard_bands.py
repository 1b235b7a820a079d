"""Guard bands around outputs: each output tensor handed to the library is a
view into a larger buffer whose head and tail hold a canary value; after the
call both bands must be unchanged (no write outside an output), and the
outputs must equal those of the same call into plain tensors.

Covers the forward (its routing weights, selected experts and out; the
one-CTA, CTA-pair and SIMT GEMM paths; the two-stream shared expert) and the
fp32 backward (every gradient)."""

import math

import pytest
import torch

import sparse_top_mixture_b200 as stm
import workloads
from workloads import CONFIGS, reduced

pytestmark = pytest.mark.gpu

BAND = 64  # elements before and after each output (128-512 bytes: keeps 16-byte alignment)
CANARY = {torch.bfloat16: -1024.0, torch.float32: -1024.0, torch.int64: -7777}

FORWARD = {
    "tiny_fp32": CONFIGS["tiny_fp32"],
    "ragged_bf16_shared": CONFIGS["dsv4_flash_ablation"].replace(name="ragged", T=37, H=40, E=5, k=3, I=24,
                                                                 I_shared=16),
    "pairs_tails": CONFIGS["qwen3_30b_a3b"].replace(name="pairs_tails", T=2300, H=320, E=8, k=2, I=200),
    "decode_gated": reduced(CONFIGS["decode_weight_streaming"], T=16, H=1024, I=256, I_shared=256),
}


def _guarded(shape, dtype):
    n = math.prod(shape)
    buf = torch.full((BAND + n + BAND,), CANARY[dtype], dtype=dtype, device="cuda")
    return buf, buf[BAND:BAND + n].view(*shape)


def _bands_intact(buf, shape) -> bool:
    n = math.prod(shape)
    c = CANARY[buf.dtype]
    head, tail = buf[:BAND], buf[BAND + n:]
    return bool((head == c).all().item()) and bool((tail == c).all().item())


@pytest.mark.parametrize("name", list(FORWARD))
def test_forward_writes_only_its_outputs(name):
    cfg = FORWARD[name]
    cpu = workloads.generate(cfg, "cpu")
    dev = {k: (v.cuda() if v is not None else None) for k, v in cpu.items()}
    p = stm.Problem.from_config(cfg)
    moe = stm.SparseMoE(p, dev)
    ob, out = _guarded((p.T, p.H), p.torch_dtype)
    wb, rw = _guarded((p.T, p.k), torch.float32)
    sb, sel = _guarded((p.T, p.k), torch.int64)
    moe.forward(dev["x"], out, rw, sel)
    ref_out, ref_rw, ref_sel = moe.forward(dev["x"])
    torch.cuda.synchronize()
    assert moe.read_device_error() == 0
    for buf, shape, what in ((ob, (p.T, p.H), "out"), (wb, (p.T, p.k), "routing_weights"),
                             (sb, (p.T, p.k), "selected_experts")):
        assert _bands_intact(buf, shape), f"{name}: a write landed outside {what}"
    assert torch.equal(out, ref_out) and torch.equal(rw, ref_rw) and torch.equal(sel, ref_sel)


BACKWARD = {
    "softmax_logit_gated": CONFIGS["tiny_fp32"].replace(name="bw_gated", T=45, H=40, E=6, k=3, I=24, I_shared=16,
                                                        bias_mode="logit", bias_kind="uniform0.1",
                                                        shared="sigmoid_gated"),
    "qwen3_shape_f32": reduced(CONFIGS["qwen3_30b_a3b"], T=300, H=328, I=200).replace(dtype="f32"),
}


@pytest.mark.parametrize("name", list(BACKWARD))
def test_backward_writes_only_its_gradients(name):
    cfg = BACKWARD[name]
    cpu = workloads.generate(cfg, "cpu")
    dev = {k: (v.cuda() if v is not None else None) for k, v in cpu.items()}
    p = stm.Problem.from_config(cfg)
    sel = stm.SparseMoE(p, dev)(dev["x"])[2]
    dout = torch.randn(p.T, p.H, generator=torch.Generator().manual_seed(3)).cuda()
    ref = stm.backward(p, dev, dev["x"], dout, sel)
    shapes = {key: tuple(t.shape) for key, t in ref.items() if t is not None}
    bufs, outs = {}, {}
    for key, shape in shapes.items():
        bufs[key], outs[key] = _guarded(shape, torch.float32)
    got = stm.backward(p, dev, dev["x"], dout, sel, out=outs)
    torch.cuda.synchronize()
    for key, shape in shapes.items():
        assert got[key] is outs[key]
        assert _bands_intact(bufs[key], shape), f"{name}: a write landed outside {key}"
        assert torch.equal(outs[key], ref[key]), f"{name}: {key} differs from the unguarded call"
