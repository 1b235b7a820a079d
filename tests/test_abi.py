"""The C-ABI library loads, exports every symbol include/moe.h declares, and
its host-side validation behaves (no GPU: only calls that return before any
CUDA work)."""

import ctypes
import os
import re

import pytest

import sparse_top_mixture_b200 as stm

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(moe_\w+)\s*\(", text))
    return sorted(names)


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(stm.LIB_PATH):
        stm.build_lib = __import__("sparse_top_mixture_b200.build", fromlist=["build"])
        stm.build_lib.build()
    return stm.lib()


def test_every_declared_symbol_is_exported(L):
    syms = header_symbols()
    assert len(syms) >= 13
    for s in syms:
        assert hasattr(L, s), f"{s} declared in include/ but not exported"
    assert set(syms) == set(stm.SIGNATURES), "binding signatures out of sync with the header"


def test_status_strings(L):
    assert L.moe_status_string(0) == b"ok"
    assert b"workspace" in L.moe_status_string(3)
    assert L.moe_status_string(99) == b"unknown status"


def _p(**kw):
    base = dict(T=64, H=256, E=8, k=2, I=128, dtype="bf16")
    base.update(kw)
    return stm.Problem(**base)


def test_workspace_size_grows_with_problem(L):
    a = stm.workspace_size(_p())
    b = stm.workspace_size(_p(T=128))
    c = stm.workspace_size(_p(shared="plain", I_shared=256))
    assert 0 < a < b and a < c
    # x_perm + h + y_perm dominate
    assert a >= 64 * 2 * (256 + 128 + 256) * 2


@pytest.mark.parametrize("bad", [
    dict(k=0), dict(k=9), dict(E=0), dict(E=257, k=2), dict(H=250), dict(I=100), dict(T=-1),
    dict(dtype="f32", shared="plain", I_shared=0), dict(shared="plain", I_shared=12),
])
def test_invalid_problems_rejected(L, bad):
    with pytest.raises(stm.MoeError) as ei:
        stm.workspace_size(_p(**bad))
    assert ei.value.status == 1


def test_gemm_path(L):
    # 0 = SIMT fp32; 1 = tcgen05 one CTA per 128-row tile; 2 = CTA pairs (gate_up GEMM reported)
    assert stm.gemm_path(_p(dtype="f32")) == 0
    assert stm.gemm_path(_p()) == 1  # 64*2 pairs over 8 experts: 16 rows per expert
    assert stm.gemm_path(_p(T=4096, E=128, k=8)) == 2  # 256 rows per expert: gate_up on pairs
    assert stm.gemm_path(_p(T=8192, E=64, k=6)) == 2  # 768 rows per expert
    assert stm.gemm_path(_p(T=16, E=256, k=8)) == 1


def test_launch_counts(L):
    # route 2 (logits, top-k), dispatch 2 (histogram + scan, permute + gather), combine 1, plus the expert GEMMs
    assert stm.launches_per_forward(_p()) == 5 + 2
    assert stm.launches_per_forward(_p(T=8192, E=64, k=6)) == 5 + 2
    assert stm.launches_per_forward(_p(T=8192, E=64, k=6, shared="plain", I_shared=256)) == 5 + 2 + 2
    assert stm.launches_per_forward(_p(T=8192, E=64, k=6, shared="plain", I_shared=256, dtype="f32")) == 5 + 4
    assert stm.launches_per_forward(_p(dtype="f32", shared="plain", I_shared=256)) == 5 + 4
    assert stm.launches_per_forward(_p(T=0)) == 0
    gated = _p(shared="sigmoid_gated", I_shared=256)  # small shared expert: runs on the aux stream
    assert stm.launches_per_forward(gated, two_streams=True) == stm.launches_per_forward(gated) + 1
    big = _p(T=8192, shared="sigmoid_gated", I_shared=2048)  # fills the GPU: beside the dispatch, no gate kernel
    assert stm.launches_per_forward(big, two_streams=True) == stm.launches_per_forward(big)


def test_calls_validate_before_launching(L):
    p = _p().c()
    # null / misaligned pointers are rejected on the host, before any CUDA call
    st = L.moe_route(ctypes.byref(p), None, None, None, None, None, None, None, None, 0, None)
    assert st == 1
    # x given without x_perm
    st = L.moe_dispatch(ctypes.byref(p), 16, 16, 16, 16, 16, 16, None, 16, 1 << 30, None)
    assert st == 1
    st = L.moe_combine(ctypes.byref(p), 8, 16, None, 16, None)
    assert st == 1  # y_perm misaligned
    # workspace too small
    st = L.moe_grouped_swiglu(ctypes.byref(p), 16, 16, 16, 16, None, None, 16, 16, 1024, None)
    assert st == 3
    # bias mode without a bias
    pb = _p(bias_mode="select").c()
    st = L.moe_topk_from_logits(ctypes.byref(pb), 16, None, 16, 16, None)
    assert st == 1


def test_empty_batch_is_a_noop(L):
    """T == 0 returns OK without launching anything (no GPU needed)."""
    p = _p(T=0).c()
    w = stm.moe_weights(16, None, 16, 16, None, None, None)
    n = ctypes.c_size_t(0)
    assert L.moe_workspace_size(ctypes.byref(p), ctypes.byref(n)) == 0
    st = L.moe_forward(ctypes.byref(p), ctypes.byref(w), 16, 16, 16, 16, 16, n.value, None)
    assert st == 0


def test_backward_validates_before_launching(L):
    """moe_backward rejects bad arguments on the host (no GPU needed)."""
    w = stm.moe_weights(16, None, 16, 16, None, None, None)
    g = stm.moe_grads(16, 16, None, 16, 16, None, None, None)
    n = ctypes.c_size_t(0)
    p32 = _p(dtype="f32").c()
    assert L.moe_backward_workspace_size(ctypes.byref(p32), ctypes.byref(n)) == 0
    assert n.value >= 256
    # bf16 problems have their own (larger) workspace: the fp32 size is too small for them
    pb = _p(dtype="bf16").c()
    nb = ctypes.c_size_t(0)
    assert L.moe_backward_workspace_size(ctypes.byref(pb), ctypes.byref(nb)) == 0
    assert nb.value > n.value
    assert L.moe_backward(ctypes.byref(pb), ctypes.byref(w), 16, 16, 16, ctypes.byref(g), 16, n.value, None) == 3
    # misaligned dout
    assert L.moe_backward(ctypes.byref(p32), ctypes.byref(w), 16, 8, 16, ctypes.byref(g), 16, n.value, None) == 1
    # logit bias without a d_bias output
    pl = _p(dtype="f32", bias_mode="logit").c()
    wl = stm.moe_weights(16, 16, 16, 16, None, None, None)
    assert L.moe_backward(ctypes.byref(pl), ctypes.byref(wl), 16, 16, 16, ctypes.byref(g), 16, 1 << 40, None) == 1
    # workspace too small
    assert L.moe_backward(ctypes.byref(p32), ctypes.byref(w), 16, 16, 16, ctypes.byref(g), 16, 16, None) == 3
    # gated shared expert without its gate gradient
    pg = _p(dtype="f32", shared="sigmoid_gated", I_shared=64).c()
    wg = stm.moe_weights(16, None, 16, 16, 16, 16, 16)
    gg = stm.moe_grads(16, 16, None, 16, 16, 16, 16, None)
    assert L.moe_backward(ctypes.byref(pg), ctypes.byref(wg), 16, 16, 16, ctypes.byref(gg), 16, 1 << 40, None) == 1


def test_ep_arena_layout(L):
    """The expert-parallel arena's regions: 256-byte aligned, in order, each
    large enough for what the exchange stores there (host-only calls)."""
    from sparse_top_mixture_b200.ep_peer import ep_arena_offsets, ep_arena_size

    for kw, G in ((dict(T=64, H=256, E=8, k=2), 2), (dict(T=300, H=328, E=128, k=8), 4),
                  (dict(T=16, H=7168, E=256, k=8, dtype="f32"), 8), (dict(T=0, H=64, E=4, k=1), 1)):
        p = _p(**kw)
        C, es = p.T * p.k, (4 if p.dtype == "f32" else 2)
        off = ep_arena_offsets(p, G)
        order = ["rows_flag", "ret_flag", "x", "w", "id", "y"]
        assert all(off[n] % 256 == 0 for n in order)
        assert [off[n] for n in order] == sorted(off[n] for n in order)
        assert off["ret_flag"] - off["rows_flag"] >= 8 * G
        assert off["w"] - off["x"] >= G * C * p.H * es
        assert off["id"] - off["w"] >= G * C * 4 and off["y"] - off["id"] >= G * C * 8
        assert ep_arena_size(p, G) >= off["y"] + C * p.H * 4
    bad = _p(E=6, k=2)
    n = ctypes.c_size_t()
    assert L.moe_ep_arena_size(ctypes.byref(bad.c()), 4, ctypes.byref(n)) == 1  # E not divisible by G
    assert L.moe_ep_arena_size(ctypes.byref(bad.c()), 0, ctypes.byref(n)) == 1
