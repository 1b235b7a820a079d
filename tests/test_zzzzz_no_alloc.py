"""moe_dispatch_noalloc, the dispatch entry point that allocates nothing.

It serves callers that may not allocate device memory (a thread running
while a CUDA graph is captured in global mode, a plug-in inside a framework
whose memory pool owns the GPU, an allocator-free latency path): instead of
a caller workspace it keeps its count matrix and its histogram ticket in
fixed device arrays inside the library. These checks call it through the C
ABI and compare it with moe_dispatch and with the oracle's stable argsort on
the same inputs -- bit for bit, as for all index work -- on two calls in a
row with different inputs, so that anything left in the shared arrays by the
first call would show up in the second. One check runs it inside a CUDA graph
captured in global mode (any allocation during the capture would fail it),
after a first call outside the capture has looked up the arrays' addresses.

This file is collected last (its name sorts after every other test file),
so that a run stopping at the first failure has already run all the others.
"""

import numpy as np
import pytest
import torch

import gpu_check as gc
import sparse_top_mixture_b200 as stm

pytestmark = pytest.mark.gpu


def _case(T, E, k, H, seed):
    g = torch.Generator().manual_seed(seed)
    sel = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).to(torch.int64)
    x = torch.randn(T, H, generator=g).to(torch.bfloat16)
    return stm.Problem(T=T, H=H, E=E, k=k, I=8), sel.cuda(), x.cuda()


KEYS = ("counts", "offsets", "sorted_pairs", "pair_pos", "x_perm")


def test_no_alloc_dispatch_matches_workspace_dispatch_and_oracle():
    for T, E, k, H, seed in ((1000, 128, 8, 72, 11), (333, 64, 6, 40, 12)):
        p, sel, x = _case(T, E, k, H, seed)
        ref = stm.dispatch(p, sel, x)
        got = stm.dispatch_noalloc(p, sel, x)
        torch.cuda.synchronize()
        for key in KEYS:
            assert torch.equal(got[key], ref[key]), f"{key} differs (T={T}, E={E}, k={k})"
        d = gc.assert_dispatch_exact(got, sel.cpu().numpy(), E)
        assert torch.equal(got["x_perm"].cpu(), x.cpu()[torch.from_numpy(d["sorted_pairs"] // k)])


def test_no_alloc_dispatch_skips_bad_ids_without_a_flag():
    p, sel, x = _case(50, 8, 2, 16, 13)
    sel[7, 1] = p.E  # one past the last expert
    sel[20, 0] = -1
    ws = stm.new_workspace(p)
    ref = stm.dispatch(p, sel, x, ws=ws)
    got = stm.dispatch_noalloc(p, sel, x)
    torch.cuda.synchronize()
    assert stm.read_device_error(ws) == stm.DEVERR_BAD_EXPERT_ID  # the workspace call flags it
    pp = got["pair_pos"].cpu().numpy()
    assert pp[7 * p.k + 1] == -1 and pp[20 * p.k] == -1
    used = int(got["offsets"][-1])
    assert used == p.T * p.k - 2
    # positions past the dispatched pairs are not written by either call
    for key in ("counts", "offsets", "pair_pos"):
        assert torch.equal(got[key], ref[key]), key
    assert torch.equal(got["sorted_pairs"][:used], ref["sorted_pairs"][:used])
    assert torch.equal(got["x_perm"][:used], ref["x_perm"][:used])


def test_no_alloc_dispatch_empty_batch():
    p = stm.Problem(T=0, H=16, E=8, k=2, I=8)
    sel = torch.empty(0, 2, dtype=torch.int64, device="cuda")
    got = stm.dispatch_noalloc(p, sel)
    torch.cuda.synchronize()
    assert got["counts"].sum().item() == 0 and torch.count_nonzero(got["offsets"]).item() == 0


def test_no_alloc_dispatch_size_limit():
    # ceil(T / (256 / k)) * E count entries must fit the static 2^18-entry
    # array: exactly 2^18 is accepted, one more dispatch block is rejected
    E, k = 256, 8
    T = (1 << 18) // E * (256 // k)
    p = stm.Problem(T=T, H=8, E=E, k=k, I=8)
    g = torch.Generator(device="cuda").manual_seed(14)
    sel = torch.randint(0, E, (T, k), generator=g, device="cuda", dtype=torch.int64)
    got = stm.dispatch_noalloc(p, sel)
    ref = stm.dispatch(p, sel)
    torch.cuda.synchronize()
    for key in ("counts", "offsets", "sorted_pairs", "pair_pos"):
        assert torch.equal(got[key], ref[key]), key
    big = stm.Problem(T=T + 1, H=8, E=E, k=k, I=8)
    sel_big = torch.zeros(big.T, k, dtype=torch.int64, device="cuda")
    with pytest.raises(stm.MoeError) as ei:
        stm.dispatch_noalloc(big, sel_big)
    assert ei.value.status == 2


def test_no_alloc_dispatch_inside_a_global_mode_capture():
    p, sel, x = _case(700, 64, 6, 48, 15)
    ref = stm.dispatch(p, sel, x)
    out = {key: torch.empty_like(v) for key, v in ref.items()}
    stm.dispatch_noalloc(p, sel, x, out=out)  # outside any capture: looks up the arrays' addresses
    torch.cuda.synchronize()
    for v in out.values():
        v.zero_()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, capture_error_mode="global"):
        stm.dispatch_noalloc(p, sel, x, out=out)
    for _ in range(2):
        graph.replay()
        torch.cuda.synchronize()
        for key in KEYS:
            assert torch.equal(out[key], ref[key]), key
    del graph
