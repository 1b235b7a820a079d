"""moe_dispatch_noalloc, the dispatch entry point that allocates nothing.

It serves callers that may not allocate device memory (a thread running
while a CUDA graph is captured in global mode, a plug-in inside a framework
whose memory pool owns the GPU, an allocator-free latency path): instead of
a caller workspace it keeps its count matrix in a fixed device array inside
the library. These checks call it through the C ABI and compare it with
moe_dispatch on the same inputs -- bit for bit, as for all index work --
on two calls in a row with different inputs, so that anything left in the
shared array by the first call would show up in the second.

This file is collected after the parity tests (only the guard-band checks
come later) so that a run stopping at the first failure has already run
them.
"""

import pytest
import torch

import sparse_top_mixture_b200 as stm

pytestmark = pytest.mark.gpu


def _case(T, E, k, H, seed):
    g = torch.Generator().manual_seed(seed)
    sel = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).to(torch.int64)
    x = torch.randn(T, H, generator=g).to(torch.bfloat16)
    return stm.Problem(T=T, H=H, E=E, k=k, I=8), sel.cuda(), x.cuda()


def test_no_alloc_dispatch_matches_workspace_dispatch():
    for T, E, k, H, seed in ((1000, 128, 8, 72, 11), (333, 64, 6, 40, 12)):
        p, sel, x = _case(T, E, k, H, seed)
        ref = stm.dispatch(p, sel, x)
        got = stm.dispatch_noalloc(p, sel, x)
        torch.cuda.synchronize()
        for key in ("counts", "offsets", "sorted_pairs", "pair_pos", "x_perm"):
            assert torch.equal(got[key], ref[key]), f"{key} differs (T={T}, E={E}, k={k})"


def test_no_alloc_dispatch_rejects_oversized_problems():
    # ceil(T / (256 / k)) * E count entries must fit the static 2^18-entry array
    p = stm.Problem(T=40000, H=8, E=256, k=8, I=8)
    sel = torch.zeros(p.T, p.k, dtype=torch.int64, device="cuda")
    with pytest.raises(stm.MoeError) as ei:
        stm.dispatch_noalloc(p, sel)
    assert ei.value.status == 2
