"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Sizes: each named problem at a reduced size the oracle finishes in seconds
(ragged K/N tails, several row tiles per expert), the tiny fp32 problem at full
size, plus every named problem at its full size with sampled tokens checked
one by one against the oracle and the dispatch checked in full.
"""

import numpy as np
import pytest
import torch

import gpu_check as gc
import oracle
import sparse_top_mixture_b200 as stm
import workloads
from workloads import CONFIGS, reduced

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny_fp32": CONFIGS["tiny_fp32"],
    "qwen3_30b_a3b": reduced(CONFIGS["qwen3_30b_a3b"], T=300, H=328, I=200),
    "deepseek_v2_lite_zipf": reduced(CONFIGS["deepseek_v2_lite_zipf"], T=512, H=256, I=136, I_shared=272),
    "dsv4_flash_ablation": reduced(CONFIGS["dsv4_flash_ablation"], T=384, H=512, I=256, I_shared=256),
    "decode_weight_streaming": reduced(CONFIGS["decode_weight_streaming"], T=16, H=1024, I=256, I_shared=256),
}

EDGE = {
    "single_token": reduced(CONFIGS["qwen3_30b_a3b"], T=1, H=256, I=128),
    "k_equals_E": CONFIGS["tiny_fp32"].replace(name="k_eq_E", T=40, H=64, E=8, k=8, I=64, dtype="bf16"),
    "one_expert": CONFIGS["tiny_fp32"].replace(name="E1", T=130, H=128, E=1, k=1, I=136, dtype="bf16"),
    "tiny_ragged_bf16": CONFIGS["dsv4_flash_ablation"].replace(name="ragged", T=37, H=40, E=5, k=3, I=24,
                                                               I_shared=16),
    "tiny_ragged_f32": CONFIGS["decode_weight_streaming"].replace(name="ragged32", T=29, H=24, E=6, k=3, I=40,
                                                                  I_shared=8, dtype="f32"),
    "many_tiles_one_expert": CONFIGS["qwen3_30b_a3b"].replace(name="skew", T=700, H=192, E=4, k=1, I=136),
    # routed segments averaging >= 128 rows run on CTA pairs (256-row tiles)
    "pairs_ragged": CONFIGS["qwen3_30b_a3b"].replace(name="pairs", T=1731, H=384, E=8, k=2, I=200),
    # ~575 rows per expert: two 256-row pair tiles plus a ~40..100-row tail (M=128 pair MMA)
    "pairs_tails": CONFIGS["qwen3_30b_a3b"].replace(name="pairs_tails", T=2300, H=320, E=8, k=2, I=200),
    "pairs_shared_skew": CONFIGS["deepseek_v2_lite_zipf"].replace(name="pairs_zipf", T=4200, H=256, I=136,
                                                                  I_shared=272),
    # k > 8: 12 top-k rounds per token, dispatch blocks of 21 tokens
    "k_above_8": CONFIGS["qwen3_30b_a3b"].replace(name="k12", T=100, H=128, E=16, k=12, I=64),
    # a sigmoid-gated shared expert too large to overlap the routed GEMMs
    # (8 x 16 row x column tiles): it runs beside the dispatch
    "large_shared_gated": CONFIGS["decode_weight_streaming"].replace(name="large_gated", T=1000, H=512, E=32, k=4,
                                                                     I=128, I_shared=2048),
}


def _inputs(cfg, device="cuda"):
    cpu = workloads.generate(cfg, "cpu")
    dev = {k: (v.to(device) if v is not None else None) for k, v in cpu.items()}
    return cpu, dev


def _moe(cfg, dev):
    return stm.SparseMoE(stm.Problem.from_config(cfg), dev)


def _forward_and_check(cfg, cpu, dev):
    moe = _moe(cfg, dev)
    out, rw, sel = moe(dev["x"])
    torch.cuda.synchronize()
    assert moe.read_device_error() == 0
    r = gc.oracle_route(cfg, cpu)
    gsel = sel.cpu().numpy()
    ntie = gc.check_selection(cfg, r, gsel)
    o = gc.oracle_forward(cfg, cpu, selected=gsel)
    assert np.abs(rw.cpu().double().numpy() - o["routing_weights"]).max() <= 1e-5
    stats = gc.assert_close(out.cpu().double().numpy(), o["out"], cfg.dtype, cfg.name)
    return moe, out, o, ntie, stats


@pytest.mark.parametrize("name", list(SMALL))
def test_forward_parity(name):
    cfg = SMALL[name]
    cpu, dev = _inputs(cfg)
    moe, out, o, ntie, stats = _forward_and_check(cfg, cpu, dev)
    print(f"{name}: near-tie tokens {ntie}, {stats}")
    assert ntie == gc.expected_near_ties(cfg.name), f"{cfg.name}: {ntie} tokens took the near-tie escape"
    assert stm.gemm_path(moe.p) == (1 if cfg.dtype == "bf16" else 0)


@pytest.mark.parametrize("name", list(EDGE))
def test_forward_edge_cases(name):
    cfg = EDGE[name]
    cpu, dev = _inputs(cfg)
    _, _, _, ntie, _ = _forward_and_check(cfg, cpu, dev)
    assert ntie == gc.expected_near_ties(cfg.name), f"{cfg.name}: {ntie} tokens took the near-tie escape"


def test_both_tensor_core_variants_are_exercised():
    """The one-CTA (128-row tiles) and CTA-pair (256-row tiles) tcgen05
    kernels are both reached by the parity cases above."""
    paths = {name: stm.gemm_path(stm.Problem.from_config(cfg)) for name, cfg in {**SMALL, **EDGE}.items()}
    assert paths["tiny_fp32"] == 0
    assert paths["pairs_ragged"] == 2 and paths["pairs_shared_skew"] == 2 and paths["pairs_tails"] == 2
    assert paths["qwen3_30b_a3b"] == 1 and paths["decode_weight_streaming"] == 1


@pytest.mark.parametrize("name", list(SMALL) + ["pairs_shared_skew", "large_shared_gated", "pairs_tails",
                                                 "k_above_8"])
def test_staged_calls_match_forward(name):
    """route -> dispatch -> grouped_swiglu -> shared_expert -> combine through
    the separate entry points equals moe_forward bit for bit (also with a
    shared expert large enough to run beside the dispatch), and each stage
    matches the oracle; the forward's expert counts (read back from its
    workspace) equal the staged dispatch's."""
    cfg = EDGE.get(name) or SMALL[name]
    cpu, dev = _inputs(cfg)
    p = stm.Problem.from_config(cfg)
    ws = stm.new_workspace(p)
    moe = _moe(cfg, dev)
    out_f, rw_f, sel_f = moe(dev["x"])
    rw, sel, gam = stm.route(p, dev["x"], dev["gate_w"], dev["bias"], dev["shared_gate"], ws=ws)
    d = stm.dispatch(p, sel, dev["x"], ws=ws)
    y = stm.grouped_swiglu(p, d["x_perm"], d["offsets"], dev["gate_up"], dev["down"], rw, d["sorted_pairs"], ws=ws)
    sh = None
    if cfg.shared != "none":
        sh = stm.shared_expert(p, dev["x"], dev["shared_gate_up"], dev["shared_down"], gam, ws=ws)
    out = stm.combine(p, y, d["pair_pos"], sh)
    torch.cuda.synchronize()
    assert torch.equal(sel, sel_f) and torch.equal(rw, rw_f) and torch.equal(out, out_f)
    assert torch.equal(moe.forward_counts(), d["counts"])
    # stage-level parity
    gsel = sel.cpu().numpy()
    r = gc.oracle_route(cfg, cpu)
    assert gc.check_selection(cfg, r, gsel) == gc.expected_near_ties(cfg.name)
    dd = gc.assert_dispatch_exact(d, gsel, cfg.E)
    xs = d["x_perm"].cpu()
    assert torch.equal(xs, cpu["x"][torch.from_numpy(dd["sorted_pairs"] // cfg.k)])
    if gam is not None:
        ref_g = oracle.shared_gate_values(gc.np64(cpu["x"]), gc.np64(cpu["shared_gate"]), cfg.shared)
        assert np.abs(gam.cpu().double().numpy() - ref_g).max() <= 1e-5
    w_ref = oracle.topk_weights(r["scores"], gsel, cfg.renormalize).reshape(-1)
    xn = gc.np64(cpu["x"])
    y_ref = np.zeros((cfg.P, cfg.H))
    y_bnd = np.zeros((cfg.P, cfg.H))
    for e in range(cfg.E):
        a, b = dd["offsets"][e], dd["offsets"][e + 1]
        if a == b:
            continue
        q = dd["sorted_pairs"][a:b]
        y_ref[a:b], y_bnd[a:b] = gc.swiglu_with_bound(xn[q // cfg.k], gc.np64(cpu["gate_up"][e]),
                                                      gc.np64(cpu["down"][e]), w_ref[q], cfg.dtype)
    gc.assert_within_bound(y.cpu().double().numpy(), y_ref, y_bnd, "y_perm")
    if sh is not None:
        gam_ref = oracle.shared_gate_values(xn, gc.np64(cpu["shared_gate"]), cfg.shared)
        s_ref, s_bnd = gc.swiglu_with_bound(xn, gc.np64(cpu["shared_gate_up"]), gc.np64(cpu["shared_down"]),
                                            gam_ref, cfg.dtype)
        gc.assert_within_bound(sh.cpu().double().numpy(), s_ref, s_bnd, "shared")


@pytest.mark.parametrize("I", [192, 200])
@pytest.mark.parametrize("counts", [
    [1, 64, 65, 127, 128, 129, 255, 256, 257, 300, 383, 384, 385, 512, 600, 641],
    [300, 290, 257, 310, 384, 260, 270, 280],
    [8, 16, 17, 33, 48, 49, 80, 95, 97, 112, 113, 120, 256 + 15, 256 + 16, 256 + 31, 256 + 100, 900, 1000],
])
def test_segment_sizes_around_pair_tile_edges(counts, I):
    """Segments whose sizes sit on every edge of the CTA-pair tiling (pieces
    of at most 128 rows, full and partial 256-row tiles): every y row of the
    grouped SwiGLU matches the fp64 per-segment reference within the
    arithmetic bound. Pieces of at most 128 rows run with the operands
    swapped (their rows as the MMA's N, 16 to 128 in steps of 16, all of
    which occur here); with I = 200 (not a multiple of 16) gate_up runs them
    unswapped as M=128 pair MMAs and down still swapped. Routing is planted,
    so the sizes are exact."""
    E, H = len(counts), 256
    T = sum(counts)
    g = torch.Generator().manual_seed(len(counts))
    ids = torch.cat([torch.full((c,), e, dtype=torch.int64) for e, c in enumerate(counts)])
    sel = ids[torch.randperm(T, generator=g)].reshape(T, 1)
    x = torch.randn(T, H, generator=g).to(torch.bfloat16)
    gu = (torch.randn(E, 2 * I, H, generator=g) / H ** 0.5).to(torch.bfloat16)
    dn = (torch.randn(E, H, I, generator=g) / I ** 0.5).to(torch.bfloat16)
    rw = torch.rand(T, 1, generator=g) + 0.5
    p = stm.Problem(T=T, H=H, E=E, k=1, I=I, dtype="bf16")
    assert stm.gemm_path(p) == 2
    ws = stm.new_workspace(p)
    d = stm.dispatch(p, sel.cuda(), x.cuda(), ws=ws)
    y = stm.grouped_swiglu(p, d["x_perm"], d["offsets"], gu.cuda(), dn.cuda(), rw.cuda(), d["sorted_pairs"], ws=ws)
    torch.cuda.synchronize()
    assert stm.read_device_error(ws) == 0
    dd = gc.assert_dispatch_exact(d, sel.numpy(), E)
    assert dd["counts"].tolist() == counts
    xn, w = gc.np64(x), rw.double().numpy().reshape(-1)
    y_ref = np.zeros((T, H))
    y_bnd = np.zeros((T, H))
    for e in range(E):
        a, b = dd["offsets"][e], dd["offsets"][e + 1]
        q = dd["sorted_pairs"][a:b]
        y_ref[a:b], y_bnd[a:b] = gc.swiglu_with_bound(xn[q], gc.np64(gu[e]), gc.np64(dn[e]), w[q], "bf16")
    gc.assert_within_bound(y.cpu().double().numpy(), y_ref, y_bnd, "y_perm")


def test_topk_from_identical_logits_is_bit_exact():
    """On identical fp32 logits (with planted exact ties) the CUDA selection
    equals the oracle's, for every score function without a selection bias."""
    g = torch.Generator().manual_seed(7)
    T, E = 333, 64
    L = torch.randn(T, E, generator=g) * 2
    L[::7, 3] = L[::7, 9]          # exact two-way ties
    L[::11, 10:14] = L[::11, 20:21]  # four-way ties
    Ld = L.cuda()
    for score in ("softmax", "sigmoid", "sqrtsoftplus"):
        for k in (1, 6, 8, 64):
            for renorm in (True, False):
                p = stm.Problem(T=T, H=8, E=E, k=k, I=8, score=score, renormalize=renorm)
                w, sel = stm.topk_from_logits(p, Ld)
                S = oracle.scores(L.double().numpy(), score)
                ref_sel = oracle.select_topk(S, k)
                assert np.array_equal(sel.cpu().numpy(), ref_sel), (score, k)
                ref_w = oracle.topk_weights(S, ref_sel, renorm)
                assert np.abs(w.cpu().double().numpy() - ref_w).max() <= 1e-5


def test_topk_selection_bias_within_tie_margin():
    g = torch.Generator().manual_seed(8)
    T, E, k = 500, 64, 6
    L = torch.randn(T, E, generator=g)
    b = (torch.rand(E, generator=g) * 0.2 - 0.1).float()
    p = stm.Problem(T=T, H=8, E=E, k=k, I=8, score="sqrtsoftplus", bias_mode="select")
    w, sel = stm.topk_from_logits(p, L.cuda(), b.cuda())
    S = oracle.scores(L.double().numpy(), "sqrtsoftplus")
    r = {"keys": S + b.double().numpy()[None, :], "logits": L.double().numpy(),
         "selected_experts": oracle.select_topk(S + b.double().numpy()[None, :], k)}
    cfg = workloads.MoEConfig("t", T, 8, E, k, 8, 0, "bf16", "sqrtsoftplus", "select", True, "none")
    gc.check_selection(cfg, r, sel.cpu().numpy())
    ref_w = oracle.topk_weights(S, sel.cpu().numpy(), True)
    assert np.abs(w.cpu().double().numpy() - ref_w).max() <= 1e-5


@pytest.mark.parametrize("T,E,k", [(1, 1, 1), (5, 3, 2), (257, 8, 2), (1000, 128, 8), (300, 64, 6), (64, 256, 256),
                                   (4096, 128, 8), (8192, 256, 8)])
def test_dispatch_bit_exact(T, E, k):
    """Counting-sort dispatch equals the oracle's stable argsort bit for bit,
    from one token up to a 256-block x 256-expert count matrix."""
    g = torch.Generator().manual_seed(T * 31 + E)
    sel = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).to(torch.int64)
    x = (torch.randn(T, 16, generator=g)).to(torch.bfloat16)
    p = stm.Problem(T=T, H=16, E=E, k=k, I=8)
    d = stm.dispatch(p, sel.cuda(), x.cuda())
    torch.cuda.synchronize()
    dd = gc.assert_dispatch_exact(d, sel.numpy(), E)
    assert torch.equal(d["x_perm"].cpu(), x[torch.from_numpy(dd["sorted_pairs"] // k)])


def test_dispatch_flags_bad_expert_id():
    T, E, k = 50, 8, 2
    g = torch.Generator().manual_seed(1)
    sel = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).to(torch.int64)
    sel[7, 1] = E + 3
    sel[20, 0] = -1
    p = stm.Problem(T=T, H=16, E=E, k=k, I=8)
    ws = stm.new_workspace(p)
    d = stm.dispatch(p, sel.cuda(), None, ws=ws)
    assert stm.read_device_error(ws) == stm.DEVERR_BAD_EXPERT_ID
    assert stm.read_device_error(ws) == 0  # read clears
    pp = d["pair_pos"].cpu().numpy()
    assert pp[7 * k + 1] == -1 and pp[20 * k] == -1
    assert int(d["offsets"][-1]) == T * k - 2
    good = sel.numpy().reshape(-1)
    valid = (good >= 0) & (good < E)
    counts = np.bincount(good[valid], minlength=E)
    assert np.array_equal(d["counts"].cpu().numpy(), counts)


def test_empty_experts_are_never_read():
    """Experts that receive no token get NaN weights; the output must stay
    finite and bit-identical ("feat: Phase 43", empty expert group skipped)."""
    cfg = SMALL["deepseek_v2_lite_zipf"]  # 4 dead experts
    cpu, dev = _inputs(cfg)
    moe = _moe(cfg, dev)
    out, _, sel = moe(dev["x"])
    counts = torch.bincount(sel.reshape(-1).cpu(), minlength=cfg.E)
    dead = torch.nonzero(counts == 0).reshape(-1)
    assert dead.numel() >= 4
    gu, dn = dev["gate_up"].clone(), dev["down"].clone()
    gu[dead] = float("nan")
    dn[dead] = float("nan")
    dev2 = dict(dev, gate_up=gu, down=dn)
    out2, _, _ = _moe(cfg, dev2)(dev["x"])
    torch.cuda.synchronize()
    assert torch.isfinite(out2.float()).all() and torch.equal(out, out2)


def test_down_scaling_is_exact():
    """Doubling every down projection doubles the output bit for bit (bf16
    power-of-two scaling commutes with every rounding on the path)."""
    cfg = SMALL["dsv4_flash_ablation"]
    cpu, dev = _inputs(cfg)
    out, _, _ = _moe(cfg, dev)(dev["x"])
    dev2 = dict(dev, down=dev["down"] * 2, shared_down=dev["shared_down"] * 2)
    out2, _, _ = _moe(cfg, dev2)(dev["x"])
    torch.cuda.synchronize()
    assert torch.equal(out2, out * 2)


def test_repeat_runs_are_bit_identical():
    cfg = SMALL["qwen3_30b_a3b"]
    cpu, dev = _inputs(cfg)
    moe = _moe(cfg, dev)
    a = [t.clone() for t in moe(dev["x"])]
    b = moe(dev["x"])
    torch.cuda.synchronize()
    assert all(torch.equal(u, v) for u, v in zip(a, b))


@pytest.mark.parametrize("name", ["deepseek_v2_lite_zipf", "decode_weight_streaming", "dsv4_flash_ablation",
                                  "pairs_shared_skew", "large_shared_gated"])
def test_two_stream_forward_matches_one_stream(name):
    """The shared expert on a second stream gives the same bits as the
    single-stream forward: a small one beside the whole routed path (its gate
    from its own kernel), a large one (more row x column tiles than half the
    SMs) beside the dispatch only, joined before the routed GEMMs."""
    cfg = EDGE.get(name) or SMALL[name]
    cpu, dev = _inputs(cfg)
    p = stm.Problem.from_config(cfg)
    large = (cfg.T + 127) // 128 * ((cfg.I_shared + 127) // 128) > 74
    assert large == (name in ("pairs_shared_skew", "large_shared_gated"))
    a = stm.SparseMoE(p, dev, overlap_shared=True)
    b = stm.SparseMoE(p, dev, overlap_shared=False)
    assert a.aux is not None and b.aux is None
    ra = [t.clone() for t in a(dev["x"])]
    rb = b(dev["x"])
    torch.cuda.synchronize()
    assert all(torch.equal(u, v) for u, v in zip(ra, rb))


def test_host_pipeline_matches_forward():
    """Batches from pinned host memory through the double-buffered pipeline
    equal direct device forwards, bit for bit."""
    cfg = SMALL["dsv4_flash_ablation"]
    cpu, dev = _inputs(cfg)
    p = stm.Problem.from_config(cfg)
    moe = stm.SparseMoE(p, dev)
    g = torch.Generator().manual_seed(3)
    xs = [(torch.randn(cfg.T, cfg.H, generator=g)).to(torch.bfloat16).pin_memory() for _ in range(5)]
    outs = [torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16).pin_memory() for _ in range(5)]
    pipe = stm.HostPipeline(moe, depth=2)
    for xh, oh in zip(xs, outs):
        pipe.submit(xh, oh)
    pipe.synchronize()
    for xh, oh in zip(xs, outs):
        ref, _, _ = moe(xh.cuda())
        torch.cuda.synchronize()
        assert torch.equal(oh, ref.cpu())


@pytest.mark.parametrize("name,overlap", [("pairs_shared_skew", False), ("pairs_shared_skew", True),
                                           ("decode_weight_streaming", True), ("pairs_tails", False)])
def test_graph_replay_matches_eager_forward(name, overlap):
    """A forward captured as a CUDA graph (with the shared expert on its
    second stream where it overlaps) gives the eager forward's bits, and
    replays pick up new contents of the captured input buffer."""
    cfg = EDGE.get(name) or SMALL[name]
    cpu, dev = _inputs(cfg)
    p = stm.Problem.from_config(cfg)
    moe = stm.SparseMoE(p, dev, overlap_shared=overlap)
    assert (moe.aux is not None) == (overlap and p.shared != "none")
    x = dev["x"].clone()
    gf = stm.GraphedForward(moe, x)
    ref = stm.SparseMoE(p, dev, overlap_shared=False)
    g = torch.Generator(device="cuda").manual_seed(5)
    for it in range(3):
        if it:
            x.copy_(torch.randn(x.shape, generator=g, device="cuda").to(x.dtype))
        got = [t.clone() for t in gf.replay()]
        want = ref(x)
        torch.cuda.synchronize()
        assert all(torch.equal(u, v) for u, v in zip(got, want))
    assert moe.read_device_error() == 0


def test_graph_replay_records_stage_events():
    """Stage events passed at capture become event record nodes: every
    replay records them, in stage order, and the output is unchanged."""
    cfg = EDGE["pairs_tails"]
    cpu, dev = _inputs(cfg)
    p = stm.Problem.from_config(cfg)
    moe = stm.SparseMoE(p, dev)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(stm.STAGES) + 1)]
    for e in evs:
        e.record()
    gf = stm.GraphedForward(moe, dev["x"].clone(), events=evs)
    ref = stm.SparseMoE(p, dev, overlap_shared=False)(dev["x"])[0]
    for _ in range(2):
        out = gf.replay()[0]
        torch.cuda.synchronize()
        times = [evs[i].elapsed_time(evs[i + 1]) for i in range(len(stm.STAGES))]
        assert all(t >= 0 for t in times) and times[stm.STAGES.index("gate_up")] > 0
        assert torch.equal(out, ref)


def test_bounded_wait_reports_timeout_and_context_survives():
    """A pipeline wait that runs out (a barrier nothing arrives on) returns an
    error status the host reads; the CUDA context then still runs a forward."""
    cfg = SMALL["qwen3_30b_a3b"]
    cpu, dev = _inputs(cfg)
    moe = _moe(cfg, dev)
    assert stm.selftest_wait_timeout(moe.ws) == stm.DEVERR_WAIT_TIMEOUT
    assert moe.read_device_error() == 0  # reading cleared the flag
    out, _, _ = moe(dev["x"])
    torch.cuda.synchronize()
    assert moe.read_device_error() == 0 and torch.isfinite(out.float()).all()


def test_empty_batch():
    cfg = SMALL["qwen3_30b_a3b"].replace(T=0)
    cpu, dev = _inputs(cfg)
    out, rw, sel = _moe(cfg, dev)(dev["x"])
    assert out.shape == (0, cfg.H) and sel.shape == (0, cfg.k)


# ----------------------------------------------------------------------------
# Full sizes: all tokens routed and dispatched on the GPU and checked in full
# (routing and dispatch), expert outputs checked on sampled tokens.

@pytest.mark.slow
@pytest.mark.parametrize("name", workloads.CONFIG_ORDER)
def test_full_size_sampled(name):
    cfg = CONFIGS[name]
    r_cpu = workloads.router_inputs(cfg)
    dev = {k: (v.cuda() if v is not None else None) for k, v in r_cpu.items()}
    dev.update(workloads.expert_weights(cfg, "cuda"))
    p = stm.Problem.from_config(cfg)
    moe = stm.SparseMoE(p, dev)
    out, rw, sel = moe(dev["x"])
    torch.cuda.synchronize()
    assert moe.read_device_error() == 0
    gsel = sel.cpu().numpy()
    r = gc.oracle_route(cfg, r_cpu)
    ntie = gc.check_selection(cfg, r, gsel)
    w_ref = oracle.topk_weights(r["scores"], gsel, cfg.renormalize)
    assert np.abs(rw.cpu().double().numpy() - w_ref).max() <= 1e-5
    # dispatch of the whole batch, bit-exact
    d = stm.dispatch(p, sel, None)
    gc.assert_dispatch_exact(d, gsel, cfg.E)
    assert ntie == gc.expected_near_ties(name), f"{name}: {ntie} tokens took the near-tie escape"
    # sampled tokens through the oracle: every token of the small problems,
    # 128 (the first, the last and 126 drawn) of the large ones
    rng = np.random.RandomState(5)
    if cfg.T <= 256:
        rows = np.arange(cfg.T)
    else:
        pick = rng.choice(np.arange(1, cfg.T - 1), 126, replace=False)
        rows = np.unique(np.concatenate([[0, cfg.T - 1], pick]))
        assert rows.size == 128
    x_rows = gc.np64(r_cpu["x"])[rows]
    inp = dict(r_cpu, gate_up=dev["gate_up"], down=dev["down"], shared_gate_up=dev["shared_gate_up"],
               shared_down=dev["shared_down"])
    inp_np = {k: v for k, v in inp.items()}
    o = gc.oracle_forward(cfg, inp_np, x_rows=x_rows, selected=gsel[rows], lazy=True, skip_unrouted=True)
    stats = gc.assert_close(out[torch.from_numpy(rows).cuda()].cpu().double().numpy(), o["out"], cfg.dtype, name)
    print(f"{name}: near-tie tokens {ntie}, sampled {len(rows)} rows, {stats}")
