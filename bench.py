"""Benchmark of the B200 sparse top-k MoE FFN forward.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config NAME]

A step is one whole forward (route, dispatch, grouped SwiGLU, shared expert,
combine) over one batch of synthetic tokens. Default workload: the
DSV4-Flash-ablation-shaped problem (T=8192, H=4096, 64 routed experts + 1
shared, top-6 sqrtsoftplus with an fp32 selection bias, I=2048, bf16), the
largest of the named problems. With N > 1 (torchrun, one process per GPU)
every rank runs its own batch with the same weights (weak scaling, no
collective on the data path); the time is the max over ranks.

Rank 0 prints one JSON line. ``value`` is tokens/s with inputs resident in
HBM; ``e2e`` is the same metric through the public API from pinned host
memory (host->device copy of x and device->host copy of out inside the timed
region); ``roofline`` describes the dominant kernel (the routed gate_up
GEMM), timed with CUDA events on its stream inside graph replays, against its
algorithmic FLOPs and bytes (active expert weights read once, x read once);
``forward_roofline`` does the same for the whole forward; ``per_config``
repeats the measurement on every named problem; ``cpu_baseline`` is the fp64
oracle timed on a bounded token sample on the host cores. ``--impl
reference`` times that oracle as the reference arm.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads  # noqa: E402

DEFAULT_CONFIG = "dsv4_flash_ablation"
L2_BYTES = 126 * 1024 * 1024


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ----------------------------------------------------------------------------
# clocks

class ClockSampler:
    """NVML sampling of SM clock and clock-event reasons on a thread."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.samples, self.reasons, self.ok = [], 0, False
        self.period = period_s
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= int(self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        rs = [name for bit, name in self.REASONS.items() if self.reasons & bit and name != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz, "reasons": rs,
                "samples": len(self.samples)}


# ----------------------------------------------------------------------------
# workload accounting (algorithmic work only: the active experts' weights read
# once, x read once, out written once; the implementation's own intermediates
# x_perm, h and y rows are not counted)

def active_experts(sel: torch.Tensor, E: int) -> int:
    return int((torch.bincount(sel.reshape(-1), minlength=E) > 0).sum().item())


def flops_and_bytes(cfg, n_active: int):
    """Algorithmic FLOPs and bytes of the whole forward and of its two grouped
    GEMMs, for ``n_active`` experts that receive at least one row."""
    P = cfg.T * cfg.k
    es = 4 if cfg.dtype == "f32" else 2
    f_routed = 6.0 * cfg.H * cfg.I * P
    f_shared = 6.0 * cfg.H * cfg.I_shared * cfg.T if cfg.shared != "none" else 0.0
    f_router = 2.0 * cfg.T * cfg.H * cfg.E
    x_bytes = cfg.T * cfg.H * es
    # routed gate_up GEMM: 4*H*I flops per (token, expert) row; the active
    # experts' gate_up weights read once and x read once
    gu_flops = 4.0 * cfg.H * cfg.I * P
    gu_bytes = n_active * 2 * cfg.I * cfg.H * es + x_bytes
    # routed down GEMM: 2*H*I flops per row; the active down weights once and
    # the output written once
    dn_flops = 2.0 * cfg.H * cfg.I * P
    dn_bytes = n_active * cfg.I * cfg.H * es + x_bytes
    # whole forward: active weights once (+ router and shared weights), x in, out back
    w_bytes = n_active * 3 * cfg.I * cfg.H * es + cfg.E * cfg.H * es
    if cfg.shared != "none":
        w_bytes += 3 * cfg.I_shared * cfg.H * es
    min_bytes = w_bytes + 2 * x_bytes
    return {"active_flops": f_routed + f_shared, "router_flops": f_router, "gate_up_flops": gu_flops,
            "gate_up_bytes": gu_bytes, "down_flops": dn_flops, "down_bytes": dn_bytes, "min_bytes": min_bytes,
            "weight_bytes": w_bytes}


def total_weight_bytes(cfg) -> int:
    """Bytes of every expert weight of the problem (all E routed + shared)."""
    es = 4 if cfg.dtype == "f32" else 2
    b = cfg.E * 3 * cfg.I * cfg.H * es + cfg.E * cfg.H * es
    if cfg.shared != "none":
        b += 3 * cfg.I_shared * cfg.H * es
    return b


FP32_LANES_PER_SM = 128  # FFMA lanes per Blackwell SM (4 sub-partitions x 32)
NUM_SMS = 148


def ffma_peak_tflops(mhz: float) -> float:
    """fp32 FFMA peak from the unit counts at the given SM clock."""
    return NUM_SMS * FP32_LANES_PER_SM * 2 * mhz * 1e6 / 1e12


def roofline_entry(flops: float, nbytes: float, ms: float, pk: dict, dtype: str, mhz: float = None) -> dict:
    """Bound, achieved and fraction of one kernel (or of the whole forward)
    from its algorithmic FLOPs and bytes and its measured time: the bound is
    the larger of FLOPs / tensor peak (burst: the kernels are timed inside
    sub-10-ms replays) and bytes / HBM copy bandwidth; bf16 contractions use
    the measured bf16 peak, fp32 ones the FFMA peak from the unit counts."""
    s = ms / 1e3
    if dtype == "f32":
        peak_t = ffma_peak_tflops(mhz or 1965.0)
        t_src = f"148 SMs x 128 FFMA lanes x 2 flop x {mhz or 1965.0:.0f} MHz"
    else:
        peak_t = pk["bf16_tflops"]
        t_src = pk["source"] + " bf16 (burst)"
    t_tensor = flops / (peak_t * 1e12)
    t_hbm = nbytes / (pk["hbm_gbs"] * 1e9)
    if t_tensor >= t_hbm:
        e = {"bound": "alu" if dtype == "f32" else "tensor", "achieved": flops / s / 1e12, "peak": peak_t,
             "unit": "TFLOP/s", "peak_source": t_src}
        if dtype != "f32":
            e["frac_of_sustained"] = e["achieved"] / pk["bf16_tflops_sustained"]
    else:
        e = {"bound": "hbm", "achieved": nbytes / s / 1e9, "peak": pk["hbm_gbs"], "unit": "GB/s",
             "peak_source": pk["source"] + " copy bandwidth"}
        e["frac_of_nominal_8000gbs"] = e["achieved"] / 8000.0
    e["frac"] = e["achieved"] / e["peak"]
    e["t_roof_ms"] = 1e3 * max(t_tensor, t_hbm)
    e["algorithmic"] = {"flops": flops, "bytes": nbytes, "ms": ms}
    return e


GEMM_SOURCES = ("gemm_tc.cu", "gemm_tc2.cu", "tc_ptx.cuh", "tc_epilogue.cuh", "tiles.cuh", "common.cuh")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")


def kernel_source_hash() -> str:
    """sha256 over the sources of the grouped-GEMM kernels."""
    h = hashlib.sha256()
    for name in GEMM_SOURCES:
        with open(os.path.join(ROOT, "sparse_top_mixture_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def recorded_traffic(cfg_name: str, kernel: str = "gate_up"):
    """Per-launch DRAM traffic (read + write bytes) of a grouped GEMM from the
    ncu record in ``profiles/traffic.json``, if the kernel sources are
    unchanged since it was taken; else None."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        entries = json.load(f).get("entries", [])
    sha = kernel_source_hash()
    for e in entries:
        if e.get("config") == cfg_name and e.get("kernel") == kernel and e.get("kernel_sources_sha256") == sha:
            return float(e["bytes_per_launch"])
    return None


# ----------------------------------------------------------------------------
# CPU oracle timing (baseline and reference arm)

def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = [i.get("num_threads") for i in info if i.get("user_api") == "blas"]
        return int(max(n)) if n else None
    except Exception:
        return None


class OracleTimer:
    """Times the fp64 dense-masked oracle on a sample of tokens (each token
    runs through every routed expert, as the oracle is defined)."""

    def __init__(self, cfg, dev_inputs):
        import numpy as np
        self.np = np
        self.cfg = cfg
        f64 = workloads.to_numpy64
        self.x = f64(dev_inputs["x"])
        self.gw = f64(dev_inputs["gate_w"])
        self.bias = f64(dev_inputs.get("bias"))
        self.sg = f64(dev_inputs.get("shared_gate"))
        self.sgu = f64(dev_inputs.get("shared_gate_up"))
        self.sdn = f64(dev_inputs.get("shared_down"))
        # expert weights converted once (input preparation, outside timing)
        self.gu = [f64(dev_inputs["gate_up"][e]) for e in range(cfg.E)]
        self.dn = [f64(dev_inputs["down"][e]) for e in range(cfg.E)]

    def run(self, n_tokens: int, start: int = 0) -> float:
        import oracle
        c = self.cfg
        rows = (start + self.np.arange(n_tokens)) % c.T
        t0 = time.perf_counter()
        oracle.moe_forward(self.x[rows], self.gw, self.gu, self.dn, k=c.k, score=c.score,
                           renormalize=c.renormalize, bias=self.bias, bias_mode=c.bias_mode, shared=c.shared,
                           shared_gate_up=self.sgu, shared_down=self.sdn, shared_gate=self.sg)
        return time.perf_counter() - t0

    def calibrate(self, target_s: float, max_tokens: int) -> int:
        n = 4
        t = self.run(n)
        while t < target_s / 4 and n < max_tokens:
            n = min(max_tokens, n * 4)
            t = self.run(n)
        per = t / n
        return int(max(1, min(max_tokens, target_s / max(per, 1e-9))))


def cpu_baseline(cfg, dev_inputs, target_s: float = 12.0):
    need = 8.0 * total_weight_bytes(cfg) / (4 if cfg.dtype == "f32" else 2)
    have = host_memory_available()
    if have < 1.5 * need:
        return {"value": None, "unit": "tokens/s", "kind": "oracle",
                "skipped": f"fp64 weights need ~{need / 1e9:.1f} GB of host memory, {have / 1e9:.1f} GB available"}
    ot = OracleTimer(cfg, dev_inputs)
    n = ot.calibrate(target_s, cfg.T)
    t = ot.run(n)
    return {"value": n / t, "unit": "tokens/s", "cores": _blas_threads() or os.cpu_count(), "kind": "oracle",
            "sample": f"{n} of the {cfg.T} tokens of {cfg.name}, fp64 dense-masked (all {cfg.E} experts per token), "
                      f"{t:.1f} s"}


# ----------------------------------------------------------------------------

def backward_flops(cfg) -> float:
    """Algorithmic FLOPs of one backward (moe_backward): per routed pair the
    recomputed [g | u] (4HI), dhu = dout Wd (2HI), dx rows (4HI) and the two
    weight gradients (2HI + 4HI); the router's logits, dgate_w and dx (2EH
    each per token); the shared expert like one routed pair per token."""
    P = cfg.T * cfg.k
    return 16.0 * P * cfg.H * cfg.I + 6.0 * cfg.T * cfg.E * cfg.H + 16.0 * cfg.T * cfg.H * cfg.I_shared


def backward_bytes(cfg, active: int, es: int) -> float:
    """Algorithmic bytes of one backward: the active experts' weights, the
    router's and the shared expert's read once (``es`` bytes an element), x
    and dout read once, every weight gradient (all E experts: an expert
    without rows gets zeros) and dx written once in fp32."""
    w_routed = 3.0 * cfg.H * cfg.I
    w_other = cfg.E * cfg.H + 3.0 * cfg.H * cfg.I_shared + (cfg.H if cfg.shared == "sigmoid_gated" else 0)
    reads = (active * w_routed + w_other) * es + 2.0 * cfg.T * cfg.H * es
    writes = (cfg.E * w_routed + w_other + (cfg.E if cfg.bias_mode == "logit" else 0)) * 4 + cfg.T * cfg.H * 4
    return reads + writes


def host_memory_available() -> float:
    """Bytes this process may still allocate: the smaller of the host's
    available memory and what its cgroup (v2 or v1) limit leaves."""
    import psutil
    avail = float(psutil.virtual_memory().available)
    for limit_f, usage_f in (("/sys/fs/cgroup/memory.max", "/sys/fs/cgroup/memory.current"),
                             ("/sys/fs/cgroup/memory/memory.limit_in_bytes",
                              "/sys/fs/cgroup/memory/memory.usage_in_bytes")):
        try:
            with open(limit_f) as f:
                lim = f.read().strip()
            with open(usage_f) as f:
                used = float(f.read().strip())
        except OSError:
            continue
        if lim.isdigit():
            avail = min(avail, float(lim) - used)
    return avail


def backward_cpu_baseline(cfg32, inp, dout, target_s: float = 8.0) -> dict:
    """The fp64 backward oracle, as it stands, on the first n tokens of the
    fp32 workload (its own top-k choice), n sized so that one call takes about
    ``target_s``. Each call also builds the oracle's gradient of every expert
    weight, a fixed cost that dominates small samples; n is sized from two
    short runs that separate it from the per-token cost."""
    import numpy as np

    import oracle.backward as ob
    # fp64 weights, the oracle's per-expert weight gradients and their stacked copy
    need = 3.0 * 8 * (cfg32.E * 3 * cfg32.I * cfg32.H + 3 * cfg32.I_shared * cfg32.H)
    have = host_memory_available()
    if have < 1.5 * need:
        return {"value": None, "unit": "tokens/s", "kind": "oracle",
                "skipped": f"needs ~{need / 1e9:.1f} GB of host memory, {have / 1e9:.1f} GB available"}
    f64 = workloads.to_numpy64
    x, do = f64(inp["x"]), f64(dout)
    gw, bias = f64(inp["gate_w"]), f64(inp.get("bias"))
    gu = [f64(inp["gate_up"][e]) for e in range(cfg32.E)]
    dn = [f64(inp["down"][e]) for e in range(cfg32.E)]
    sgu, sdn, sg = f64(inp.get("shared_gate_up")), f64(inp.get("shared_down")), f64(inp.get("shared_gate"))

    def run(n: int) -> float:
        t0 = time.perf_counter()
        ob.moe_backward(x[:n], gw, gu, dn, do[:n], k=cfg32.k, score=cfg32.score, renormalize=cfg32.renormalize,
                        bias=bias, bias_mode=cfg32.bias_mode, shared=cfg32.shared, shared_gate_up=sgu,
                        shared_down=sdn, shared_gate=sg)
        return time.perf_counter() - t0

    # t(n) = fixed + per_token * n, from two short runs; then one run of ~target_s
    t_small, t_big = run(4), run(64)
    per = max((t_big - t_small) / 60.0, 1e-9)
    fixed = max(t_small - 4 * per, 0.0)
    n = int(np.clip((target_s - fixed) / per, 4, cfg32.T))
    t = run(n)
    return {"value": n / t, "unit": "tokens/s", "cores": _blas_threads() or os.cpu_count(), "kind": "oracle",
            "sample": f"backward of the first {n} of the {cfg32.T} tokens of {cfg32.name} in fp64 "
                      f"(oracle.backward, its own top-k choice), {t:.1f} s"}


def measure_backward(cfg, local: int, steps: int = 5, cpu: bool = False, dtype: str = "bf16") -> dict:
    """The backward on the given workload's shapes in ``dtype`` (bf16: the
    tensor-core path; f32: the SIMT path), timed with CUDA events on the
    current stream, as eager C-ABI calls (``eager_ms``) and as replays of the
    same call captured in a CUDA graph (``ms``); its roofline takes the larger
    of its FLOPs at the bf16 (or FFMA, at the sampled SM clock) peak and its
    algorithmic bytes at the HBM bandwidth. With ``cpu``, the backward oracle
    timed on the host beside it on the same inputs, widened to fp64."""
    import sparse_top_mixture_b200 as stm
    c = cfg.replace(dtype=dtype)
    inp = workloads.generate(c, "cuda")
    p = stm.Problem.from_config(c)
    moe = stm.SparseMoE(p, inp)
    out, _, sel = moe(inp["x"])
    dout = torch.randn(out.shape, generator=torch.Generator("cuda").manual_seed(7), device="cuda").to(out.dtype)
    ws = torch.zeros(stm.backward_workspace_size(p), dtype=torch.uint8, device="cuda")
    grads = stm.backward(p, inp, inp["x"], dout, sel, ws=ws)
    for _ in range(2):
        stm.backward(p, inp, inp["x"], dout, sel, ws=ws, out=grads)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # eager: one C-ABI call per step (its ~25 launches issued from the host)
    a.record(stream)
    for _ in range(steps):
        stm.backward(p, inp, inp["x"], dout, sel, ws=ws, out=grads)
    b.record(stream)
    torch.cuda.synchronize()
    eager_ms = a.elapsed_time(b) / steps
    # the same call captured once as a CUDA graph and replayed, as the forward is timed
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        stm.backward(p, inp, inp["x"], dout, sel, ws=ws, out=grads)
    for _ in range(2):
        graph.replay()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        a.record(stream)
        for _ in range(steps):
            graph.replay()
        b.record(stream)
        torch.cuda.synchronize()
    del graph
    if stm.read_device_error(ws) != 0:
        raise RuntimeError("device error flag set during the backward")
    ms = a.elapsed_time(b) / steps
    fl = backward_flops(c)
    ck = clk.summary()
    mhz = ck["sm_mhz"] or ck["sm_max_mhz"] or 1965
    active = int(torch.unique(sel[(sel >= 0) & (sel < c.E)]).numel())
    nbytes = backward_bytes(c, active, 4 if dtype == "f32" else 2)
    roof = roofline_entry(fl, nbytes, ms, peaks(), dtype, mhz)
    res = {"workload": f"{cfg.name} shapes in {dtype} (T={c.T}, H={c.H}, E={c.E}, k={c.k}, I={c.I}, "
                       f"I_shared={c.I_shared})",
           "dtype": dtype, "ms": ms, "launch": "cuda_graph", "eager_ms": eager_ms,
           "tokens_per_s": c.T / (ms / 1e3), "steps": steps, "flops": fl,
           "active_experts": active, "tflops": fl / (ms / 1e3) / 1e12, **roof, "traffic": None, "clocks": ck}
    if cpu:
        try:
            res["cpu_baseline"] = backward_cpu_baseline(cfg.replace(dtype="f32"), inp, dout.float())
        except Exception as exc:  # the host baseline never costs the bench line
            res["cpu_baseline"] = {"value": None, "error": repr(exc)[:200]}
    del moe, grads, ws, inp
    torch.cuda.empty_cache()
    return res


def init_dist(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
    return rank, local, world


def dist_max(v: float, world: int) -> float:
    """Max of v over ranks (the job's time is the slowest rank's)."""
    if world == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, tokens_per_rank: int, steps: int, elapsed_ms_max: float) -> float:
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
    return world * tokens_per_rank * steps / (elapsed_ms_max / 1e3)


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def make_inputs(cfg, rank: int):
    r = workloads.router_inputs(cfg, rank=rank)
    dev = {k: (v.cuda() if v is not None else None) for k, v in r.items()}
    dev.update(workloads.expert_weights(cfg, "cuda"))
    return r, dev


def metric_name() -> str:
    return "MoE FFN tokens/s and active-expert TFLOP/s (fraction of bf16/HBM roofline)"


def l2_policy(cfg) -> str:
    """How the timed steps keep L2 from serving the next step's inputs."""
    wb = total_weight_bytes(cfg)
    if wb > L2_BYTES:
        return f"inputs larger than L2: {wb / 1e9:.2f} GB of expert weights > 126 MB L2, no flush"
    return f"L2 flushed between timed steps ({FLUSH_BYTES >> 20} MB write); weights {wb / 1e6:.1f} MB"


def config_dict(cfg) -> dict:
    """The workload's name and shape (the same for both arms of the bench)."""
    return {"workload": cfg.name, "T": cfg.T, "H": cfg.H, "E": cfg.E, "k": cfg.k, "I": cfg.I,
            "I_shared": cfg.I_shared, "score": cfg.score, "bias_mode": cfg.bias_mode,
            "renormalize": cfg.renormalize, "shared": cfg.shared, "seed": cfg.seed, "l2": l2_policy(cfg)}


def run_reference(args, cfg, rank, world):
    """Reference arm: the fp64 oracle on the host cores, rank 0 only."""
    if rank != 0:
        return
    torch.manual_seed(0)
    r = workloads.router_inputs(cfg)
    w = workloads.expert_weights(cfg, "cuda" if torch.cuda.is_available() else "cpu")
    ot = OracleTimer(cfg, dict(r, **w))
    del w
    n = ot.calibrate(max(1.0, 60.0 / max(1, args.steps + args.warmup)), cfg.T)
    for i in range(args.warmup):
        ot.run(n, start=i * n)
    total = 0.0
    for i in range(args.steps):
        total += ot.run(n, start=(args.warmup + i) * n)
    value = n * args.steps / total
    line = {"impl": "reference", "metric": metric_name(), "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_dict(cfg),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "kind": "oracle",
                             "cores": _blas_threads() or os.cpu_count(),
                             "sample": f"{n} tokens per step of {cfg.name}, fp64 dense-masked"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


FLUSH_BYTES = 256 << 20


class ForwardRun:
    """One problem's inputs, module and graphs on this rank's GPU, and the
    device-timed measurement of its forward."""

    def __init__(self, cfg, rank: int, graph: bool = True):
        import sparse_top_mixture_b200 as stm
        self.stm = stm
        self.cfg = cfg
        self.r_cpu, self.dev = make_inputs(cfg, rank)
        self.p = stm.Problem.from_config(cfg)
        self.moe = stm.SparseMoE(self.p, self.dev)
        dt = self.p.torch_dtype
        self.x = self.dev["x"]
        self.out = torch.empty(cfg.T, cfg.H, dtype=dt, device="cuda")
        self.rw = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device="cuda")
        self.sel = torch.empty(cfg.T, cfg.k, dtype=torch.int64, device="cuda")
        self.use_graph = graph
        self.flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda") \
            if total_weight_bytes(cfg) <= L2_BYTES else None

    def warm(self, warmup: int):
        for _ in range(warmup):
            self.moe.forward(self.x, self.out, self.rw, self.sel)
        torch.cuda.synchronize()
        if self.moe.read_device_error() != 0:
            raise RuntimeError(f"{self.cfg.name}: device error flag set during warm-up")
        self.n_active = active_experts(self.sel, self.cfg.E)
        self.fb = flops_and_bytes(self.cfg, self.n_active)
        # The timed steps replay the forward as one CUDA graph (the same kernels
        # on the same buffers as the eager call, launched as one graph).
        self.graphed = self.stm.GraphedForward(self.moe, self.x, self.out, self.rw, self.sel) \
            if self.use_graph else None
        for _ in range(warmup):
            self.step()
        torch.cuda.synchronize()

    def step(self):
        if self.graphed is not None:
            self.graphed.replay()
        else:
            self.moe.forward(self.x, self.out, self.rw, self.sel)

    def timed(self, steps: int, local: int, world: int):
        """Device time of `steps` forwards (ms, max over ranks) and the clocks
        sampled meanwhile. Problems whose weights fit in L2 flush it between
        steps (outside the timed intervals)."""
        stream = torch.cuda.current_stream()
        barrier(world)
        torch.cuda.synchronize()
        with ClockSampler(local) as clocks:
            if self.flush is None:
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                for _ in range(steps):
                    self.step()
                b.record(stream)
                torch.cuda.synchronize()
                ms = a.elapsed_time(b)
            else:
                ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                      for _ in range(steps)]
                for a, b in ev:
                    self.flush.zero_()
                    a.record(stream)
                    self.step()
                    b.record(stream)
                torch.cuda.synchronize()
                ms = sum(a.elapsed_time(b) for a, b in ev)
        barrier(world)
        if self.moe.read_device_error() != 0:
            raise RuntimeError(f"{self.cfg.name}: device error flag set during the timed region")
        return dist_max(ms, world), clocks.summary()

    def stages(self, steps: int, local: int):
        """Median device time of each stage: the same forward with CUDA events
        between the stages (recorded inside the graph at every replay), one
        step at a time."""
        stm = self.stm
        stream = torch.cuda.current_stream()
        nst = len(stm.STAGES) + 1
        sev = [torch.cuda.Event(enable_timing=True) for _ in range(nst)]
        for e in sev:  # torch creates the CUDA event on its first record
            e.record(stream)
        torch.cuda.synchronize()
        staged = stm.GraphedForward(self.moe, self.x, self.out, self.rw, self.sel, events=sev) \
            if self.use_graph else None
        samples = []
        with ClockSampler(local) as clk:
            for _ in range(steps):
                if self.flush is not None:
                    self.flush.zero_()
                if staged is not None:
                    staged.replay()
                else:
                    self.moe.forward(self.x, self.out, self.rw, self.sel, events=sev)
                torch.cuda.synchronize()
                samples.append([sev[si].elapsed_time(sev[si + 1]) for si in range(nst - 1)])
        stage_ms = {name: statistics.median(row[si] for row in samples) for si, name in enumerate(stm.STAGES)}
        return stage_ms, statistics.median(sum(row) for row in samples), clk.summary()

    def release(self):
        for name in ("graphed", "moe", "dev", "x", "out", "rw", "sel", "flush"):
            if hasattr(self, name):
                delattr(self, name)
        torch.cuda.synchronize()
        torch.cuda.empty_cache()


def forward_summary(cfg, fb, n_active, ms_per_step, stage_ms, clocks, pk, world: int = 1) -> dict:
    """Throughput, the whole forward's roofline fraction and the dominant
    kernel's (the routed gate_up GEMM) from algorithmic work and device times."""
    mhz = clocks.get("sm_mhz") or clocks.get("sm_max_mhz") or 1965.0
    whole = roofline_entry(fb["active_flops"] + fb["router_flops"], fb["min_bytes"], ms_per_step, pk, cfg.dtype, mhz)
    gu = roofline_entry(fb["gate_up_flops"], fb["gate_up_bytes"], stage_ms["gate_up"], pk, cfg.dtype, mhz)
    dn = roofline_entry(fb["down_flops"], fb["down_bytes"], stage_ms["down"], pk, cfg.dtype, mhz)
    return {
        "workload": cfg.name, "ms_per_step": ms_per_step, "tokens_per_s": world * cfg.T / (ms_per_step / 1e3),
        "active_expert_tflops": world * fb["active_flops"] / (ms_per_step / 1e3) / 1e12,
        "active_experts": n_active, "forward_roofline": whole,
        "dominant_kernel": dict(gu, kernel="gate_up"), "down_kernel": dict(dn, kernel="down"),
        "stage_ms": stage_ms, "clocks": clocks,
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default=DEFAULT_CONFIG, choices=list(workloads.CONFIGS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=None)
    ap.add_argument("--no-graph", action="store_true", help="launch each kernel from the host every step")
    ap.add_argument("--no-backward", action="store_true", help="skip the backward measurements (bf16 and fp32)")
    ap.add_argument("--no-per-config", action="store_true", help="skip the per_config block (the other workloads)")
    ap.add_argument("--per-config-steps", type=int, default=50)
    ap.add_argument("--backward-only", action="store_true",
                    help="profiling only: run just the bf16 backward measurement on --config and print it")
    ap.add_argument("--tokens", type=int, default=None,
                    help="profiling only: override T (the line then names a reduced workload, not a bench line)")
    ap.add_argument("--experts", type=int, default=None,
                    help="profiling only: override E (with --tokens, keeps rows per expert for smaller captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    cfg = workloads.CONFIGS[args.config]
    if args.tokens is not None or args.experts is not None:
        T, E = args.tokens or cfg.T, args.experts or cfg.E
        cfg = cfg.replace(name=f"{cfg.name}@T{T}E{E}", T=T, E=E, bias_kind="none" if cfg.bias_kind == "zipf"
                          else cfg.bias_kind, bias_mode="none" if cfg.bias_kind == "zipf" else cfg.bias_mode)
        args.no_per_config = True
    rank, local, world = init_dist(args.gpus)
    if args.impl == "reference":
        run_reference(args, cfg, rank, world)
        if world > 1:
            barrier(world)
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    import sparse_top_mixture_b200 as stm
    if not os.path.exists(stm.LIB_PATH):  # the CUDA library is built in-tree
        from sparse_top_mixture_b200 import build
        build.build()
    pk = peaks()
    if args.backward_only:  # not a bench line: the backward block alone, for profiling captures
        print(json.dumps({"backward_only": measure_backward(cfg, local, steps=args.steps, dtype="bf16")}), flush=True)
        return

    run = ForwardRun(cfg, rank, graph=not args.no_graph)
    run.warm(args.warmup)
    elapsed_ms, clocks = run.timed(args.steps, local, world)
    stage_steps = min(args.steps, 100)
    stage_ms, staged_ms, stage_clocks = run.stages(stage_steps, local)
    ms_per_step = elapsed_ms / args.steps
    fb, n_active = run.fb, run.n_active
    summ = forward_summary(cfg, fb, n_active, ms_per_step, stage_ms, clocks, pk, world)
    tokens_per_s = job_throughput(world, cfg.T, args.steps, elapsed_ms)
    moe, p, x, out = run.moe, run.p, run.x, run.out
    stream = torch.cuda.current_stream()
    dt = p.torch_dtype

    # e2e: pinned host x in, host out back, through the public API. Batches go
    # through a three-slot HostPipeline: every step still copies its own input
    # in and its result out inside the timed region, overlapped with the
    # neighbouring steps' compute.
    e2e_steps = args.e2e_steps or max(4, min(args.steps, 50))
    x_host = [run.r_cpu["x"].pin_memory(), run.r_cpu["x"].clone().pin_memory(), run.r_cpu["x"].clone().pin_memory()]
    out_host = [torch.empty(cfg.T, cfg.H, dtype=dt).pin_memory() for _ in range(3)]
    pipe = stm.HostPipeline(moe, depth=3)
    for i in range(4):
        pipe.submit(x_host[i % 3], out_host[i % 3])
    pipe.synchronize()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(e2e_steps):
        pipe.submit(x_host[i % 3], out_host[i % 3])
    for slot in pipe.slots:
        stream.wait_stream(slot["stream"])
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = dist_max(e0.elapsed_time(e1), world)
    e2e_tps = job_throughput(world, cfg.T, e2e_steps, e2e_ms)
    del pipe

    # The balancer's deferred bias update (stash this forward's counts, then
    # one sign-controller step), timed on its own: two one-block launches.
    bal_stash = torch.zeros(cfg.E, dtype=torch.int64, device="cuda")
    bal_bias = torch.zeros(cfg.E, dtype=torch.float32, device="cuda")
    counts = moe.forward_counts()
    b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(3):
        stm.bias_stash(p, counts, bal_stash)
        stm.bias_update(p, bal_stash, bal_bias, 1e-3)
    b0.record(stream)
    for _ in range(100):
        stm.bias_stash(p, counts, bal_stash)
        stm.bias_update(p, bal_stash, bal_bias, 1e-3)
    b1.record(stream)
    torch.cuda.synchronize()
    balance_us = b0.elapsed_time(b1) * 1e3 / 100

    roof = dict(summ["dominant_kernel"])
    roof["traffic"] = recorded_traffic(cfg.name, "gate_up")
    roof["kernel"] = {0: "simt_grouped_kernel<gate_up>", 1: "tc_grouped_gemm_kernel<gate_up>",
                      2: "tc2_grouped_gemm_kernel<gate_up> (CTA pairs)"}[stm.gemm_path(p)]
    if roof["traffic"] is not None:
        roof["traffic_over_algorithmic"] = roof["traffic"] / roof["algorithmic"]["bytes"]

    line = {
        "metric": metric_name(), "value": tokens_per_s, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic (seeded; weights ~N(0,1/fan_in))",
        "config": config_dict(cfg),
        "parallelism": f"replicas x{world} (independent batches, no collective on the data path)",
        "active_expert_tflops": summ["active_expert_tflops"],
        "forward_roofline_frac": summ["forward_roofline"]["frac"],
        "forward_roofline": summ["forward_roofline"],
        "active_experts": n_active,
        "stage_ms": stage_ms,
        "launch": "cuda_graph" if run.graphed is not None else "eager",
        "bias_update_us": balance_us,
        "stage_pass_ms_per_step": staged_ms,
        "stage_clocks": stage_clocks,
        "roofline": roof,
        "down_kernel": summ["down_kernel"],
        "e2e": {"value": e2e_tps, "unit": "tokens/s", "h2d_bytes_per_step": x.numel() * x.element_size(),
                "d2h_bytes_per_step": out.numel() * out.element_size(), "steps": e2e_steps,
                "how": "HostPipeline depth 3: per step H2D of x, forward (graph replay), D2H of out on the step's stream"},
        "gpu_launches": stm.launches_per_forward(p, two_streams=moe.aux is not None) * args.steps,
        "clocks": clocks,
    }
    cpu_inputs = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu_inputs = dict(run.r_cpu, **{k: run.dev[k] for k in ("gate_up", "down", "shared_gate_up", "shared_down")})
    run.release()
    del moe, x, out, counts

    if world == 1 and not args.no_per_config:
        # Every named workload, each measured the same way (graph replays,
        # per-stage events) on this GPU, one after the other.
        per = {}
        for name in workloads.CONFIG_ORDER:
            if name == cfg.name:
                per[name] = dict(summ, steps=args.steps)
                continue
            c = workloads.CONFIGS[name]
            r = ForwardRun(c, rank, graph=not args.no_graph)
            r.warm(5)
            ms, clk = r.timed(args.per_config_steps, local, world)
            st, _, _ = r.stages(min(args.per_config_steps, 20), local)
            per[name] = dict(forward_summary(c, r.fb, r.n_active, ms / args.per_config_steps, st, clk, pk),
                             steps=args.per_config_steps, l2=l2_policy(c))
            r.release()
        line["per_config"] = per
    if world == 1 and not args.no_backward:
        # the backward on the Qwen3-shaped problem: bf16 on the tensor cores
        # (with the oracle's host baseline), and the fp32 SIMT path beside it
        bw_cfg = workloads.CONFIGS["qwen3_30b_a3b"]
        line["backward"] = measure_backward(bw_cfg, local, cpu=not args.no_cpu_baseline, dtype="bf16")
        line["backward_f32"] = measure_backward(bw_cfg, local, dtype="f32")
    if cpu_inputs is not None:
        line["cpu_baseline"] = cpu_baseline(cfg, cpu_inputs)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        barrier(world)
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
