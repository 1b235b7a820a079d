"""CPU stand-ins for the library's stage calls (route, dispatch,
grouped_swiglu, shared_expert, combine) with the same contracts: fp32
tensors in and out, fp64 arithmetic inside, built from the oracle. Tests of
the multi-rank orchestration install them into the orchestration module of
their own test processes, so that gloo ranks on the CPU can run the exchange
logic end to end; the library itself never uses them."""

import numpy as np
import torch


def install(module) -> None:
    """Replace ``module``'s stage calls (and its workspace allocator) with
    the CPU stand-ins."""
    import oracle

    def f64(t):
        return None if t is None else t.detach().to(torch.float64).numpy()

    def route(p, x, gate_w, bias=None, shared_gate=None, ws=None):
        r = oracle.route(f64(x), f64(gate_w), p.k, p.score, f64(bias), p.bias_mode, p.renormalize)
        gam = None
        if shared_gate is not None:
            gam = torch.from_numpy(oracle.shared_gate_values(f64(x), f64(shared_gate), p.shared)).float()
        return (torch.from_numpy(r["routing_weights"]).float(), torch.from_numpy(r["selected_experts"]), gam)

    def dispatch(p, selected, x=None, ws=None):
        d = oracle.dispatch(selected.numpy(), p.E)
        return {"counts": torch.from_numpy(d["counts"]).int(), "offsets": torch.from_numpy(d["offsets"]).int(),
                "sorted_pairs": torch.from_numpy(d["sorted_pairs"]).int(),
                "pair_pos": torch.from_numpy(d["pair_pos"]).int(),
                "x_perm": None if x is None else x[torch.from_numpy(d["sorted_pairs"] // p.k)]}

    def grouped_swiglu(p, x_perm, offsets, gate_up, down, routing_weights=None, sorted_pairs=None, ws=None):
        assert tuple(gate_up.shape) == (p.E, 2 * p.I, p.H) and tuple(down.shape) == (p.E, p.H, p.I)
        xp, off = f64(x_perm), offsets.numpy()
        w = f64(routing_weights).reshape(-1)
        y = np.zeros((p.T * p.k, p.H))
        for e in range(p.E):
            a, b = off[e], off[e + 1]
            if b > a:
                rows = oracle.swiglu_mlp(xp[a:b], f64(gate_up[e]), f64(down[e]))
                y[a:b] = w[sorted_pairs[a:b].numpy()][:, None] * rows
        return torch.from_numpy(y).float()

    def shared_expert(p, x, shared_gate_up, shared_down, gamma=None, ws=None):
        assert tuple(shared_gate_up.shape) == (2 * p.I_shared, p.H)
        s = oracle.swiglu_mlp(f64(x), f64(shared_gate_up), f64(shared_down))
        if gamma is not None:
            s = f64(gamma)[:, None] * s
        return torch.from_numpy(s).float()

    def combine(p, y_perm, pair_pos, shared_out=None):
        y, pp = f64(y_perm), pair_pos.numpy().reshape(p.T, p.k)
        out = np.zeros((p.T, p.H))
        for j in range(p.k):
            ok = pp[:, j] >= 0
            out[ok] += y[pp[ok, j]]
        if shared_out is not None:
            out += f64(shared_out)
        return torch.from_numpy(out).float()

    def new_workspace(p, device="cpu"):  # the stand-ins keep no state in a workspace
        return torch.zeros(256, dtype=torch.uint8)

    for name, fn in dict(route=route, dispatch=dispatch, grouped_swiglu=grouped_swiglu,
                         shared_expert=shared_expert, combine=combine, new_workspace=new_workspace).items():
        if hasattr(module, name):
            setattr(module, name, fn)
