"""Oracle of the aux-loss-free balancer's bias update (sign controller).

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import or run anything under
``oracle/``. The CUDA library and its Python binding never import it.

What the page fixes ("Sparse MoE FFN for DFlash-family drafters", What's
here, MoEGate, and the balance-update bullet after SparseMoE; Tests,
balance-update semantics):

* the balancing bias is an fp32 buffer, moved by a sign controller from the
  expert loads summed over all ranks, never by gradients;
* updates are deferred: a forward stashes its routing counts and the update
  is applied before the next forward; applying twice in a row changes the
  bias once (the second apply finds nothing stashed);
* the step size is a configured update rate.

Readings taken where the page is silent:

* loads L[e] = routing counts stashed since the last update, summed over
  data-parallel ranks; the target is their mean m = sum(L) / E;
* bias[e] += rate * sign(m - L[e]) with sign(0) = 0: an expert above the mean
  is pushed down, one below it up, one exactly at it keeps its bias;
* the addition is one fp32 add (the bias stays fp32); the comparison with the
  mean is exact (E * L[e] against sum(L) in integers);
* applying clears the stash.
"""

from __future__ import annotations

from typing import Tuple

import numpy as np


def stash_counts(stash: np.ndarray, counts: np.ndarray) -> np.ndarray:
    """The stash after one forward: stashed loads plus this forward's counts."""
    return np.asarray(stash, dtype=np.int64) + np.asarray(counts, dtype=np.int64)


def bias_update(bias: np.ndarray, loads: np.ndarray, rate: float) -> Tuple[np.ndarray, np.ndarray]:
    """One sign-controller step. Returns (new fp32 bias, cleared stash).

    bias [E] fp32, loads [E] integer counts (already summed over ranks),
    rate: the update rate, taken as an fp32 value."""
    b = np.asarray(bias, dtype=np.float32)
    L = np.asarray(loads, dtype=np.int64)
    E = L.shape[0]
    total = int(L.sum())
    r = float(np.float32(rate))
    out = b.astype(np.float64)
    for e in range(E):
        under = total - E * int(L[e])  # > 0: below the mean load
        if under > 0:
            out[e] = float(b[e]) + r
        elif under < 0:
            out[e] = float(b[e]) - r
    # fp32(b) +- fp32(r) is exact in fp64 for the magnitudes involved; one
    # rounding to fp32 gives the fp32 sum.
    return out.astype(np.float32), np.zeros_like(L)
