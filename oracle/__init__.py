"""fp64 CPU oracle of the sparse top-k MoE FFN forward.

TEST INFRASTRUCTURE ONLY: only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import it. The CUDA library
(``sparse_top_mixture_b200``) shares no code with it and never imports it.
"""

from .moe import (  # noqa: F401
    BIAS_LOGIT, BIAS_NONE, BIAS_SELECT, SHARED_GATED, SHARED_NONE, SHARED_PLAIN, SIGMOID, SOFTMAX, SQRTSOFTPLUS,
    decision_margins, dispatch, moe_forward, route, router_logits, routing_matrix, scores, select_topk,
    selection_keys, shared_gate_values, sigmoid, silu, softmax_rows, softplus, swiglu_mlp, topk_weights,
)
from .brute import brute_dispatch, brute_forward  # noqa: F401
