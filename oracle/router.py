"""Oracle: the router projection and the routed layer-by-layer chain.

Test infrastructure only (parity checks); nothing in the library's product
path calls it.

[EB] is the paper "EasyBalance: Cross-Layer Load Balancing in Distributed MoE
Inference".  §2.1 there: a gating network scores the experts from the token's
hidden state, W_l, I_l = topk(G(h'_l)).  With a linear router the scores are
the projection h'_l W_r^T of the hidden state onto one row per expert, and
G is the softmax over them.  The projection is computed here in float64
from the stored values and handed to routing as float32, the precision in
which the library's routing takes its top-k decision.
"""
from __future__ import annotations

from typing import Callable, Sequence, Tuple

import numpy as np

from .moe import ExpertGetter, moe_layer
from .routing import route


def router_logits(h, w_router) -> np.ndarray:
    """Scores of every expert for every token: h [n, H] times w_router [E, H]
    transposed, in float64 -> [n, E]."""
    return np.asarray(h, dtype=np.float64) @ np.asarray(w_router, dtype=np.float64).T


def router_logits_loops(h, w_router) -> np.ndarray:
    """The same projection written out as plain loops (small cases)."""
    h = np.asarray(h, dtype=np.float64)
    w = np.asarray(w_router, dtype=np.float64)
    n, H = h.shape
    E = w.shape[0]
    out = np.zeros((n, E), dtype=np.float64)
    for t in range(n):
        for e in range(E):
            acc = 0.0
            for i in range(H):
                acc += h[t, i] * w[e, i]
            out[t, e] = acc
    return out


def forward_tokens_routed(h0, router_getter: Callable[[int], np.ndarray],
                          tokens: Sequence[Tuple[int, int]], L: int, E: int, k: int,
                          n_shared: int, dtype: str, get_expert: ExpertGetter,
                          renorm: bool = True, residual: bool = True,
                          layers: Sequence[int] = None):
    """Trajectory of the given tokens when each layer's router logits come
    from the token's current hidden state ([EB] §2.1, attention taken as the
    identity).  router_getter(l) returns the [E, H] router of layer l.
    Returns (final hidden [n, H], per-layer float32 logits [n, E] list)."""
    h = np.asarray(h0, dtype=np.float64).copy()
    seen = []
    for l in (range(L) if layers is None else layers):
        lg = router_logits(h, router_getter(l)).astype(np.float32)
        seen.append(lg)
        idx, gate = route(lg, k, renorm)
        h = moe_layer(h, idx, gate, l, get_expert, E, n_shared, dtype, residual)
    return h, seen
