"""Oracle: router top-k, per-expert histograms and virtual-rank loads.

Test infrastructure only (parity checks, the smoke check, and the CPU
baseline and reference arm of the benchmark); nothing in the library's
product path calls it.

Citations name the paper "EasyBalance: Cross-Layer Load Balancing in
Distributed MoE Inference" (Wu, Gao, Li, Wu) as [EB], the deep-read page
"EasyBalance：分布式 MoE 推理的跨层负载均衡" as [EB-read], and the page
"系统侧负载均衡：EPLB、LPLB、UltraEP 与 MoonEP" as [SysLB].
"""
from __future__ import annotations

import numpy as np


def route(logits: np.ndarray, k: int, renorm: bool = True):
    """Top-k gating  W_l, I_l = topk(G(h'_l))  for one block of tokens.

    [EB] §2.1 (the router selects the top-k experts by the gating function G,
    Eq. (1) then weighs each selected expert).  The pages leave G open; it is
    read here as the softmax over the E router logits, the selected weights
    renormalised to sum to one.

    Readings where the pages are silent:
      * the k experts are the k largest *logits* (softmax is monotone, so this
        is the same set as the k largest probabilities, without ties created
        by rounding exp); equal logits go to the lower expert index;
      * slots are ordered by descending logit (then ascending index).

    logits: [T, E] float32.  Returns idx [T, k] int32 and gate [T, k] float64.
    """
    x = np.asarray(logits, dtype=np.float32)
    if x.ndim != 2:
        raise ValueError("logits must be [T, E]")
    T, E = x.shape
    if not (1 <= k <= E):
        raise ValueError("need 1 <= k <= E")
    if not np.all(np.isfinite(x)):
        raise ValueError("non-finite router logit")
    # a stable sort of the negated logits keeps the lower index first on ties
    order = np.argsort(-x, axis=1, kind="stable")
    idx = order[:, :k]
    xd = x.astype(np.float64)
    mx = xd.max(axis=1, keepdims=True)
    p = np.exp(xd - mx)
    p = p / p.sum(axis=1, keepdims=True)          # softmax over all E experts
    gate = np.take_along_axis(p, idx, axis=1)
    if renorm:
        gate = gate / gate.sum(axis=1, keepdims=True)
    return idx.astype(np.int32), gate


def histogram(idx: np.ndarray, E: int) -> np.ndarray:
    """Per-expert token counts T_e of one (micro-batch, layer).

    [SysLB] §1: T_e is the number of this batch's tokens routed to expert e;
    every (token, slot) pair counts once.  Returns int64 [E].
    """
    return np.bincount(np.asarray(idx).reshape(-1), minlength=E).astype(np.int64)


def loads(hist: np.ndarray, D: int, expert_rank=None) -> np.ndarray:
    """Virtual-rank workload vector w = (w_1..w_D) of one (micro-batch, layer).

    [SysLB] §1: the load of rank r is the sum of T_e over its local experts.
    [EB] §5 Models: experts are evenly distributed over the devices; read as the
    contiguous map, rank d holding experts [d E/D, (d+1) E/D).
    [EB] §2.3 writes this vector as w^(l) = (w_1^(l), ..., w_D^(l)).
    expert_rank (length E, values in [0, D)) replaces the contiguous map by
    an arbitrary placement, as a load balancer such as EPLB would choose
    ([EB] §5.3 treats placement as orthogonal to scheduling); E need not then
    be a multiple of D.
    """
    hist = np.asarray(hist, dtype=np.int64)
    E = hist.shape[-1]
    if D < 1:
        raise ValueError("D must be positive")
    if expert_rank is None:
        if E % D != 0:
            raise ValueError("E must be a multiple of D")
        expert_rank = [e // (E // D) for e in range(E)]
    expert_rank = list(expert_rank)
    if len(expert_rank) != E or any(not (0 <= r < D) for r in expert_rank):
        raise ValueError("expert_rank must give a rank in [0, D) for each of the E experts")
    w = np.zeros(hist.shape[:-1] + (D,), dtype=np.int64)
    for e, r in enumerate(expert_rank):
        w[..., r] += hist[..., e]
    return w
