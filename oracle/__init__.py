"""CPU oracle for the EasyBalance cross-layer MoE step.

TEST INFRASTRUCTURE ONLY.  This package is a plain, slow, float64 / exact-
integer restatement of what the cross-layer MoE step computes, written from
the paper "EasyBalance: Cross-Layer Load Balancing in Distributed MoE
Inference" (Wu, Gao, Li, Wu) and the pages that restate it.  Only the tests,
``__graft_entry__.smoke()`` and two parts of ``bench.py`` may import it: the
CPU-baseline leg and the reference arm (``--impl reference``, the sweep's
included).  It shares no code with the CUDA library
(``cross_layer_expert_b200``) and imports nothing from it; both take their
inputs from ``synth``.

Modules:
  routing   top-k gating, per-expert histograms T_e, virtual-rank loads w
  schedule  Eq. (2) effective workload, Eq. (3) utilisation, U(S), CumUtil,
            MaxUtil, DiffPeak, lock-step, Algorithm 1 episodes
  moe       SwiGLU experts, the gated combine (Eq. (1)), token trajectories
"""
from __future__ import annotations

import numpy as np

from . import moe, routing, schedule  # noqa: F401
from .routing import histogram, loads, route  # noqa: F401
from .schedule import (CUMUTIL, DIFFPEAK, LOCKSTEP, MAXUTIL, run_episode,  # noqa: F401
                       set_utilization, utilization)


def route_all(logits: np.ndarray, k: int, D: int, renorm: bool = True, expert_rank=None):
    """Route every (micro-batch, layer) block of logits [M, L, T, E].

    Returns idx [M, L, T, k] int32, gate [M, L, T, k] float64, hist [M, L, E]
    and loads [M, L, D] (int64) under the contiguous map, or under
    expert_rank if given.
    """
    M, L, T, E = logits.shape
    idx = np.empty((M, L, T, k), dtype=np.int32)
    gate = np.empty((M, L, T, k), dtype=np.float64)
    hist = np.empty((M, L, E), dtype=np.int64)
    for j in range(M):
        for l in range(L):
            idx[j, l], gate[j, l] = route(logits[j, l], k, renorm)
            hist[j, l] = histogram(idx[j, l], E)
    return idx, gate, hist, loads(hist, D, expert_rank)
