"""Oracle: effective workload, utilisation and the RunSet schedulers.

Test infrastructure only (parity checks, the smoke check, and the CPU
baseline and reference arm of the benchmark); nothing in the library's
product path calls it.

[EB] is the paper "EasyBalance: Cross-Layer Load Balancing in Distributed MoE
Inference"; [EB-read] the deep-read page "EasyBalance：分布式 MoE 推理的跨层负载均衡".

Utilisation values are exact rationals (``fractions.Fraction``); workloads are
Python integers.
"""
from __future__ import annotations

import itertools
from fractions import Fraction
from typing import Iterable, List, Sequence

import numpy as np

CUMUTIL, MAXUTIL, LOCKSTEP, DIFFPEAK = 0, 1, 2, 3
POLICY_NAMES = {CUMUTIL: "cumutil", MAXUTIL: "maxutil", LOCKSTEP: "lockstep",
                DIFFPEAK: "diffpeak"}


def effective_workload(w: Sequence[int]) -> int:
    """w_hat = max_d w_d.  [EB] §2.3 Eq. (2): the slowest device bounds the layer."""
    return max(int(x) for x in w)


def utilization(per_layer_loads: Iterable[Sequence[int]]) -> Fraction:
    """u = sum_l sum_d w_d^(l) / (sum_l w_hat^(l) * D).  [EB] §2.3 Eq. (3)."""
    num = 0
    den = 0
    D = None
    for w in per_layer_loads:
        w = [int(x) for x in w]
        D = len(w) if D is None else D
        if len(w) != D:
            raise ValueError("all workload vectors need the same D")
        num += sum(w)
        den += effective_workload(w) * D
    if den == 0:
        raise ValueError("utilisation of an empty or all-zero workload is undefined")
    return Fraction(num, den)


def combined(ws: Sequence[Sequence[int]]) -> List[int]:
    """Load of a set of workloads run in one step: W_d = sum_j w_{j,d}.

    [EB] §1 (Cross-Layer Workload Combination): the combined workload of w1, w2
    is w1 + w2.
    """
    D = len(ws[0])
    return [sum(int(w[d]) for w in ws) for d in range(D)]


def set_utilization(ws: Sequence[Sequence[int]]) -> Fraction:
    """U(S): the device utilisation of the combined workload of set S.

    [EB] §5.2 (CumUtil: "U(.) denotes GPU utilization"); read as Eq. (3)
    applied to the one step that runs S: sum_d W_d / (D * max_d W_d).
    A set that carries no work at all leaves every device idle and is given
    U = 0 (a reading: Eq. (3) is 0/0 there; in an episode every micro-batch
    carries T k > 0 token-expert pairs, so this only concerns stand-alone
    calls on arbitrary loads).
    """
    W = combined(ws)
    if max(W) == 0:
        return Fraction(0)
    return utilization([W])


def _pad_to_m(chosen: List[int], pending: Sequence[int], m: int) -> List[int]:
    """Meet |RunSet| >= m by adding skipped candidates in ascending index.

    [EB] §4.2 requires |RunSet| >= m but does not say how the O(n) heuristics
    meet it; this ascending-index padding is the reading taken here.
    """
    out = list(chosen)
    for j in pending:
        if len(out) >= m:
            break
        if j not in out:
            out.append(j)
    return sorted(out)


def cumutil(pending: Sequence[int], w: dict, m: int) -> List[int]:
    """CumUtil.  [EB] §5.2: scan micro-batches in order 0..N-1, the first is
    always scheduled, and batch j+1 joins iff U(S ∪ {w_{j+1}}) > U(S)
    (strictly).  [EB-read] §2.4 restates the same rule.
    """
    pending = sorted(pending)
    if len(pending) <= m:
        return list(pending)
    S = [pending[0]]
    for j in pending[1:]:
        if set_utilization([w[i] for i in S + [j]]) > set_utilization([w[i] for i in S]):
            S.append(j)
    return _pad_to_m(S, pending, m)


def maxutil(pending: Sequence[int], w: dict, m: int) -> List[int]:
    """MaxUtil.  [EB] §4.2 / §5.2: among the candidate subsets pick the one
    whose combined workload has the highest utilisation; O(2^n).

    Candidates are all subsets S of the pending set with |S| >= m ([EB] §4.2).
    The pages give no tie-break; the reading taken: higher U, then larger
    |S| (more work advances), then the smaller bitmask sum_j 2^j.
    """
    pending = sorted(pending)
    if len(pending) <= m:
        return list(pending)
    best = None
    best_key = None
    for size in range(m, len(pending) + 1):
        for S in itertools.combinations(pending, size):
            U = set_utilization([w[i] for i in S])
            mask = sum(1 << i for i in S)
            key = (U, len(S), -mask)
            if best_key is None or key > best_key:
                best_key = key
                best = list(S)
    return best


def peak_device(w: Sequence[int]) -> int:
    """argmax_d w_d with ties to the lower device index (a reading)."""
    w = [int(x) for x in w]
    return w.index(max(w))


def diffpeak(pending: Sequence[int], w: dict, m: int) -> List[int]:
    """DiffPeak.  [EB] §5.2: batch j+1 joins iff its peak device
    argmax_d w_{j+1} is not among the peak devices of the batches already
    chosen; the first is always chosen.  Padded to m like CumUtil.
    """
    pending = sorted(pending)
    if len(pending) <= m:
        return list(pending)
    S = [pending[0]]
    peaks = {peak_device(w[pending[0]])}
    for j in pending[1:]:
        p = peak_device(w[j])
        if p not in peaks:
            S.append(j)
            peaks.add(p)
    return _pad_to_m(S, pending, m)


def lockstep(pending: Sequence[int], w: dict, m: int) -> List[int]:
    """Every pending micro-batch runs: strict layer-by-layer execution."""
    return sorted(pending)


SCHEDULERS = {CUMUTIL: cumutil, MAXUTIL: maxutil, LOCKSTEP: lockstep, DIFFPEAK: diffpeak}


def schedule(policy: int, pending: Sequence[int], w: dict, m: int) -> List[int]:
    """RunSet_i = Schedule(S_{i-1}, m).  [EB] §4.2 Algorithm 1."""
    if m < 1:
        raise ValueError("m must be >= 1")
    return SCHEDULERS[policy](pending, w, m)


def run_episode(loads_all: np.ndarray, policy: int, m: int, maxutil_impl=None):
    """Algorithm 1 of [EB] §4.2 over pre-routed workloads.

    loads_all[j, l] is the D-vector w of micro-batch j at MoE layer l (the
    routed tokens of a (micro-batch, layer) do not depend on when it runs).

    Start: l_j = 0 and S_0 = all micro-batches.  Each step picks
    RunSet_i = Schedule(S_{i-1}, m), runs it, advances l_j for j in the RunSet
    and drops the micro-batches that reached l_max.  Stops when S is empty.

    maxutil_impl optionally replaces the Python MaxUtil enumeration by another
    implementation of the same definition (oracle.native.maxutil, plain C).

    Returns a dict with the per-step list of (runset, layers, sumW, maxW,
    summax) and the episode totals num = sum sumW, den = D sum maxW (the
    scheduled run's Eq. (3) denominator) and den_sep = D sum_{j,l} max_d w_{j,l}
    (every micro-batch executed on its own: the "maximum workload" of the
    paper's Fig. 6).
    """
    loads_all = np.asarray(loads_all, dtype=np.int64)
    M, L, D = loads_all.shape
    layer = [0] * M
    S = set(range(M))
    steps = []
    while S:
        pending = sorted(S)
        w = {j: [int(x) for x in loads_all[j, layer[j]]] for j in pending}
        if policy == MAXUTIL and maxutil_impl is not None:
            run = maxutil_impl(pending, w, m)
        else:
            run = schedule(policy, pending, w, m)
        if not run:
            raise RuntimeError("empty RunSet")
        W = combined([w[j] for j in run])
        steps.append(dict(runset=list(run), layers={j: layer[j] for j in run},
                          sumW=sum(W), maxW=max(W),
                          summax=sum(effective_workload(w[j]) for j in run)))
        for j in run:
            layer[j] += 1
        S = {j for j in range(M) if layer[j] < L}
    num = sum(s["sumW"] for s in steps)
    den = D * sum(s["maxW"] for s in steps)
    den_sep = D * int(sum(effective_workload(loads_all[j, l])
                          for j in range(M) for l in range(L)))
    return dict(steps=steps, num=num, den=den, den_sep=den_sep)
