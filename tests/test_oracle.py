"""Pins for the CPU oracle: the pages' worked example, hand-derived cases,
closed forms, invariants and brute force on tiny inputs.  None of these runs
on a GPU; they fix the oracle before any CUDA result is compared to it.
"""
import itertools
import os
import random
from fractions import Fraction

import numpy as np
import pytest
import scipy.special
import torch

import oracle
import synth
from oracle import moe as omoe
from oracle import schedule as osch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]


# ---------------------------------------------------------------- Eq. (2), (3)

def test_worked_example_effective_workload():
    lines = dict(ln.split(None, 1) for ln in _read_golden("worked_example_eq2.txt"))
    loads = [int(x) for x in lines["loads"].split()]
    assert osch.effective_workload(loads) == int(lines["effective_workload"])
    # Eq. (3) for that one layer, by hand: (10+9+...+3) / (10 * 8) = 52 / 80
    assert osch.utilization([loads]) == Fraction(52, 80)


def test_utilization_bounds_and_special_cases():
    rng = np.random.default_rng(1)
    for _ in range(200):
        D = int(rng.integers(1, 9))
        layers = [rng.integers(0, 50, size=D) + (rng.integers(0, 2, size=D) if D else 0)
                  for _ in range(int(rng.integers(1, 6)))]
        layers = [w if w.sum() > 0 else w + 1 for w in layers]
        u = osch.utilization(layers)
        assert Fraction(1, D) <= u <= 1
        assert 0 <= 1 - u < 1
    assert osch.utilization([[7]]) == 1                       # D = 1
    assert osch.utilization([[3, 3, 3, 3], [5, 5, 5, 5]]) == 1  # balanced
    assert osch.utilization([[0, 9, 0, 0]]) == Fraction(1, 4)   # one hot device
    with pytest.raises(ValueError):
        osch.utilization([[0, 0]])


def test_combination_is_worst_case_safe():
    """max_d sum_j w_{j,d} <= sum_j max_d w_{j,d}; equality when every peak
    falls on one device, strict when the unique peaks differ."""
    rng = np.random.default_rng(2)
    for _ in range(300):
        D = int(rng.integers(1, 9))
        n = int(rng.integers(1, 6))
        ws = [list(rng.integers(0, 20, size=D)) for _ in range(n)]
        lhs = max(osch.combined(ws))
        rhs = sum(max(w) for w in ws)
        assert lhs <= rhs
        # force a common peak device
        ws2 = [list(w) for w in ws]
        for w in ws2:
            w[0] = max(w) + 1
        assert max(osch.combined(ws2)) == sum(max(w) for w in ws2)
    assert max(osch.combined([[5, 1], [1, 5]])) < 5 + 5


# ------------------------------------------------------------------ schedulers

_POL = {"cumutil": osch.CUMUTIL, "maxutil": osch.MAXUTIL, "diffpeak": osch.DIFFPEAK}


def test_hand_worked_scheduler_cases():
    cases = _read_golden("cumutil_maxutil_hand.txt")
    assert len(cases) >= 10
    for ln in cases:
        head, ws, want = [x.strip() for x in ln.split("|")]
        pol, m = head.split()
        w = {j: [int(x) for x in v.split()] for j, v in enumerate(ws.split(";"))}
        got = osch.schedule(_POL[pol], sorted(w), w, int(m))
        assert got == [int(x) for x in want.split()], ln


def _u_cross(ws):
    W = osch.combined(ws)
    return sum(W), max(W)


def _brute_maxutil(pending, w, m):
    """Independent brute force: enumerate bitmasks, compare U by int64-style
    cross multiplication instead of rationals."""
    best = None
    P = sorted(pending)
    for mask in range(1, 1 << len(P)):
        S = [P[i] for i in range(len(P)) if mask >> i & 1]
        if len(S) < min(m, len(P)):
            continue
        s, mx = _u_cross([w[j] for j in S])
        bm = sum(1 << j for j in S)
        if best is None:
            best = (s, mx, len(S), bm, S)
            continue
        bs, bmx, bl, bbm, _ = best
        better = (s * bmx > bs * mx) or (s * bmx == bs * mx and (len(S) > bl or (len(S) == bl and bm < bbm)))
        if better:
            best = (s, mx, len(S), bm, S)
    return best[4]


def test_maxutil_matches_brute_force_on_all_subsets():
    rng = np.random.default_rng(3)
    for trial in range(300):
        M = int(rng.integers(1, 9))
        D = int(rng.integers(1, 6))
        pending = sorted(rng.choice(M, size=int(rng.integers(1, M + 1)), replace=False).tolist())
        w = {j: [int(x) for x in rng.integers(0, 6, size=D) + (1 if rng.random() < .5 else 0)] for j in pending}
        for j in pending:
            if sum(w[j]) == 0:
                w[j][0] = 1
        m = int(rng.integers(1, M + 1))
        assert osch.maxutil(pending, w, m) == _brute_maxutil(pending, w, m)


def test_tiny_config_maxutil_brute_force_2_pow_4():
    """Tiny fp32 workload (M = 4): at every step of a MaxUtil episode the
    choice is the best of all 2^4 subsets of the pending micro-batches."""
    wl = synth.get("tiny_f32")
    lg = synth.logits(wl)
    _, _, _, ld = oracle.route_all(lg, wl.k, wl.D)
    for m in (1, 2, 3, 4):
        ep = oracle.run_episode(ld, osch.MAXUTIL, m)
        layer = [0] * wl.M
        for st in ep["steps"]:
            pending = [j for j in range(wl.M) if layer[j] < wl.L]
            w = {j: [int(x) for x in ld[j, layer[j]]] for j in pending}
            assert st["runset"] == _brute_maxutil(pending, w, m)
            for j in st["runset"]:
                layer[j] += 1


def test_scheduler_invariants_random():
    rng = np.random.default_rng(4)
    for trial in range(200):
        M = int(rng.integers(1, 9))
        D = int(rng.integers(1, 9))
        w = {j: [int(x) for x in rng.integers(0, 30, size=D)] for j in range(M)}
        for j in w:
            if sum(w[j]) == 0:
                w[j][int(rng.integers(0, D))] = 1
        pending = sorted(rng.choice(M, size=int(rng.integers(1, M + 1)), replace=False).tolist())
        m = int(rng.integers(1, M + 1))
        res = {p: osch.schedule(p, pending, w, m) for p in (0, 1, 2, 3)}
        for p, S in res.items():
            assert S == sorted(set(S)) and set(S) <= set(pending)
            assert len(S) >= min(m, len(pending))
            if len(pending) <= m:
                assert S == pending
        assert res[osch.LOCKSTEP] == pending
        # MaxUtil's choice is a best candidate: no other admissible set beats it
        u_best = osch.set_utilization([w[j] for j in res[osch.MAXUTIL]])
        for p in (0, 2, 3):
            assert osch.set_utilization([w[j] for j in res[p]]) <= u_best
        # CumUtil and DiffPeak always keep the first pending micro-batch
        assert pending[0] in res[osch.CUMUTIL] and pending[0] in res[osch.DIFFPEAK]


# --------------------------------------------------------------- Algorithm 1

@pytest.mark.parametrize("policy", [0, 1, 2, 3])
def test_episode_invariants(policy):
    rng = np.random.default_rng(5 + policy)
    for trial in range(20):
        M, L, D = int(rng.integers(1, 7)), int(rng.integers(1, 6)), int(rng.integers(1, 5))
        ld = rng.integers(0, 9, size=(M, L, D))
        ld[..., 0] += 1
        m = int(rng.integers(1, M + 1))
        ep = oracle.run_episode(ld, policy, m)
        seen = {}
        for st in ep["steps"]:
            for j in st["runset"]:
                l = st["layers"][j]
                assert seen.get(j, -1) == l - 1      # layers in order, once each
                seen[j] = l
        assert all(seen[j] == L - 1 for j in range(M))
        assert L <= len(ep["steps"]) <= M * L
        assert ep["num"] == int(ld.sum())
        assert ep["den"] <= ep["den_sep"]            # worst-case safe
        assert ep["num"] <= ep["den"]
        if policy == osch.LOCKSTEP:
            assert len(ep["steps"]) == L
    # m = M is lock-step for every policy
    ld = rng.integers(1, 9, size=(5, 4, 3))
    lock = oracle.run_episode(ld, osch.LOCKSTEP, 5)
    for p in (0, 1, 3):
        assert oracle.run_episode(ld, p, 5)["steps"] == lock["steps"]


def test_episode_equal_peaks_gives_no_gain():
    """When every (micro-batch, layer) peaks on the same device the combined
    denominator equals the separate one (the equality case)."""
    rng = np.random.default_rng(6)
    ld = rng.integers(0, 9, size=(4, 5, 4))
    ld[..., 2] = ld.max(axis=-1) + 1
    for p in (0, 1, 2, 3):
        ep = oracle.run_episode(ld, p, 2)
        assert ep["den"] == ep["den_sep"]


# --------------------------------------------------------------------- routing

def _brute_topk(row, k):
    chosen = []
    for _ in range(k):
        best = None
        for e, v in enumerate(row):
            if e in chosen:
                continue
            if best is None or v > row[best]:
                best = e
        chosen.append(best)
    return chosen


def test_route_matches_brute_force_topk_with_ties():
    rng = np.random.default_rng(7)
    for _ in range(50):
        T, E = int(rng.integers(1, 9)), int(rng.integers(1, 13))
        k = int(rng.integers(1, E + 1))
        x = rng.integers(-3, 4, size=(T, E)).astype(np.float32)  # many ties
        idx, gate = oracle.route(x, k)
        for t in range(T):
            assert idx[t].tolist() == _brute_topk(x[t].tolist(), k)
            assert abs(gate[t].sum() - 1) < 1e-12
            assert all(gate[t][i] >= gate[t][i + 1] for i in range(k - 1))


def test_route_all_equal_logits_and_full_softmax():
    idx, gate = oracle.route(np.zeros((3, 10), np.float32), 4)
    assert (idx == np.arange(4)).all() and np.allclose(gate, 0.25, atol=0, rtol=1e-15)
    rng = np.random.default_rng(8)
    x = rng.standard_normal((5, 7)).astype(np.float32)
    idx, gate = oracle.route(x, 7)               # k = E: the full softmax
    ref = scipy.special.softmax(x.astype(np.float64), axis=1)
    assert np.allclose(np.take_along_axis(ref, idx.astype(np.int64), 1), gate, rtol=1e-13, atol=0)
    # without renormalisation the gate is the softmax probability itself
    idx2, gate2 = oracle.route(x, 3, renorm=False)
    assert np.allclose(np.take_along_axis(ref, idx2.astype(np.int64), 1), gate2, rtol=1e-13, atol=0)
    with pytest.raises(ValueError):
        oracle.route(np.array([[0, np.nan]], np.float32), 1)


def test_histogram_and_loads():
    rng = np.random.default_rng(9)
    x = rng.standard_normal((50, 12)).astype(np.float32)
    idx, _ = oracle.route(x, 3)
    h = oracle.histogram(idx, 12)
    brute = [0] * 12
    for t in range(50):
        assert len(set(idx[t].tolist())) == 3
        for e in idx[t]:
            brute[int(e)] += 1
    assert h.tolist() == brute and h.sum() == 150
    assert oracle.loads(h, 1).tolist() == [150]
    assert oracle.loads(h, 12).tolist() == brute
    assert oracle.loads(h, 4).tolist() == [sum(brute[3 * d:3 * d + 3]) for d in range(4)]
    with pytest.raises(ValueError):
        oracle.loads(h, 5)


def test_loads_with_expert_map():
    """An arbitrary expert -> rank placement: each rank sums exactly the
    experts mapped to it (brute force per rank), the contiguous map is the
    default, E need not be a multiple of D, and bad maps are rejected."""
    rng = np.random.default_rng(10)
    h = rng.integers(0, 50, size=(3, 12))
    contiguous = [e // 3 for e in range(12)]
    assert np.array_equal(oracle.loads(h, 4, contiguous), oracle.loads(h, 4))
    for D in (1, 3, 5, 7):
        emap = rng.integers(0, D, size=12).tolist()
        w = oracle.loads(h, D, emap)
        for j in range(3):
            for d in range(D):
                assert w[j, d] == sum(int(h[j, e]) for e in range(12) if emap[e] == d)
        assert np.array_equal(w.sum(axis=-1), h.sum(axis=-1))
    # a rank with no experts carries no load; a permutation of the contiguous
    # map permutes the loads
    w = oracle.loads(h, 5, [0] * 6 + [2] * 6)
    assert (w[:, [1, 3, 4]] == 0).all()
    perm = [3, 0, 2, 1]
    w = oracle.loads(h, 4, [perm[e // 3] for e in range(12)])
    assert np.array_equal(w[:, perm], oracle.loads(h, 4))
    for bad in ([0] * 11, [0] * 11 + [4], [-1] + [0] * 11):
        with pytest.raises(ValueError):
            oracle.loads(h, 4, bad)


# ------------------------------------------------------------ expert / combine

def test_round_bf16():
    one = 1.0
    assert omoe.round_bf16(one + 2.0 ** -8) == 1.0                  # tie -> even
    assert omoe.round_bf16(one + 3 * 2.0 ** -8) == one + 2.0 ** -6  # tie -> even
    assert omoe.round_bf16(one + 2.0 ** -8 + 2.0 ** -30) == one + 2.0 ** -7
    assert omoe.round_bf16(-3.0) == -3.0 and omoe.round_bf16(0.0) == 0.0
    rng = np.random.default_rng(10)
    x = (rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000)).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(omoe.round_bf16(x.astype(np.float64)), ref)


def test_silu_closed_forms():
    z = np.linspace(-20, 20, 401)
    s = omoe.silu(z)
    assert omoe.silu(0.0) == 0.0
    assert np.allclose(s - omoe.silu(-z), z, atol=1e-12)          # silu(z) - silu(-z) = z
    assert abs(omoe.silu(40.0) - 40.0) < 1e-12 and abs(omoe.silu(-40.0)) < 1e-12
    assert abs(omoe.silu(1.0) - 1.0 / (1.0 + np.exp(-1.0))) < 1e-15


def test_expert_ffn_brute_force():
    rng = np.random.default_rng(11)
    H, F, n = 5, 3, 4
    x = rng.standard_normal((n, H))
    wg, wu, wd = rng.standard_normal((F, H)), rng.standard_normal((F, H)), rng.standard_normal((H, F))
    y = omoe.expert_ffn(x, wg, wu, wd, "f32")
    for t in range(n):
        a = []
        for f in range(F):
            g = sum(x[t, h] * wg[f, h] for h in range(H))
            u = sum(x[t, h] * wu[f, h] for h in range(H))
            a.append(float(np.float32(g / (1 + np.exp(-g)) * u)))
        for h in range(H):
            want = float(np.float32(sum(a[f] * wd[h, f] for f in range(F))))
            assert abs(y[t, h] - want) <= 1e-6 * max(1.0, abs(want))


def test_identical_experts_reduce_to_one_dense_ffn():
    """All experts of a layer equal and gates summing to one: the MoE layer is
    one dense SwiGLU FFN (checked with torch's float64 matmul)."""
    rng = np.random.default_rng(12)
    E, k, H, F, n = 6, 3, 16, 8, 10
    wg, wu, wd = (rng.standard_normal((F, H)) * .3, rng.standard_normal((F, H)) * .3,
                  rng.standard_normal((H, F)) * .3)
    get = lambda l, e: (wg, wu, wd)
    h = rng.standard_normal((n, H))
    idx, gate = oracle.route(rng.standard_normal((n, E)).astype(np.float32), k)
    out = omoe.moe_layer(h, idx, gate, 0, get, E, 0, "f32")
    th = torch.from_numpy(h)
    a = torch.nn.functional.silu(th @ torch.from_numpy(wg).T) * (th @ torch.from_numpy(wu).T)
    a = a.to(torch.float32).to(torch.float64)
    dense = (a @ torch.from_numpy(wd).T).to(torch.float32).to(torch.float64)
    want = (th + dense).to(torch.float32).to(torch.float64).numpy()
    assert np.allclose(out, want, rtol=0, atol=1e-6)


def test_shared_experts_and_single_slot():
    rng = np.random.default_rng(13)
    E, H, F, n = 4, 8, 4, 5
    W = {e: (rng.standard_normal((F, H)), rng.standard_normal((F, H)), rng.standard_normal((H, F)))
         for e in range(E + 1)}
    get = lambda l, e: W[e]
    h = omoe.round_bf16(rng.standard_normal((n, H)))
    idx = np.array([[2]] * n)
    gate = np.ones((n, 1))
    out = omoe.moe_layer(h, idx, gate, 0, get, E, 1, "bf16")
    want = omoe.round_bf16(h + omoe.expert_ffn(h, *W[2], "bf16") + omoe.expert_ffn(h, *W[E], "bf16"))
    assert np.array_equal(out, want)
    out0 = omoe.moe_layer(h, idx, gate, 0, get, E, 0, "bf16", residual=False)
    assert np.array_equal(out0, omoe.round_bf16(omoe.expert_ffn(h, *W[2], "bf16")))


def test_forward_tokens_single_layer_k1():
    rng = np.random.default_rng(14)
    E, H, F = 3, 6, 4
    W = {e: (rng.standard_normal((F, H)), rng.standard_normal((F, H)), rng.standard_normal((H, F)))
         for e in range(E)}
    lg = rng.standard_normal((1, 1, 4, E)).astype(np.float32)
    h0 = rng.standard_normal((4, H)).astype(np.float32).astype(np.float64)
    out = omoe.forward_tokens(h0, lambda j, l: lg[j, l], [(0, t) for t in range(4)], 1, E, 1, 0,
                              "f32", lambda l, e: W[e])
    for t in range(4):
        e = int(np.argmax(lg[0, 0, t]))
        want = (h0[t] + omoe.expert_ffn(h0[t:t + 1], *W[e], "f32")[0]).astype(np.float32)
        assert np.array_equal(out[t], want.astype(np.float64))


def test_moe_layer_slot_gates_brute_force():
    """Eq. (1) token by token: out = h + sum_s gate_s * expert_{idx_s}(h)."""
    rng = np.random.default_rng(15)
    E, k, H, F, n = 5, 2, 6, 3, 7
    W = {e: (rng.standard_normal((F, H)), rng.standard_normal((F, H)), rng.standard_normal((H, F)))
         for e in range(E)}
    h = rng.standard_normal((n, H)).astype(np.float32).astype(np.float64)
    idx, gate = oracle.route(rng.standard_normal((n, E)).astype(np.float32), k)
    out = omoe.moe_layer(h, idx, gate, 0, lambda l, e: W[e], E, 0, "f32")
    for t in range(n):
        acc = h[t].copy()
        for s in range(k):
            e = int(idx[t, s])
            acc = acc + gate[t, s] * omoe.expert_ffn(h[t:t + 1], *W[e], "f32")[0]
        assert np.array_equal(out[t], acc.astype(np.float32).astype(np.float64))
    # gates differ between slots, so swapping them changes the result
    out_sw = omoe.moe_layer(h, idx, gate[:, ::-1], 0, lambda l, e: W[e], E, 0, "f32")
    assert not np.array_equal(out, out_sw)


def test_zero_work_sets_rank_lowest():
    """Reading for loads with no work: U = 0, so such a set never beats one
    that carries work, and adding it never raises U (CumUtil skips it)."""
    w = {0: [0, 0], 1: [3, 1], 2: [0, 0]}
    assert osch.set_utilization([w[0]]) == 0
    assert osch.cumutil([0, 1, 2], w, 1) == [0, 1]
    # every set holding micro-batch 1 has U = 4/6; the largest one wins
    assert osch.maxutil([0, 1, 2], w, 1) == [0, 1, 2]


def test_native_maxutil_matches_python():
    """The plain-C exhaustive MaxUtil agrees with the Python one."""
    from oracle import native
    rng = np.random.default_rng(16)
    for trial in range(300):
        M = int(rng.integers(1, 11))
        D = int(rng.integers(1, 9))
        pending = sorted(rng.choice(M, size=int(rng.integers(1, M + 1)), replace=False).tolist())
        hi = int(rng.choice([2, 5, 50]))
        w = {j: [int(x) for x in rng.integers(0, hi, size=D)] for j in pending}
        m = int(rng.integers(1, M + 1))
        assert native.maxutil(pending, w, m) == osch.maxutil(pending, w, m), (pending, w, m)
    # golden hand cases
    for ln in _read_golden("cumutil_maxutil_hand.txt"):
        head, ws, want = [x.strip() for x in ln.split("|")]
        pol, m = head.split()
        if pol != "maxutil":
            continue
        w = {j: [int(x) for x in v.split()] for j, v in enumerate(ws.split(";"))}
        assert native.maxutil(sorted(w), w, int(m)) == [int(x) for x in want.split()]


def test_native_maxutil_plain_pins_the_complement_enumeration():
    """The forward enumeration over every bitmask (oracle_maxutil_plain) is
    pinned against the Python enumeration of [EB] §4.2's candidate subsets up
    to 16 pending micro-batches; the complement enumeration (used for pending
    sets of 32) is pinned against the forward one up to 20, with many equal-U
    ties (small loads) and pending sets with holes."""
    from oracle import native
    rng = np.random.default_rng(1620)
    for trial in range(200):
        M = int(rng.integers(1, 13))
        D = int(rng.integers(1, 9))
        pending = sorted(rng.choice(M, size=int(rng.integers(1, M + 1)), replace=False).tolist())
        hi = int(rng.choice([2, 4, 60]))
        w = {j: [int(x) for x in rng.integers(0, hi, size=D)] for j in pending}
        m = int(rng.integers(1, M + 1))
        assert native.maxutil_plain(pending, w, m) == osch.maxutil(pending, w, m), (pending, w, m)
    for trial in range(2):  # 16 pending micro-batches: 65 536 subsets in Python
        pending = list(range(16))
        w = {j: [int(x) for x in rng.integers(0, 6, size=4)] for j in pending}
        assert native.maxutil_plain(pending, w, 12) == osch.maxutil(pending, w, 12)
    for trial in range(120):
        M = int(rng.integers(12, 21))
        D = int(rng.choice([1, 3, 8, 16, 64]))
        pending = sorted(rng.choice(32, size=M, replace=False).tolist())
        hi = int(rng.choice([2, 3, 1000]))
        w = {j: [int(x) for x in rng.integers(0, hi, size=D)] for j in pending}
        m = int(rng.integers(max(1, M - 6), M + 1)) if trial % 3 else int(rng.integers(1, M + 1))
        a, b = native.maxutil(pending, w, m), native.maxutil_plain(pending, w, m)
        assert a == b, (pending, m, a, b)


# ------------------------------------------------------------ router projection

def test_router_projection_pins():
    """The router projection: written-out loops on a small case, one-hot
    router rows pick hidden columns exactly, a zero router gives equal scores
    (so the top-k falls back to experts 0..k-1 with equal gates), and the
    routed chain with identical experts equals the dense SwiGLU chain."""
    from oracle import router as orouter
    rng = np.random.default_rng(40)
    h = omoe.round_bf16(rng.standard_normal((5, 24)))
    w = omoe.round_bf16(rng.standard_normal((6, 24)) * 0.3)
    assert np.allclose(orouter.router_logits(h, w), orouter.router_logits_loops(h, w),
                       rtol=0, atol=1e-12)
    cols = [3, 0, 23, 7, 7, 11]
    onehot = np.zeros((6, 24))
    onehot[np.arange(6), cols] = 1.0
    assert np.array_equal(orouter.router_logits(h, onehot), h[:, cols])
    zero = orouter.router_logits(h, np.zeros((6, 24)))
    idx, gate = oracle.route(zero.astype(np.float32), 3)
    assert (idx == [0, 1, 2]).all() and np.allclose(gate, 1.0 / 3)
    # identical experts: the MoE layer is one dense SwiGLU FFN whatever the
    # router picks (gates sum to 1), so the routed chain is the dense chain
    H, F, E, k, L = 24, 16, 6, 2, 3
    wg = [omoe.round_bf16(rng.standard_normal((F, H)) * 0.2) for _ in range(L)]
    wu = [omoe.round_bf16(rng.standard_normal((F, H)) * 0.2) for _ in range(L)]
    wd = [omoe.round_bf16(rng.standard_normal((H, F)) * 0.2) for _ in range(L)]
    routers = [omoe.round_bf16(rng.standard_normal((E, H))) for _ in range(L)]
    get = lambda l, e: (wg[l], wu[l], wd[l])
    out, seen = orouter.forward_tokens_routed(h, lambda l: routers[l], [(0, t) for t in range(5)],
                                              L, E, k, 0, "f32", get)
    import torch
    x = torch.tensor(h, dtype=torch.float64)
    for l in range(L):
        g = x @ torch.tensor(wg[l]).T
        u = x @ torch.tensor(wu[l]).T
        y = (g * torch.sigmoid(g) * u) @ torch.tensor(wd[l]).T
        x = x + y
    assert np.allclose(out, x.numpy(), rtol=1e-5, atol=1e-5)
    assert len(seen) == L and seen[0].dtype == np.float32
    # the first layer's scores are the projection of h_0 itself
    assert np.array_equal(seen[0], orouter.router_logits(h, routers[0]).astype(np.float32))
