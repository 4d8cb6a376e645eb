"""GPU parity tests: every stage of the cross-layer MoE step, called through
the C ABI, against the CPU oracle on the same seeded inputs.

Integers (indices, histograms, loads, RunSets, traces, utilisation numerators
and denominators) must match bit for bit; outputs within max-abs 2e-2 /
relative 1e-2 in bf16 and 1e-5 in fp32.
"""
import os

import numpy as np
import pytest

import oracle
import synth
from oracle import schedule as osch

from _common import (Inputs, assert_close, check_schedule, oracle_episode, oracle_hidden,
                     run_episode)

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def torch():
    import torch as t
    from cross_layer_expert_b200 import build
    build.build()
    return t


# ------------------------------------------------------------------ routing

@pytest.mark.parametrize("E,k,n,ties", [(16, 2, 200, False), (12, 3, 77, True), (64, 6, 513, False),
                                        (128, 8, 1000, False), (128, 8, 300, True),
                                        (256, 8, 129, False), (33, 32, 64, True), (5, 1, 1, False)])
def test_route_matches_oracle(torch, E, k, n, ties):
    import cross_layer_expert_b200 as eb
    rng = np.random.default_rng(E * 1000 + k)
    x = (rng.integers(-3, 4, size=(n, E)) if ties else rng.standard_normal((n, E))).astype(np.float32)
    lg = torch.from_numpy(x).cuda()
    for renorm in (True, False):
        idx = torch.empty((n, k), dtype=torch.int32, device="cuda")
        gate = torch.empty((n, k), dtype=torch.float32, device="cuda")
        hist = torch.empty((E,), dtype=torch.int32, device="cuda")
        eb.eb_route(lg, k, renorm, idx, gate, hist)
        torch.cuda.synchronize()
        ridx, rgate = oracle.route(x, k, renorm)
        assert np.array_equal(idx.cpu().numpy(), ridx)
        assert np.array_equal(hist.cpu().numpy(), oracle.histogram(ridx, E))
        g = gate.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(g - rgate) <= 1e-6 * np.abs(rgate) + 1e-12)


def test_route_nonfinite_sets_status(torch):
    import cross_layer_expert_b200 as eb
    x = torch.randn(70, 16, device="cuda")
    x[65, 3] = float("nan")
    idx = torch.empty((70, 2), dtype=torch.int32, device="cuda")
    gate = torch.empty((70, 2), dtype=torch.float32, device="cuda")
    hist = torch.empty((16,), dtype=torch.int32, device="cuda")
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    eb.eb_route(x, 2, True, idx, gate, hist, status)
    assert int(status.item()) == eb.EB_ERR_NONFINITE
    assert int(hist.sum().item()) == 140
    x[65, 3] = 0.0
    status.zero_()
    eb.eb_route(x, 2, True, idx, gate, hist, status)
    assert int(status.item()) == eb.EB_OK


def test_loads_match_oracle(torch):
    import cross_layer_expert_b200 as eb
    rng = np.random.default_rng(5)
    for (M, E, D) in [(8, 128, 8), (32, 128, 64), (3, 12, 3), (1, 16, 1), (5, 16, 16)]:
        h = rng.integers(0, 1000, size=(M, E)).astype(np.int32)
        w = torch.empty((M, D), dtype=torch.int32, device="cuda")
        eb.eb_loads(torch.from_numpy(h).cuda(), D, w)
        assert np.array_equal(w.cpu().numpy(), oracle.loads(h, D))


# ------------------------------------------------------------------ scheduler

def _gpu_schedule(torch, w, pending, m, policy):
    import cross_layer_expert_b200 as eb
    wt = torch.from_numpy(np.asarray(w, dtype=np.int32)).cuda()
    rs = torch.zeros((1,), dtype=torch.int32, device="cuda")
    stats = torch.zeros((3,), dtype=torch.int64, device="cuda")
    eb.eb_schedule(wt, pending, m, policy, rs, stats)
    return int(rs.item()) & 0xFFFFFFFF, stats.cpu().numpy().tolist()


def test_schedule_hand_cases(torch):
    pol = {"cumutil": 0, "maxutil": 1, "diffpeak": 3}
    for ln in open(os.path.join(GOLDEN, "cumutil_maxutil_hand.txt")):
        ln = ln.strip()
        if not ln or ln.startswith("#"):
            continue
        head, ws, want = [x.strip() for x in ln.split("|")]
        p, m = head.split()
        w = [[int(x) for x in v.split()] for v in ws.split(";")]
        mask, _ = _gpu_schedule(torch, w, (1 << len(w)) - 1, int(m), pol[p])
        assert mask == sum(1 << int(x) for x in want.split()), ln


@pytest.mark.parametrize("policy", [0, 1, 2, 3])
def test_schedule_random_matches_oracle(torch, policy):
    rng = np.random.default_rng(100 + policy)
    for trial in range(150):
        M = int(rng.choice([1, 2, 3, 4, 5, 8, 12, 16]))
        D = int(rng.choice([1, 2, 4, 8, 16, 64]))
        hi = int(rng.choice([3, 10, 1000]))
        w = rng.integers(0, hi, size=(M, D))
        w[:, 0] += rng.integers(0, 2, size=M)
        pend = [j for j in range(M) if rng.random() < 0.8] or [0]
        m = int(rng.integers(1, M + 1))
        mask, stats = _gpu_schedule(torch, w, sum(1 << j for j in pend), m, policy)
        wd = {j: [int(x) for x in w[j]] for j in pend}
        ref = osch.schedule(policy, pend, wd, m)
        assert mask == sum(1 << j for j in ref), (trial, M, D, m, pend)
        W = osch.combined([wd[j] for j in ref])
        assert stats == [sum(W), max(W), sum(max(wd[j]) for j in ref)]


@pytest.mark.parametrize("D,m,holes", [(8, 15, False), (16, 10, True), (64, 18, False)])
def test_maxutil_m20_forward_enumeration(torch, D, m, holes):
    """MaxUtil with 20 pending micro-batches against the oracle's forward
    enumeration of every subset (2^20 bitmasks, W summed from the member
    rows), which shares no structure with the kernel's search."""
    from oracle import native
    rng = np.random.default_rng(2000 + D + m)
    for trial in range(3):
        w = rng.integers(0, 3 if trial == 0 else 300, size=(32, D))
        pend = [j for j in range(32) if (j % 3 != 1 if holes else j < 20)][:20]
        mask, stats = _gpu_schedule(torch, w, sum(1 << j for j in pend), m, osch.MAXUTIL)
        wd = {j: [int(x) for x in w[j]] for j in pend}
        ref = native.maxutil_plain(pend, wd, m)
        assert mask == sum(1 << j for j in ref), (trial, D, m)
        W = osch.combined([wd[j] for j in ref])
        assert stats == [sum(W), max(W), sum(max(wd[j]) for j in ref)]


def test_maxutil_m32_sampled(torch):
    """MaxUtil at M = 32, m = 24 (about 15M admissible subsets per call)
    against the oracle's exhaustive enumeration (plain C, by complements;
    pinned against the forward enumeration up to 20 micro-batches)."""
    from oracle import native
    rng = np.random.default_rng(7)
    for trial, D in enumerate((8, 16)):
        w = rng.integers(0, 200, size=(32, D))
        mask, _ = _gpu_schedule(torch, w, 0xFFFFFFFF, 24, osch.MAXUTIL)
        pend = list(range(32))
        ref = native.maxutil(pend, {j: [int(x) for x in w[j]] for j in pend}, 24)
        assert mask == sum(1 << j for j in ref)
    # a pending set with holes: 28 of 32
    pend = [j for j in range(32) if j % 8 != 3]
    w = rng.integers(0, 50, size=(32, 8))
    mask, _ = _gpu_schedule(torch, w, sum(1 << j for j in pend), 22, osch.MAXUTIL)
    ref = native.maxutil(pend, {j: [int(x) for x in w[j]] for j in pend}, 22)
    assert mask == sum(1 << j for j in ref)


# ------------------------------------------------------------------ episodes

SMALL = ["tiny_f32", "small_bf16", "small_shared_bf16"]


@pytest.fixture(scope="module")
def small_inputs(torch):
    return {name: Inputs(synth.get(name)) for name in SMALL}


@pytest.fixture(scope="module")
def small_expected(small_inputs):
    out = {}
    for name, inp in small_inputs.items():
        wl = inp.wl
        toks = [(j, t) for j in range(wl.M) for t in range(wl.T)]
        out[name] = oracle_hidden(inp, toks).reshape(wl.M, wl.T, wl.H)
    return out


@pytest.mark.parametrize("name", SMALL)
@pytest.mark.parametrize("policy", [0, 1, 2, 3])
@pytest.mark.parametrize("gemm", [0, 1, 2, 6, 7])
def test_small_episode_matches_oracle(small_inputs, small_expected, name, policy, gemm):
    """gemm 0: default engine (token-major tensor-core engine for bf16, SIMT
    for fp32); 1: weight-major; 2: SIMT; 6: token-major with GEMM 1 gathering
    its rows from the hidden states; 7: token-major with the combine fused
    into GEMM 2 (the tensor-core engines take bf16 only)."""
    inp = small_inputs[name]
    wl = inp.wl
    if wl.dtype == "f32" and gemm in (1, 6, 7):
        pytest.skip("the tensor-core engines take bf16 operands")
    hidden, rows, layers, util, steps = run_episode(inp, policy, gemm=gemm)
    check_schedule(rows, layers, util, steps, oracle_episode(inp, policy), wl.M)
    assert_close(hidden.float().cpu().numpy(), small_expected[name], wl.dtype, f"{name} p{policy}")


@pytest.mark.parametrize("name", ["small_bf16", "small_shared_bf16"])
def test_scheduled_equals_lockstep_bitwise(small_inputs, name):
    """Scheduling moves only timing: every policy's final hidden states equal
    the lock-step run's bit for bit (fixed K order, fixed combine order)."""
    inp = small_inputs[name]
    import torch
    lock = run_episode(inp, osch.LOCKSTEP)[0].cpu()
    for policy in (0, 1, 3):
        h = run_episode(inp, policy)[0].cpu()
        assert torch.equal(h.view(torch.int16), lock.view(torch.int16)), policy


@pytest.mark.parametrize("name", ["small_bf16", "small_shared_bf16"])
@pytest.mark.parametrize("policy", [0, 1])
def test_fused_combine_bitwise_equals_unfused(small_inputs, name, policy):
    """The combine fused into GEMM 2 (engine 7) does the stand-alone combine's
    arithmetic in the same slot order, so whole episodes agree bit for bit
    with the token-major engine (4).  Two episodes on one context agree too:
    the arrival counters are back at zero after every step."""
    import torch
    import cross_layer_expert_b200 as eb
    from _common import lib_config
    inp = small_inputs[name]
    ref = run_episode(inp, policy, gemm=4)[0].cpu()
    ctx = eb.Context(lib_config(inp.wl, policy, gemm=7))
    try:
        for rep in range(2):
            hidden = inp.h0.clone()
            ctx.eb_episode(inp.logits, hidden, inp.w_gateup, inp.w_down)
            assert ctx.eb_sync_status() == eb.EB_OK
            assert torch.equal(hidden.cpu().view(torch.int16), ref.view(torch.int16)), rep
    finally:
        ctx.close()


@pytest.mark.parametrize("name", ["small_bf16", "small_shared_bf16"])
@pytest.mark.parametrize("policy", [0, 1])
def test_row_placement_in_copy_equals_positions_pass(small_inputs, name, policy):
    """The token-major engine (4) places the rows in its row copy, from the
    ranks and chunk offsets routing computed; the gathering engine (6) takes
    them from the separate positions pass.  Each row's arithmetic is the
    same on both, so whole episodes agree bit for bit only if every (token,
    slot) pair lands on a row of its own segment in both."""
    import torch
    inp = small_inputs[name]
    placed = run_episode(inp, policy, gemm=4)[0].cpu()
    passed = run_episode(inp, policy, gemm=6)[0].cpu()
    assert torch.equal(placed.view(torch.int16), passed.view(torch.int16))


@pytest.mark.parametrize("name", ["small_bf16", "small_shared_bf16"])
@pytest.mark.parametrize("gemm", [4, 7, 1])
def test_routing_ahead_equals_step_by_step(small_inputs, name, gemm):
    """eb_episode routes step i+1 beside step i's GEMM 2, into the gate buffer
    the micro-batch's current routing does not use; eb_moe_step routes every
    step at its start.  Both paths must give the same RunSets, trace,
    utilisation and final hidden states, bit for bit, on the token-major,
    fused-combine and weight-major engines."""
    import torch
    import cross_layer_expert_b200 as eb
    from _common import lib_config
    inp = small_inputs[name]
    for policy in (0, 1):
        h_ep, rows_ep, layers_ep, util_ep, steps_ep = run_episode(inp, policy, gemm=gemm)
        ctx = eb.Context(lib_config(inp.wl, policy, gemm=gemm))
        try:
            hidden = inp.h0.clone()
            ctx.eb_reset()
            for _ in range(steps_ep):
                assert ctx.eb_moe_step(inp.logits, hidden, inp.w_gateup, inp.w_down,
                                       want_runset=True) != 0
            assert ctx.eb_moe_step(inp.logits, hidden, inp.w_gateup, inp.w_down,
                                   want_runset=True) == 0
            assert ctx.eb_sync_status() == eb.EB_OK
            rows, layers = ctx.eb_trace()
            util = ctx.eb_utilization()
        finally:
            ctx.close()
        assert np.array_equal(rows, rows_ep) and np.array_equal(layers, layers_ep), policy
        assert util == util_ep, policy
        assert torch.equal(hidden.cpu().view(torch.int16), h_ep.cpu().view(torch.int16)), policy


def test_overlapped_episodes_repeat_and_mix_with_single_steps(small_inputs):
    """One context: an episode, a second episode, a reset and a few single
    steps, then a third episode.  The overlapped episodes leave nothing
    pending (the last step's deferred combine is flushed, the routing done
    ahead of a step that never comes changes nothing), so every episode
    equals the first bit for bit."""
    import torch
    import cross_layer_expert_b200 as eb
    from _common import lib_config
    inp = small_inputs["small_bf16"]
    ctx = eb.Context(lib_config(inp.wl, osch.MAXUTIL, gemm=4))
    try:
        outs = []
        for rep in range(2):
            hidden = inp.h0.clone()
            ctx.eb_episode(inp.logits, hidden, inp.w_gateup, inp.w_down)
            assert ctx.eb_sync_status() == eb.EB_OK
            outs.append(hidden.cpu())
        ctx.eb_reset()
        hidden = inp.h0.clone()
        for _ in range(3):
            ctx.eb_moe_step(inp.logits, hidden, inp.w_gateup, inp.w_down)
        hidden = inp.h0.clone()
        ctx.eb_episode(inp.logits, hidden, inp.w_gateup, inp.w_down)
        assert ctx.eb_sync_status() == eb.EB_OK
        outs.append(hidden.cpu())
    finally:
        ctx.close()
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))


@pytest.mark.parametrize("m", [1, 2, 4])
def test_small_episode_m_sweep(small_inputs, small_expected, m):
    inp = small_inputs["small_bf16"]
    for policy in (0, 1, 3):
        hidden, rows, layers, util, steps = run_episode(inp, policy, m=m)
        check_schedule(rows, layers, util, steps, oracle_episode(inp, policy, m), inp.wl.M)
        assert_close(hidden.float().cpu().numpy(), small_expected["small_bf16"], "bf16")


def test_step_by_step_runset_and_noop_after_finish(small_inputs):
    """eb_moe_step returns each RunSet; once S is empty a step does nothing."""
    import cross_layer_expert_b200 as eb
    from _common import lib_config
    inp = small_inputs["small_bf16"]
    wl = inp.wl
    ref = oracle_episode(inp, osch.CUMUTIL)
    ctx = eb.Context(lib_config(wl, osch.CUMUTIL))
    hidden = inp.h0.clone()
    ctx.eb_reset()
    for st in ref["steps"]:
        got = ctx.eb_moe_step(inp.logits, hidden, inp.w_gateup, inp.w_down, want_runset=True)
        assert got == sum(1 << j for j in st["runset"])
    snap = hidden.clone()
    assert ctx.eb_moe_step(inp.logits, hidden, inp.w_gateup, inp.w_down, want_runset=True) == 0
    assert (hidden.view(-1) == snap.view(-1)).all()
    assert ctx.eb_utilization() == (ref["num"], ref["den"], ref["den_sep"])
    ctx.close()


def test_nonfinite_logit_reported_by_step(small_inputs):
    import cross_layer_expert_b200 as eb
    from _common import lib_config
    inp = small_inputs["small_bf16"]
    lg = inp.logits.clone()
    lg[2, 0, 5, 1] = float("inf")
    ctx = eb.Context(lib_config(inp.wl, osch.CUMUTIL))
    ctx.eb_episode(lg, inp.h0.clone(), inp.w_gateup, inp.w_down)
    assert ctx.eb_sync_status() == eb.EB_ERR_NONFINITE
    ctx.close()
