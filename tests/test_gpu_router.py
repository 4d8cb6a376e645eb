"""Router mode: routing scores projected from the hidden states on the
device ([EB] §2.1 topk(G(h'_l)) with a linear scorer), so the chain is
data-dependent.  The projection is checked against the oracle's float64
product; episodes against the oracle's own routed chain -- the oracle computes
its own scores from its own hidden states and takes every routing decision on
them -- and, the property the method rests on, scheduling still moves only
timing: MaxUtil's final hidden states equal the lock-step run's bit for bit."""
import numpy as np
import pytest

import synth
import oracle
from oracle import moe as omoe
from oracle import router as orouter
from oracle import schedule as osch

from _common import Inputs, assert_close, check_schedule, lib_config

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    import torch as t
    from cross_layer_expert_b200 import build
    build.build()
    return t


@pytest.mark.parametrize("n,H,E", [(1000, 2048, 128), (77, 256, 16), (300, 2048, 64),
                                   (129, 512, 256), (1, 64, 32)])
def test_router_scores_match_oracle(torch, n, H, E):
    import cross_layer_expert_b200 as eb
    g = torch.Generator().manual_seed(n * 7 + E)
    h = torch.randn((n, H), generator=g).to(torch.bfloat16)
    w = (torch.randn((E, H), generator=g) * (2.0 / H ** 0.5)).to(torch.bfloat16)
    out = torch.full((n, E), float("nan"), dtype=torch.float32, device="cuda")
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    eb.eb_router(h.cuda(), w.cuda(), out, status)
    torch.cuda.synchronize()
    assert int(status.item()) == eb.EB_OK
    ref = orouter.router_logits(h.float().numpy(), w.float().numpy())
    got = out.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - ref) <= 1e-4 + 1e-4 * np.abs(ref)), np.abs(got - ref).max()


def _episode(eb, torch, wl, inp, router, policy):
    """A router-mode episode; returns (hidden, trace rows, layers, util, steps,
    the scores every step computed [M, L, T, E])."""
    ctx = eb.Context(lib_config(wl, policy))
    scores = torch.full((wl.M, wl.L, wl.T, wl.E), float("nan"), dtype=torch.float32, device="cuda")
    ctx.eb_set_router(router, scores)
    hidden = inp.h0.clone()
    n = ctx.eb_episode(None, hidden, inp.w_gateup, inp.w_down)
    assert ctx.eb_sync_status() == eb.EB_OK
    rows, layers = ctx.eb_trace()
    util = ctx.eb_utilization()
    ctx.close()
    return hidden, rows, layers, util, n, scores.cpu().numpy()


# Bound on |device score - oracle score| at layer l: tau_l(s) = (TAU0 + TAU_L
# l) (1 + |s|).  At layer 0 both sides project the same hidden states, and
# the device projection was measured within 1e-4 + 1e-4 |s| of the float64
# product (above).  Each later layer's input also carries the rounding of the
# bf16 hidden state: the two chains round the same values, but a value close
# to a rounding boundary can land one unit in the last place apart, and the
# next layer carries that on; TAU_L per layer covers it (the largest
# deviation seen per layer is printed).
TAU0, TAU_L = 1e-4, 3e-3


def _tau(s, l):
    return (TAU0 + TAU_L * l) * (1.0 + np.abs(np.asarray(s, dtype=np.float64)))


def _topk_sets(scores, k):
    """Top-k expert sets of score rows [n, E] (descending score, lower index
    first on equal scores), as sorted index arrays [n, k]."""
    order = np.argsort(-np.asarray(scores, dtype=np.float32), axis=1, kind="stable")
    return np.sort(order[:, :k], axis=1)


def _oracle_chain(wl, inp, routers, gpu_scores):
    """The routed chain of every token on the oracle's side: each layer's
    scores are the float64 projection of the oracle's own hidden states
    (decided in float32), routed by oracle.route, then the oracle's MoE layer.

    The device's scores are used only to see which experts the device chose.
    Where the oracle's own k-th and (k+1)-th scores lie within 2 tau(s) of each
    other (a near tie: both choices are correct within the projection error),
    the device's choice is accepted if it is a valid top-k of the oracle's
    scores within that bound, and the oracle continues with it; everywhere
    else the device must have chosen exactly the oracle's set.

    Returns (final hidden [M*T, H], loads [M, L, D], near-tie count, adopted
    count, the largest |device score - oracle score| of each layer)."""
    M, L, T, E, k = wl.M, wl.L, wl.T, wl.E, wl.k
    h = inp.h0_np.reshape(M * T, wl.H).copy()
    loads = np.zeros((M, L, wl.D), dtype=np.int64)
    near = adopted = 0
    worst = []
    for l in range(L):
        osc = orouter.router_logits(h, routers[l]).astype(np.float32)
        gsc = gpu_scores[:, l].reshape(M * T, E)
        dev = np.abs(gsc.astype(np.float64) - osc)
        worst.append(float(dev.max()))
        assert np.all(dev <= _tau(osc, l)), (l, float(dev.max()))
        idx, gate = oracle.route(osc, k)
        # near ties of the oracle's own decision
        srt = -np.sort(-osc.astype(np.float64), axis=1)
        gap = srt[:, k - 1] - srt[:, k] if k < E else np.full(M * T, np.inf)
        tie = gap <= 2 * _tau(srt[:, k - 1], l)
        near += int(tie.sum())
        want = np.sort(idx, axis=1)
        got = _topk_sets(gsc, k)
        same = np.all(got == want, axis=1)
        assert np.all(same | tie), f"layer {l}: {int((~same & ~tie).sum())} tokens routed " \
                                   "differently away from a near tie"
        for t in np.nonzero(~same)[0]:
            # valid under the oracle's scores within the bound: every chosen
            # expert scores at least every unchosen one, less 2 tau
            sel = np.zeros(E, dtype=bool)
            sel[got[t]] = True
            lo = osc[t, sel].astype(np.float64).min()
            hi = osc[t, ~sel].astype(np.float64).max()
            assert lo >= hi - 2 * _tau(hi, l), (l, t)
            # the device's set, slots and renormalised gates as the oracle
            # forms them over that set (experts outside it masked far below)
            masked = np.where(sel, osc[t], np.float32(-1e30)).astype(np.float32)
            i1, g1 = oracle.route(masked[None], k)
            idx[t], gate[t] = i1[0], g1[0]
            adopted += 1
        hist = np.stack([oracle.histogram(idx[j * T:(j + 1) * T], E) for j in range(M)])
        loads[:, l] = oracle.loads(hist, wl.D)
        h = omoe.moe_layer(h, idx, gate, l, inp.expert, E, wl.n_shared, wl.dtype)
    return h, loads, near, adopted, worst


def _check_router_episode(torch, wl, inp, router, toks, policies):
    """The oracle runs its own routed chain (above) and so decides every
    routing on its own scores.  Then (1) every device score is within the
    near-tie bound of the oracle's; (2) routing equals the oracle's except at
    counted near ties, where the device's choice is valid under the oracle's
    scores; (3) the schedule, trace and utilisation equal the oracle's episode
    on that routing bit for bit; (4) the final hidden states of `toks` match
    the oracle's chain within the bf16 tolerance; (5) MaxUtil equals lock-step
    bit for bit."""
    import cross_layer_expert_b200 as eb
    routers = [router[l].float().cpu().numpy().astype(np.float64) for l in range(wl.L)]
    lock = _episode(eb, torch, wl, inp, router, osch.LOCKSTEP)
    sc = lock[5]
    assert np.isfinite(sc).all()
    final, loads, near, adopted, worst = _oracle_chain(wl, inp, routers, sc)
    print(f"router chain {wl.name} L={wl.L}: {near} near ties, {adopted} routed by the device's "
          f"valid choice, largest score deviation per layer "
          + " ".join(f"{x:.3g}" for x in worst))
    want = np.stack([final[j * wl.T + t] for (j, t) in toks])
    for policy in policies:
        hidden, rows, layers, util, n, sc2 = _episode(eb, torch, wl, inp, router, policy)
        # routing scores of a (micro-batch, layer) do not depend on the schedule
        assert np.array_equal(sc2, sc)
        check_schedule(rows, layers, util, n, oracle.run_episode(loads, policy, wl.m_default), wl.M)
        got = np.stack([hidden[j, t].float().cpu().numpy() for (j, t) in toks])
        assert_close(got, want, "bf16", f"router mode p{policy}")
        if policy == osch.MAXUTIL:
            assert torch.equal(hidden.view(torch.int16), lock[0].view(torch.int16))


def test_small_router_episode_matches_oracle(torch):
    wl = synth.get("small_bf16")
    inp = Inputs(wl)
    router = synth.router_torch(wl, device="cuda")
    toks = [(j, t) for j in range(wl.M) for t in range(wl.T)]
    _check_router_episode(torch, wl, inp, router, toks, (osch.MAXUTIL, osch.CUMUTIL, osch.DIFFPEAK))


def test_qwen3_shape_router_episode(torch):
    """Qwen3 per-layer sizes (E = 128, k = 8, H = 2048, F = 768, D = 8, M = 8),
    3 layers of 256 tokens per micro-batch: the oracle's chain covers every
    token, so every routing decision and every output is checked."""
    wl = synth.get("qwen3_bf16").replace(L=3, T=256)
    inp = Inputs(wl)
    router = synth.router_torch(wl, device="cuda")
    toks = [(j, t) for j in range(wl.M) for t in range(wl.T)]
    _check_router_episode(torch, wl, inp, router, toks, (osch.MAXUTIL, osch.CUMUTIL))


def test_router_mode_rejects_unsupported_shapes(torch):
    import cross_layer_expert_b200 as eb
    wl = synth.get("small_shared_bf16")  # E = 12: not a multiple of 16
    ctx = eb.Context(lib_config(wl, osch.CUMUTIL))
    w = torch.zeros((wl.L, wl.E, wl.H), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(eb.EbError):
        ctx.eb_set_router(w)
    ctx.close()
