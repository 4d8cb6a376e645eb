"""Router mode: routing scores projected from the hidden states on the
device ([EB] §2.1 topk(G(h'_l)) with a linear scorer), so the chain is
data-dependent.  The projection is checked against the oracle's float64
product; episodes against the oracle's routed chain, and -- the property the
method rests on -- scheduling still moves only timing: MaxUtil's final hidden
states equal the lock-step run's bit for bit."""
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


def _check_router_episode(torch, wl, inp, router, toks, policies):
    """The top-k decisions are taken on the kernel's float32 scores on both
    sides (a float decides an integer): the oracle routes the scores the GPU
    computed.  Then (1) the schedule, trace and utilisation match the oracle
    bit for bit; (2) the final hidden states of `toks` match the oracle's
    chain within the bf16 tolerance; (3) every step's scores match the
    projection of the oracle's own hidden states; (4) MaxUtil equals
    lock-step bit for bit."""
    import cross_layer_expert_b200 as eb
    routers = [router[l].float().cpu().numpy().astype(np.float64) for l in range(wl.L)]
    lock = _episode(eb, torch, wl, inp, router, osch.LOCKSTEP)
    sc = lock[5]
    assert np.isfinite(sc).all()
    loads = oracle.route_all(sc, wl.k, wl.D)[3]
    h0 = np.stack([inp.h0_np[j, t] for (j, t) in toks])
    want = omoe.forward_tokens(h0, lambda j, l: sc[j, l], toks, wl.L, wl.E, wl.k, wl.n_shared,
                               wl.dtype, inp.expert)
    # the scores are the projection of the hidden states: against the oracle's
    # own chain (which drifts from the GPU's by bf16 rounding only)
    _, seen = orouter.forward_tokens_routed(h0, lambda l: routers[l], toks, wl.L, wl.E, wl.k,
                                            wl.n_shared, wl.dtype, inp.expert)
    for l in range(wl.L):
        got = np.stack([sc[j, l, t] for (j, t) in toks]).astype(np.float64)
        assert np.all(np.abs(got - seen[l]) <= 5e-2 + 5e-2 * np.abs(seen[l])), l
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
    """Qwen3 per-layer sizes, 3 layers, sampled tokens."""
    wl = synth.get("qwen3_bf16").replace(L=3)
    inp = Inputs(wl)
    router = synth.router_torch(wl, device="cuda")
    rng = np.random.default_rng(41)
    toks = [(j, int(rng.integers(0, wl.T))) for j in range(wl.M)] + [(0, 0), (wl.M - 1, wl.T - 1)]
    _check_router_episode(torch, wl, inp, router, toks, (osch.MAXUTIL,))


def test_router_mode_rejects_unsupported_shapes(torch):
    import cross_layer_expert_b200 as eb
    wl = synth.get("small_shared_bf16")  # E = 12: not a multiple of 16
    ctx = eb.Context(lib_config(wl, osch.CUMUTIL))
    w = torch.zeros((wl.L, wl.E, wl.H), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(eb.EbError):
        ctx.eb_set_router(w)
    ctx.close()
