"""Expert placement (an arbitrary expert -> virtual-rank map, as a load
balancer such as EPLB would choose it): loads and whole episodes against the
oracle under the same placement, bit for bit."""
import numpy as np
import pytest

import synth
from oracle import schedule as osch

from _common import Inputs, check_schedule, lib_config, oracle_episode

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    import torch as t
    from cross_layer_expert_b200 import build
    build.build()
    return t


def test_loads_mapped_matches_oracle(torch):
    import cross_layer_expert_b200 as eb
    import oracle
    rng = np.random.default_rng(21)
    for (M, E, D) in [(8, 128, 8), (5, 12, 5), (3, 16, 7), (32, 256, 64), (1, 5, 1)]:
        h = rng.integers(0, 1000, size=(M, E)).astype(np.int32)
        emap = rng.integers(0, D, size=E).astype(np.int32)
        w = torch.empty((M, D), dtype=torch.int32, device="cuda")
        status = torch.zeros((1,), dtype=torch.int32, device="cuda")
        eb.eb_loads_mapped(torch.from_numpy(h).cuda(), D, torch.from_numpy(emap).cuda(), w, status)
        assert np.array_equal(w.cpu().numpy(), oracle.loads(h, D, emap.tolist()))
        assert int(status.item()) == eb.EB_OK
    # an out-of-range rank is reported, and its expert's counts dropped
    h = rng.integers(0, 10, size=(2, 8)).astype(np.int32)
    emap = np.array([0, 1, 2, 3, 0, 1, 9, 3], dtype=np.int32)
    w = torch.empty((2, 4), dtype=torch.int32, device="cuda")
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    eb.eb_loads_mapped(torch.from_numpy(h).cuda(), 4, torch.from_numpy(emap).cuda(), w, status)
    assert int(status.item()) == eb.EB_ERR_INVALID_ARG
    keep = emap.copy()
    keep[6] = 0
    want = oracle.loads(np.where(np.arange(8) == 6, 0, h), 4, keep.tolist())
    assert np.array_equal(w.cpu().numpy(), want)


@pytest.mark.parametrize("name,policy,compute", [("small_bf16", osch.MAXUTIL, True),
                                                 ("small_shared_bf16", osch.CUMUTIL, True),
                                                 ("qwen3_bf16", osch.MAXUTIL, False),
                                                 ("qwen3_bf16", osch.DIFFPEAK, False)])
def test_episode_under_placement_matches_oracle(torch, name, policy, compute):
    """A seeded random placement changes the loads, hence the schedule; the
    trace, RunSets and utilisation still match the oracle bit for bit, and
    the final hidden states still equal the lock-step run's (scheduling
    moves only timing, under any placement)."""
    import cross_layer_expert_b200 as eb
    wl = synth.get(name)
    inp = Inputs(wl, with_weights=compute)
    rng = np.random.default_rng(31)
    emap = rng.integers(0, wl.D, size=wl.E).tolist()
    ref = oracle_episode(inp, policy, expert_rank=emap)
    ctx = eb.Context(lib_config(wl, policy, compute=compute))
    ctx.eb_set_expert_map(emap)
    hidden = inp.h0.clone() if compute else None
    n = ctx.eb_episode(inp.logits, hidden, inp.w_gateup, inp.w_down)
    assert ctx.eb_sync_status() == eb.EB_OK
    rows, layers = ctx.eb_trace()
    check_schedule(rows, layers, ctx.eb_utilization(), n, ref, wl.M)
    # the placement changes the loads: the default map gives other totals
    default = oracle_episode(inp, policy)
    assert (default["num"], default["den"]) != (ref["num"], ref["den"]) or \
        default["den_sep"] != ref["den_sep"]
    # None restores the contiguous map
    ctx.eb_set_expert_map(None)
    n2 = ctx.eb_episode(inp.logits, inp.h0.clone() if compute else None, inp.w_gateup, inp.w_down)
    rows2, layers2 = ctx.eb_trace()
    check_schedule(rows2, layers2, ctx.eb_utilization(), n2, default, wl.M)
    ctx.close()
    if compute:
        lock = eb.Context(lib_config(wl, osch.LOCKSTEP))
        h_lock = inp.h0.clone()
        lock.eb_episode(inp.logits, h_lock, inp.w_gateup, inp.w_down)
        lock.close()
        assert torch.equal(hidden.view(torch.int16), h_lock.view(torch.int16))


def test_set_expert_map_rejects_bad_ranks(torch):
    import cross_layer_expert_b200 as eb
    wl = synth.get("small_bf16")
    ctx = eb.Context(lib_config(wl, osch.CUMUTIL, compute=False))
    for bad in ([wl.D] + [0] * (wl.E - 1), [-1] + [0] * (wl.E - 1)):
        with pytest.raises(eb.EbError):
            ctx.eb_set_expert_map(bad)
    ctx.close()
