"""Full-size parity: the Qwen3-30B-A3B, Moonlight-16B-A3B and long-context
workloads in the launch configuration bench.py times (eb_episode, tensor-core
GEMMs), against the oracle.

Schedules, traces and utilisation totals are compared bit for bit over the
whole episode.  Outputs are compared on sampled tokens, each followed by the
oracle through all L layers (a token's trajectory does not depend on the
schedule), within the bf16 tolerance.
"""
import gc

import numpy as np
import pytest

import synth
from oracle import schedule as osch

from _common import Inputs, assert_close, check_schedule, oracle_episode, oracle_hidden, run_episode

pytestmark = pytest.mark.gpu


def _free():
    import torch
    gc.collect()
    torch.cuda.empty_cache()


@pytest.fixture(scope="module")
def torch_mod():
    import torch
    from cross_layer_expert_b200 import build
    build.build()
    return torch


@pytest.mark.parametrize("name,policy", [("qwen3_bf16", osch.MAXUTIL),
                                         ("moonlight_bf16", osch.CUMUTIL),
                                         ("longctx_bf16", osch.MAXUTIL)])
def test_full_size_episode(torch_mod, name, policy):
    wl = synth.get(name)
    inp = Inputs(wl)
    try:
        hidden, rows, layers, util, steps = run_episode(inp, policy)
        check_schedule(rows, layers, util, steps, oracle_episode(inp, policy), wl.M)
        # rows and segments of every step are consistent with the RunSet sizes
        for r in rows:
            n_sel = bin(int(r[0])).count("1")
            assert int(r[4]) == n_sel * wl.T * (wl.k + wl.n_shared)
        # sampled tokens: the first, a middle and the last token of a few micro-batches
        toks = [(0, 0), (wl.M // 2, wl.T // 2), (wl.M - 1, wl.T - 1), (1, (7 * wl.T) // 9)]
        want = oracle_hidden(inp, toks)
        got = np.stack([hidden[j, t].float().cpu().numpy() for (j, t) in toks])
        assert_close(got, want, "bf16", name)
        # the other policies' schedules (routing + scheduling only, fast)
        from _common import lib_config
        import cross_layer_expert_b200 as eb
        for p in (osch.CUMUTIL, osch.MAXUTIL, osch.DIFFPEAK, osch.LOCKSTEP):
            if p == policy:
                continue
            ctx = eb.Context(lib_config(wl, p, compute=0))
            n = ctx.eb_episode(inp.logits, None, None, None)
            r2, l2 = ctx.eb_trace()
            check_schedule(r2, l2, ctx.eb_utilization(), n, oracle_episode(inp, p), wl.M)
            ctx.close()
    finally:
        del inp
        _free()


@pytest.mark.parametrize("M,D", [(4, 8), (8, 16), (16, 32), (32, 64), (32, 8)])
def test_sweep_schedules(torch_mod, M, D):
    """Routing + scheduling only at the Qwen3 shape with D up to 64 virtual
    ranks and M up to 32 micro-batches (T = 256): traces bit for bit.  MaxUtil
    at M = 32 runs a 4-layer stack (the exhaustive oracle enumerates ~15M
    subsets per step)."""
    import cross_layer_expert_b200 as eb
    from _common import lib_config
    for episode in (0, 1):
        wl = synth.get("sweep", M=M, D=D)
        for policy in (osch.CUMUTIL, osch.MAXUTIL, osch.DIFFPEAK, osch.LOCKSTEP):
            w2 = wl.replace(L=4) if (policy == osch.MAXUTIL and M == 32) else wl
            if episode == 1 and policy != osch.CUMUTIL:
                continue
            inp = Inputs(w2, with_weights=False)
            if episode:
                import torch
                inp.logits_np = synth.logits(w2, episode=episode)
                inp.logits = torch.from_numpy(inp.logits_np).cuda()
            ctx = eb.Context(lib_config(w2, policy, compute=0))
            n = ctx.eb_episode(inp.logits, None, None, None)
            rows, layers = ctx.eb_trace()
            check_schedule(rows, layers, ctx.eb_utilization(), n, oracle_episode(inp, policy), w2.M)
            ctx.close()
