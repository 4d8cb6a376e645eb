"""Degenerate and boundary cases of the step against the oracle: one token,
one micro-batch, one rank (u = 1), every expert per token (k = E), one
expert per rank (D = E), m = M (MaxUtil reduces to lock-step), a ragged
token count, the largest expert count and one that leaves routing lanes
padded -- on the default tensor-core engine, on SIMT and with the combine
fused into GEMM 2."""
import numpy as np
import pytest

import synth
from oracle import schedule as osch

from _common import Inputs, assert_close, check_schedule, oracle_episode, oracle_hidden, run_episode

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    import torch as t
    from cross_layer_expert_b200 import build
    build.build()
    return t


CASES = {
    # name: overrides of small_bf16 (L6 E16 k4 H256 F384 D4 M4 T200)
    "one_token": dict(M=1, T=1, m=1),
    "one_microbatch": dict(M=1, m=1, T=37),
    "one_rank": dict(D=1),
    "every_expert": dict(k=16, T=45),
    "rank_per_expert": dict(D=16),
    "m_equals_M": dict(m=4),
    "ragged_tokens": dict(T=129, M=3, m=2),
    # 8 experts per lane in routing (one row per warp) and 256 experts in the
    # rows' per-expert token masks and ranks
    "many_experts": dict(E=256, k=8, D=8, T=150),
    # experts that do not fill the last lane column (padded lanes), ragged T
    "odd_experts": dict(E=40, k=5, D=8, T=77),
}


@pytest.mark.parametrize("gemm", [0, 2, 7])
@pytest.mark.parametrize("case", sorted(CASES))
def test_edge_case_episode_matches_oracle(torch, case, gemm):
    wl = synth.get("small_bf16", L=3, **CASES[case])
    inp = Inputs(wl)
    toks = [(j, t) for j in range(wl.M) for t in range(wl.T)]
    want = oracle_hidden(inp, toks).reshape(wl.M, wl.T, wl.H)
    for policy in (osch.MAXUTIL, osch.CUMUTIL, osch.LOCKSTEP):
        hidden, rows, layers, util, steps = run_episode(inp, policy, gemm=gemm)
        ref = oracle_episode(inp, policy)
        check_schedule(rows, layers, util, steps, ref, wl.M)
        assert_close(hidden.float().cpu().numpy(), want, wl.dtype, f"{case} p{policy}")
        num, den, den_sep = util
        if wl.D == 1 or wl.k == wl.E:
            assert num == den == den_sep  # one rank, or every rank equally loaded
        if wl.m_default >= wl.M:
            assert steps == wl.L          # every step runs every micro-batch
