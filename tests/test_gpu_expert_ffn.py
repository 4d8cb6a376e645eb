"""eb_expert_ffn: the expert computation of expert parallelism ([EB] §2.2 --
between the dispatch and combine all-to-alls a rank runs its experts' SwiGLU
FFNs, [EB] Eq. (1) expert_i, on the rows it received), checked row by row
against the oracle's expert FFN on seeded rows, with segments in any order,
repeated experts, empty and ragged segments, shared experts, and the tensor-core
and SIMT engines."""
import numpy as np
import pytest

import synth
from oracle import moe as omoe

from _common import assert_close, lib_config

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    import torch as t
    from cross_layer_expert_b200 import build
    build.build()
    return t


def _segments(wl, rng, n_seg, max_rows, cap):
    """A random segment table: (layer, expert) pairs, repeats allowed, sizes
    from 0 to max_rows, total within the capacity."""
    Et = wl.E + wl.n_shared
    layers = rng.integers(0, wl.L, size=n_seg)
    experts = rng.integers(0, Et, size=n_seg)
    sizes = rng.integers(0, max_rows + 1, size=n_seg)
    sizes[rng.integers(0, n_seg)] = 0  # one empty segment
    while sizes.sum() > cap:
        sizes //= 2
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    return layers, experts, off


def _check(torch, name, n_seg, max_rows, scale, L=None, seed=0):
    import cross_layer_expert_b200 as eb
    wl = synth.get(name) if L is None else synth.get(name).replace(L=L)
    rng = np.random.default_rng(1234 + seed)
    ctx = eb.Context(lib_config(wl, eb.MAXUTIL))
    try:
        cap = wl.M * wl.T * (wl.k + wl.n_shared)
        layers, experts, off = _segments(wl, rng, n_seg, max_rows, cap)
        R = int(off[-1])
        dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
        x = torch.from_numpy(rng.standard_normal((R, wl.H)) * scale).to(dt)
        wgu, wdn = synth.weights_torch(wl, device="cuda")
        rows = x.cuda()
        out = torch.full((R, wl.H), float("nan"), dtype=dt, device="cuda")
        ctx.eb_expert_ffn(rows, off, layers, experts, out, wgu, wdn)
        got = out.float().cpu().numpy().astype(np.float64)
        xs = x.float().numpy().astype(np.float64)
        rms = []
        for i in range(len(layers)):
            a, b = int(off[i]), int(off[i + 1])
            if a == b:
                continue
            gu = wgu[int(layers[i]), int(experts[i])].float().cpu().numpy().astype(np.float64)
            dn = wdn[int(layers[i]), int(experts[i])].float().cpu().numpy().astype(np.float64)
            want = omoe.expert_ffn(xs[a:b], gu[:wl.F], gu[wl.F:], dn, wl.dtype)
            assert_close(got[a:b], want, wl.dtype, f"{name} segment {i} ({layers[i]}, {experts[i]})")
            rms.append(np.sqrt(np.mean(want ** 2)))
        # outputs of order one, so the tolerance means something
        assert np.median(rms) > 0.3, np.median(rms)
        return ctx.eb_engines()
    finally:
        ctx.close()


@pytest.mark.parametrize("name,scale", [("small_bf16", 8.0), ("small_shared_bf16", 8.0),
                                        ("tiny_f32", 6.0)])
def test_expert_ffn_matches_oracle(torch, name, scale):
    _check(torch, name, n_seg=24, max_rows=300, scale=scale)


def test_expert_ffn_full_width(torch):
    """The Qwen3-30B-A3B expert shape (H = 2048, F = 768) on two layers: the
    token-major tensor-core engine, segments spanning several 128-row chunks
    and ragged tails."""
    _check(torch, "qwen3_bf16", n_seg=10, max_rows=700, scale=3.0, L=2, seed=1)


def test_expert_ffn_rejects_bad_tables(torch):
    import cross_layer_expert_b200 as eb
    wl = synth.get("small_bf16")
    ctx = eb.Context(lib_config(wl, eb.MAXUTIL))
    try:
        wgu, wdn = synth.weights_torch(wl, device="cuda")
        rows = torch.zeros((10, wl.H), dtype=torch.bfloat16, device="cuda")
        out = torch.zeros_like(rows)
        bad = [([0, 5, 9], [0, 0], [1, 2]),     # does not end at R
               ([0, 6, 4, 10], [0, 0, 0], [1, 2, 3]),  # not ascending
               ([0, 10], [wl.L], [0]),          # layer out of range
               ([0, 10], [0], [wl.E])]          # expert out of range (no shared experts)
        for off, lay, ex in bad:
            with pytest.raises(eb.EbError) as err:
                ctx.eb_expert_ffn(rows, off, lay, ex, out, wgu, wdn)
            assert err.value.status == eb.EB_ERR_INVALID_ARG
        cap = wl.M * wl.T * wl.k
        big = torch.zeros((cap + 1, wl.H), dtype=torch.bfloat16, device="cuda")
        with pytest.raises(eb.EbError) as err:
            ctx.eb_expert_ffn(big, [0, cap + 1], [0], [0], torch.zeros_like(big), wgu, wdn)
        assert err.value.status == eb.EB_ERR_UNSUPPORTED
        # an empty call does nothing
        ctx.eb_expert_ffn(rows[:0], [0], [], [], out[:0], wgu, wdn)
    finally:
        ctx.close()
