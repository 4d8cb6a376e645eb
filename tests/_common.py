"""Shared helpers of the GPU parity tests: run episodes through the C ABI and
compute the oracle's expectations from the same seeded inputs.

Expected values come only from ``oracle`` (never from the CUDA path); inputs
come only from ``synth``.
"""
from __future__ import annotations

import numpy as np

import oracle
import synth
from oracle import moe as omoe

# outputs: bf16 max-abs 2e-2 / relative 1e-2; fp32 1e-5 (allclose semantics:
# |gpu - ref| <= atol + rtol * |ref|)
TOL = {"bf16": (2e-2, 1e-2), "f32": (1e-5, 1e-5)}


def lib_config(wl: synth.Workload, policy: int, m: int = 0, gemm: int = 0, compute=None):
    import cross_layer_expert_b200 as eb
    return eb.make_config(L=wl.L, E=wl.E, k=wl.k, H=wl.H, F=wl.F, D=wl.D, M=wl.M, T=wl.T,
                          n_shared=wl.n_shared, renorm=1,
                          dtype=eb.DTYPE_BF16 if wl.dtype == "bf16" else eb.DTYPE_F32,
                          policy=policy, m=m or wl.m_default, residual=1,
                          compute=int(wl.compute if compute is None else compute), gemm=gemm)


class Inputs:
    """Seeded inputs of one workload, on the GPU and (lazily) on the host."""

    def __init__(self, wl: synth.Workload, device="cuda", with_weights=True):
        import torch
        self.wl = wl
        self.logits_np = synth.logits(wl)
        self.logits = torch.from_numpy(self.logits_np).to(device)
        self.h0 = synth.hidden_torch(wl).to(device)
        self.h0_np = self.h0.float().cpu().numpy().astype(np.float64)
        if with_weights and wl.compute:
            self.w_gateup, self.w_down = synth.weights_torch(wl, device=device)
        else:
            self.w_gateup = self.w_down = None
        self._cache = {}
        self._cache_layer = None

    def expert(self, l: int, e: int):
        """(w_gate [F,H], w_up [F,H], w_down [H,F]) float64 on the host (only
        the current layer's experts are kept)."""
        key = (l, e)
        if l != self._cache_layer:
            self._cache = {}
            self._cache_layer = l
        if key not in self._cache:
            gu = self.w_gateup[l, e].float().cpu().numpy().astype(np.float64)
            dn = self.w_down[l, e].float().cpu().numpy().astype(np.float64)
            self._cache[key] = (gu[:self.wl.F], gu[self.wl.F:], dn)
        return self._cache[key]

    def clear_cache(self):
        self._cache = {}


def run_episode(inp: Inputs, policy: int, m: int = 0, gemm: int = 0):
    """One whole episode through eb_episode; returns (hidden, trace rows, layers,
    (num, den, den_sep), steps)."""
    import cross_layer_expert_b200 as eb
    wl = inp.wl
    ctx = eb.Context(lib_config(wl, policy, m, gemm))
    hidden = inp.h0.clone()
    steps = ctx.eb_episode(inp.logits, hidden, inp.w_gateup, inp.w_down)
    assert ctx.eb_sync_status() == eb.EB_OK
    rows, layers = ctx.eb_trace()
    util = ctx.eb_utilization()
    ctx.close()
    return hidden, rows, layers, util, steps


def oracle_loads(inp: Inputs, expert_rank=None):
    if expert_rank is not None:
        wl = inp.wl
        return oracle.route_all(inp.logits_np, wl.k, wl.D, expert_rank=expert_rank)[3]
    if getattr(inp, "_loads", None) is None:
        wl = inp.wl
        inp._loads = oracle.route_all(inp.logits_np, wl.k, wl.D)[3]
    return inp._loads


def maxutil_impl(M: int):
    """The oracle's MaxUtil for M micro-batches: the Python enumeration up to
    12, the plain-C forward enumeration over every bitmask up to 20, and the
    plain-C complement enumeration (pinned against the forward one) beyond."""
    from oracle import native
    if M <= 12:
        return None
    return native.maxutil_plain if M <= 20 else native.maxutil


def oracle_episode(inp: Inputs, policy: int, m: int = 0, expert_rank=None):
    wl = inp.wl
    return oracle.run_episode(oracle_loads(inp, expert_rank), policy, m or wl.m_default,
                              maxutil_impl=maxutil_impl(wl.M))


def check_schedule(rows, layers, util, steps, ref, M: int):
    """Bit-exact comparison of the device trace with the oracle's episode."""
    assert steps == len(ref["steps"]), (steps, len(ref["steps"]))
    assert rows.shape[0] == len(ref["steps"])
    for i, st in enumerate(ref["steps"]):
        mask = sum(1 << j for j in st["runset"])
        assert int(rows[i, 0]) == mask, (i, rows[i], st)
        assert int(rows[i, 1]) == st["sumW"] and int(rows[i, 2]) == st["maxW"]
        assert int(rows[i, 3]) == st["summax"]
        want = [st["layers"].get(j, -1) for j in range(M)]
        assert layers[i].tolist() == want, (i, layers[i], want)
    assert tuple(util) == (ref["num"], ref["den"], ref["den_sep"])


def oracle_hidden(inp: Inputs, tokens):
    """Oracle final hidden state of the listed (j, t) tokens after all L layers."""
    wl = inp.wl
    h0 = np.stack([inp.h0_np[j, t] for (j, t) in tokens])
    return omoe.forward_tokens(h0, lambda j, l: inp.logits_np[j, l], tokens, wl.L, wl.E, wl.k,
                               wl.n_shared, wl.dtype, inp.expert)


def assert_close(got, want, dtype: str, what=""):
    atol, rtol = TOL[dtype]
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    err = np.abs(got - want)
    bad = err > atol + rtol * np.abs(want)
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; "
                           f"max abs err {err.max():.3g}")
