"""Failure detection without a GPU fault: a bounded device wait that runs out
(an mbarrier nothing arrives on) reports EB_ERR_TIMEOUT through the status
word, and the context stays usable afterwards."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def test_bounded_wait_expires_with_status():
    import torch
    from cross_layer_expert_b200 import build
    build.build()
    import cross_layer_expert_b200 as eb
    import oracle
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    eb.eb_selftest_timeout(2_000_000, status)  # 2 ms
    torch.cuda.synchronize()
    assert int(status.item()) == eb.EB_ERR_TIMEOUT
    # the context is intact: a routing call still runs and is exact
    x = np.random.default_rng(3).standard_normal((100, 16)).astype(np.float32)
    idx = torch.empty((100, 2), dtype=torch.int32, device="cuda")
    gate = torch.empty((100, 2), dtype=torch.float32, device="cuda")
    hist = torch.empty((16,), dtype=torch.int32, device="cuda")
    eb.eb_route(torch.from_numpy(x).cuda(), 2, True, idx, gate, hist)
    assert np.array_equal(idx.cpu().numpy(), oracle.route(x, 2)[0])
    with pytest.raises(eb.EbError):
        eb.eb_selftest_timeout(10, status)  # below the accepted range


def test_host_side_argument_errors():
    """Bad arguments are rejected before any launch."""
    import torch
    import cross_layer_expert_b200 as eb
    from _common import lib_config
    import synth
    wl = synth.get("small_bf16")
    ctx = eb.Context(lib_config(wl, 0))
    lg = torch.zeros((wl.M, wl.L, wl.T, wl.E), device="cuda")
    with pytest.raises(eb.EbError) as e:
        ctx.eb_moe_step(lg, None, None, None)  # compute step without hidden / weights
    assert e.value.status == eb.EB_ERR_INVALID_ARG
    ctx.close()


def test_timed_out_context_refuses_steps_until_reset():
    """A step that gives up on a bounded wait can leave the fused combine's
    arrival counters part-counted.  The failure is injected on the host (the
    status word set to EB_ERR_TIMEOUT, every counter left non-zero); the
    context then refuses to step -- on the device, and on the host once the
    status has been seen -- until eb_reset, after which an episode on the
    fused engine matches the unfused engine bit for bit.  Without the reset
    the dirty counters would corrupt the combine: a control run that clears
    only the status word shows it."""
    import torch
    from cross_layer_expert_b200 import build
    build.build()
    import cross_layer_expert_b200 as eb
    import synth
    from oracle import schedule as osch
    from _common import Inputs, lib_config, run_episode
    wl = synth.get("small_bf16")
    inp = Inputs(wl)
    ref = run_episode(inp, osch.MAXUTIL, gemm=eb.GEMM_TM)[0].cpu().view(torch.int16)
    ctx = eb.Context(lib_config(wl, osch.MAXUTIL, gemm=eb.GEMM_TMC))
    try:
        assert ctx.eb_engines()[1] == eb.GEMM_TMC
        hidden = inp.h0.clone()
        ctx.eb_reset()
        assert ctx.eb_moe_step(inp.logits, hidden, inp.w_gateup, inp.w_down, want_runset=True) != 0
        ctx.eb_inject_status(eb.EB_ERR_TIMEOUT)
        snap = hidden.clone()
        with pytest.raises(eb.EbError) as e:
            ctx.eb_moe_step(inp.logits, hidden, inp.w_gateup, inp.w_down, want_runset=True)
        assert e.value.status == eb.EB_ERR_TIMEOUT
        assert torch.equal(hidden.view(torch.int16), snap.view(torch.int16))  # nothing ran
        with pytest.raises(eb.EbError) as e:  # refused on the host, nothing enqueued
            ctx.eb_moe_step(inp.logits, hidden, inp.w_gateup, inp.w_down)
        assert e.value.status == eb.EB_ERR_TIMEOUT
        assert ctx.eb_sync_status() == eb.EB_ERR_TIMEOUT
        # eb_episode starts with eb_reset: counters and status are cleared
        for _ in range(2):
            hidden = inp.h0.clone()
            ctx.eb_episode(inp.logits, hidden, inp.w_gateup, inp.w_down)
            assert ctx.eb_sync_status() == eb.EB_OK
            assert torch.equal(hidden.cpu().view(torch.int16), ref)
        # control: dirty counters with the status word cleared (never seen by
        # the host) and no reset -- the fused combine then goes wrong
        ctx.eb_reset()
        ctx.eb_inject_status(eb.EB_ERR_TIMEOUT)
        ctx.eb_inject_status(eb.EB_OK)
        hidden = inp.h0.clone()
        for _ in range(wl.M * wl.L):
            if ctx.eb_moe_step(inp.logits, hidden, inp.w_gateup, inp.w_down, want_runset=True) == 0:
                break
        assert ctx.eb_sync_status() == eb.EB_OK
        assert not torch.equal(hidden.cpu().view(torch.int16), ref)
    finally:
        ctx.close()
    with pytest.raises(eb.EbError):
        ctx2 = eb.Context(lib_config(wl, osch.MAXUTIL))
        try:
            ctx2.eb_inject_status(3)  # not a status code
        finally:
            ctx2.close()
