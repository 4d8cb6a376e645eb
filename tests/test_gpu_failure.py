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
