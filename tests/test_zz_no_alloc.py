"""The no-allocation routing + loads entry point against the allocating ones.

eb_route_loads_static is for callers that cannot allocate device memory (a
serving process whose memory is fixed at start-up, or one that must not call
cudaMalloc because it can synchronise the device).  Its counts live in the
library's fixed device array; this test calls it through the C ABI twice in a
row -- a large call, then smaller ones that leave stale counts of the earlier
calls in the array -- and checks each result against eb_route on every
micro-batch followed by eb_loads, and against the CPU oracle's routing and
loads.  It is collected last so that a failure here
stops a `-x` run only after every other test has run, and it passes both alone
in a fresh process and after the other tests.
"""
import ctypes

import numpy as np
import pytest

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    import torch  # noqa: F401
    from cross_layer_expert_b200 import build
    build.build()
    import cross_layer_expert_b200 as eb
    return eb.load()


def _reference(torch, eb, logits, k, renorm, D):
    n_mb, T, E = logits.shape
    idx = torch.empty((n_mb, T, k), dtype=torch.int32, device="cuda")
    gate = torch.empty((n_mb, T, k), dtype=torch.float32, device="cuda")
    hist = torch.empty((n_mb, E), dtype=torch.int32, device="cuda")
    for j in range(n_mb):
        eb.eb_route(logits[j], k, renorm, idx[j], gate[j], hist[j])
    w = torch.empty((n_mb, D), dtype=torch.int32, device="cuda")
    eb.eb_loads(hist, D, w)
    return idx, gate, w


def _static(torch, lib, logits, k, renorm, D):
    n_mb, T, E = logits.shape
    idx = torch.full((n_mb, T, k), -1, dtype=torch.int32, device="cuda")
    gate = torch.zeros((n_mb, T, k), dtype=torch.float32, device="cuda")
    w = torch.full((n_mb, D), -1, dtype=torch.int32, device="cuda")
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    rc = lib.eb_route_loads_static(ctypes.c_void_p(logits.data_ptr()), n_mb, T, E, k, int(renorm), D,
                                   ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(gate.data_ptr()),
                                   ctypes.c_void_p(w.data_ptr()), ctypes.c_void_p(status.data_ptr()),
                                   ctypes.c_void_p(s))
    assert rc == 0, rc
    return idx, gate, w, status


def _oracle(x, k, renorm, D):
    """idx, gate and loads of every micro-batch from the CPU oracle."""
    import oracle
    ridx, rgate, w = [], [], []
    for j in range(x.shape[0]):
        i, g = oracle.route(x[j], k, renorm)
        ridx.append(i)
        rgate.append(g)
        w.append(oracle.loads(oracle.histogram(i, x.shape[2]), D))
    return np.stack(ridx), np.stack(rgate), np.stack(w)


def test_no_alloc_route_loads_matches_allocating_entry_points(lib):
    import torch
    import cross_layer_expert_b200 as eb
    rng = np.random.default_rng(2026)
    cases = [  # (n_mb, T, E, k, D, renorm): large first, then smaller ones whose
        # counts leave stale entries of the earlier calls in the array
        (8, 1024, 128, 8, 8, True),
        (3, 200, 64, 6, 4, False),
        (2, 70, 24, 24, 8, True),  # k = E (every expert), E not a multiple of 32
        (2, 70, 40, 32, 8, False),  # the largest k, E not a multiple of 32
        (1, 17, 16, 2, 4, True),   # one micro-batch shorter than a 64-token chunk
    ]
    for (n_mb, T, E, k, D, renorm) in cases:
        x = rng.standard_normal((n_mb, T, E)).astype(np.float32)
        x[:, ::7, :] = np.round(x[:, ::7, :])  # some rows with tied logits
        logits = torch.from_numpy(x).cuda()
        idx, gate, w, status = _static(torch, lib, logits, k, renorm, D)
        ridx, rgate, rw = _reference(torch, eb, logits, k, renorm, D)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        # against the allocating entry points (same kernels' arithmetic) ...
        assert torch.equal(idx, ridx)
        assert torch.equal(w, rw)
        g, rg = gate.double().cpu().numpy(), rgate.double().cpu().numpy()
        assert np.all(np.abs(g - rg) <= 1e-6 * np.abs(rg) + 1e-12)
        # ... and against the CPU oracle, independently of any CUDA path
        oidx, ogate, ow = _oracle(x, k, renorm, D)
        assert np.array_equal(idx.cpu().numpy(), oidx)
        assert np.array_equal(w.cpu().numpy(), ow)
        assert np.all(np.abs(g - ogate) <= 1e-6 * np.abs(ogate) + 1e-12)
        assert int(w.sum().item()) == n_mb * T * k


def test_no_alloc_reports_nonfinite_logits(lib):
    """A NaN logit sets EB_ERR_NONFINITE in status_dev; the row is routed
    among the finite experts as eb_route does, and every count still lands."""
    import torch
    import cross_layer_expert_b200 as eb
    rng = np.random.default_rng(7)
    x = rng.standard_normal((2, 90, 32)).astype(np.float32)
    x[1, 65, 3] = np.nan
    logits = torch.from_numpy(x).cuda()
    idx, gate, w, status = _static(torch, lib, logits, 4, True, 4)
    ridx, rgate, rw = _reference(torch, eb, logits, 4, True, 4)
    torch.cuda.synchronize()
    assert int(status.item()) == eb.EB_ERR_NONFINITE
    assert torch.equal(idx, ridx)
    assert torch.equal(w, rw)
    assert int(w.sum().item()) == 2 * 90 * 4
    # the finite micro-batch agrees with the oracle
    oidx, _, ow = _oracle(x[:1], 4, True, 4)
    assert np.array_equal(idx[:1].cpu().numpy(), oidx)
    assert np.array_equal(w[:1].cpu().numpy(), ow)


def test_no_alloc_rejects_sizes_beyond_its_capacity(lib):
    import cross_layer_expert_b200 as eb
    P = ctypes.c_void_p(256)
    # 64 micro-batches x 8192 tokens (128 chunks) x 256 experts = 2^21 counts > 2^20
    assert lib.eb_route_loads_static(P, 64, 8192, 256, 8, 1, 8, P, P, P, None, None) == eb.EB_ERR_TOO_LARGE
    assert lib.eb_route_loads_static(P, 2, 64, 16, 20, 1, 4, P, P, P, None, None) == eb.EB_ERR_INVALID_ARG
