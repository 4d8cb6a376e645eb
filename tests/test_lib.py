"""Host-side checks of the C ABI: the library loads, exports every entry point
that include/eb.h declares, and rejects bad arguments before touching a GPU.
"""
import ctypes
import os
import re

import pytest

import cross_layer_expert_b200 as eb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "eb.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(eb_[a-z_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from cross_layer_expert_b200 import build
    build.build()
    return eb.load()


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert len(names) >= 14
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(eb.EXPORTED) == names


def test_status_strings(lib):
    for s in (0, -1, -2, -3, -4, -5, -6):
        assert lib.eb_status_string(s)
    assert lib.eb_status_string(0) == b"ok"


def _cfg(**kw):
    base = dict(L=4, E=16, k=2, H=128, F=256, D=4, M=4, T=64, n_shared=0, renorm=1,
                dtype=eb.DTYPE_F32, policy=eb.CUMUTIL, m=3, residual=1, compute=1, gemm=0)
    base.update(kw)
    return eb.make_config(**base)


def test_config_check(lib):
    assert eb.eb_config_check(_cfg()) == eb.EB_OK
    bad = [dict(E=15), dict(k=17), dict(m=5), dict(m=0), dict(T=0), dict(L=0), dict(M=0),
           dict(policy=7), dict(dtype=5), dict(D=0), dict(n_shared=-1), dict(gemm=8), dict(gemm=-1),
           dict(gemm=3), dict(gemm=5)]  # 3 and 5: retired two-SM engines
    for b in bad:
        assert eb.eb_config_check(_cfg(**b)) == eb.EB_ERR_INVALID_ARG, b
    unsup = [dict(M=33, m=3), dict(D=64, E=128 * 3), dict(k=20, n_shared=13, E=64),
             dict(H=130), dict(gemm=eb.GEMM_TC), dict(dtype=eb.DTYPE_BF16, gemm=eb.GEMM_TC, H=192),
             dict(gemm=eb.GEMM_TM), dict(dtype=eb.DTYPE_BF16, gemm=eb.GEMM_TM, F=192),
             dict(gemm=eb.GEMM_TMC), dict(dtype=eb.DTYPE_BF16, gemm=eb.GEMM_TMC, H=192),
             dict(M=32, m=8, policy=eb.MAXUTIL)]
    for u in unsup:
        assert eb.eb_config_check(_cfg(**u)) == eb.EB_ERR_UNSUPPORTED, u
    assert eb.eb_config_check(_cfg(dtype=eb.DTYPE_BF16, gemm=eb.GEMM_TM)) == eb.EB_OK
    # H = 384 is not a multiple of 256: TMC's GEMM 2 then runs weight-major
    assert eb.eb_config_check(_cfg(dtype=eb.DTYPE_BF16, gemm=eb.GEMM_TMC, H=384)) == eb.EB_OK
    # routing-only configs need no hidden / FFN sizes
    assert eb.eb_config_check(_cfg(compute=0, H=0, F=0)) == eb.EB_OK
    # MaxUtil at M = 32 with m = 24 enumerates ~15M complements: supported
    assert eb.eb_config_check(_cfg(M=32, m=24, policy=eb.MAXUTIL, compute=0)) == eb.EB_OK


def test_workspace_size_grows_with_shape(lib):
    a = eb.eb_workspace_size(_cfg())
    b = eb.eb_workspace_size(_cfg(T=128))
    c = eb.eb_workspace_size(_cfg(compute=0))
    assert 0 < c < a < b
    with pytest.raises(eb.EbError):
        eb.eb_workspace_size(_cfg(E=15))


def test_stage_argument_errors_return_before_launch(lib):
    P = ctypes.c_void_p(16)
    # k > E, E % D != 0, m > M, M > 32: all rejected on the host
    assert lib.eb_route(P, 4, 8, 9, 1, P, P, P, None, None) == eb.EB_ERR_INVALID_ARG
    assert lib.eb_route(P, 4, 300, 2, 1, P, P, P, None, None) == eb.EB_ERR_UNSUPPORTED
    assert lib.eb_route(None, 4, 8, 2, 1, P, P, P, None, None) == eb.EB_ERR_INVALID_ARG
    assert lib.eb_loads(P, 4, 10, 3, P, None) == eb.EB_ERR_INVALID_ARG
    assert lib.eb_schedule(P, 0xF, 4, 2, 5, 0, P, None, None) == eb.EB_ERR_INVALID_ARG
    assert lib.eb_schedule(P, 0xF, 33, 2, 5, 0, P, None, None) == eb.EB_ERR_UNSUPPORTED
    assert lib.eb_schedule(P, 0x1F, 4, 2, 2, 0, P, None, None) == eb.EB_ERR_INVALID_ARG
    assert lib.eb_schedule(P, 0xF, 4, 2, 2, 9, P, None, None) == eb.EB_ERR_INVALID_ARG
    assert lib.eb_schedule(None, 0xF, 4, 2, 2, 0, P, None, None) == eb.EB_ERR_INVALID_ARG
    assert lib.eb_destroy(None) == eb.EB_ERR_INVALID_ARG
    g1, g2 = ctypes.c_int(-1), ctypes.c_int(-1)
    assert lib.eb_engines(None, ctypes.byref(g1), ctypes.byref(g2)) == eb.EB_ERR_INVALID_ARG
    assert lib.eb_reset(None, None) == eb.EB_ERR_INVALID_ARG
    # placement: a map is required; E need not be a multiple of D
    assert lib.eb_loads_mapped(P, 4, 10, 3, None, P, None, None) == eb.EB_ERR_INVALID_ARG
    assert lib.eb_loads_mapped(None, 4, 10, 3, P, P, None, None) == eb.EB_ERR_INVALID_ARG
    assert lib.eb_loads_mapped(P, 0, 10, 3, P, P, None, None) == eb.EB_OK  # nothing to do
    assert lib.eb_set_expert_map(None, None) == eb.EB_ERR_INVALID_ARG
    # router projection: E a multiple of 16 (<= 256), H a multiple of 64,
    # 16-byte aligned pointers; n = 0 is a no-op
    assert lib.eb_router(P, 8, 2048, P, 12, P, None, None) == eb.EB_ERR_UNSUPPORTED
    assert lib.eb_router(P, 8, 2048, P, 512, P, None, None) == eb.EB_ERR_UNSUPPORTED
    assert lib.eb_router(P, 8, 100, P, 128, P, None, None) == eb.EB_ERR_UNSUPPORTED
    assert lib.eb_router(ctypes.c_void_p(8), 8, 2048, P, 128, P, None, None) == eb.EB_ERR_INVALID_ARG
    assert lib.eb_router(None, 8, 2048, P, 128, P, None, None) == eb.EB_ERR_INVALID_ARG
    assert lib.eb_router(None, 0, 2048, None, 128, None, None, None) == eb.EB_OK
    assert lib.eb_set_router(None, P, None) == eb.EB_ERR_INVALID_ARG
