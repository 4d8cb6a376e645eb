"""Python binding of the B200 cross-layer MoE step library (``libeb.so``).

Argument marshalling only: every stage of the step runs in the CUDA kernels
behind the C ABI declared in ``include/eb.h``.  PyTorch provides device
memory and the current CUDA stream.  There is no CPU path: if the library is
missing, loading it raises.

Entry points carry the C names: ``eb_route``, ``eb_loads``, ``eb_schedule``,
``eb_moe_step``, ``eb_episode``, ``eb_utilization``, ``eb_trace``,
``eb_sync_status``; ``Context`` bundles a context handle with its workspace.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "_lib", "libeb.so")

EB_OK = 0
EB_ERR_INVALID_ARG = -1
EB_ERR_UNSUPPORTED = -2
EB_ERR_NONFINITE = -3
EB_ERR_CUDA = -4
EB_ERR_TIMEOUT = -5
EB_ERR_WORKSPACE = -6
EB_ERR_TOO_LARGE = -7

CUMUTIL, MAXUTIL, LOCKSTEP, DIFFPEAK = 0, 1, 2, 3
DTYPE_F32, DTYPE_BF16 = 0, 1
GEMM_AUTO, GEMM_TC, GEMM_SIMT, GEMM_TM, GEMM_TMG, GEMM_TMC = 0, 1, 2, 4, 6, 7

EXPORTED = ["eb_status_string", "eb_config_check", "eb_workspace_size", "eb_create", "eb_destroy",
            "eb_reset", "eb_moe_step", "eb_episode", "eb_utilization", "eb_trace",
            "eb_sync_status", "eb_route", "eb_loads", "eb_schedule", "eb_profile",
            "eb_profile_read", "eb_launch_count", "eb_route_loads_static",
            "eb_selftest_timeout", "eb_set_expert_map", "eb_loads_mapped", "eb_set_router",
            "eb_router", "eb_engines", "eb_inject_status", "eb_expert_ffn"]

PROF_KERNELS = ("route", "schedule", "permute", "gemm_gateup", "gemm_down", "combine",
                "positions", "router")


class EbError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {_status_string(status)} ({status})")
        self.status = status


class eb_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in
                ("L", "E", "k", "H", "F", "D", "M", "T", "n_shared", "renorm", "dtype", "policy",
                 "m", "residual", "compute", "gemm")]


_lib = None


def load() -> ctypes.CDLL:
    """Loads ``libeb.so``; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"CUDA library not built: {LIB_PATH} is missing "
                           "(run `python -m cross_layer_expert_b200.build`)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, U32, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint32, ctypes.c_size_t
    cfgp = ctypes.POINTER(eb_config)
    sig = {
        "eb_status_string": (ctypes.c_char_p, [I]),
        "eb_config_check": (I, [cfgp]),
        "eb_workspace_size": (I, [cfgp, ctypes.POINTER(SZ)]),
        "eb_create": (I, [cfgp, ctypes.POINTER(P)]),
        "eb_destroy": (I, [P]),
        "eb_reset": (I, [P, P]),
        "eb_moe_step": (I, [P, P, P, P, P, P, SZ, P, ctypes.POINTER(U32)]),
        "eb_episode": (I, [P, P, P, P, P, P, SZ, P, ctypes.POINTER(I)]),
        "eb_utilization": (I, [P] + [ctypes.POINTER(ctypes.c_int64)] * 3),
        "eb_trace": (I, [P, P, P, I, ctypes.POINTER(I)]),
        "eb_sync_status": (I, [P]),
        "eb_route": (I, [P, I, I, I, I, P, P, P, P, P]),
        "eb_loads": (I, [P, I, I, I, P, P]),
        "eb_loads_mapped": (I, [P, I, I, I, P, P, P, P]),
        "eb_set_expert_map": (I, [P, P]),
        "eb_set_router": (I, [P, P, P]),
        "eb_router": (I, [P, I, I, P, I, P, P, P]),
        "eb_schedule": (I, [P, U32, I, I, I, I, P, P, P]),
        "eb_profile": (I, [P, I]),
        "eb_profile_read": (I, [P, P, P]),
        "eb_launch_count": (I, [P, ctypes.POINTER(ctypes.c_int64)]),
        "eb_engines": (I, [P, ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]),
        "eb_route_loads_static": (I, [P, I, I, I, I, I, I, P, P, P, P, P]),
        "eb_selftest_timeout": (I, [ctypes.c_int64, P, P]),
        "eb_inject_status": (I, [P, I, P]),
        "eb_expert_ffn": (I, [P, P, I, P, P, P, I, P, P, P, P, SZ, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _status_string(s: int) -> str:
    try:
        return load().eb_status_string(s).decode()
    except Exception:  # pragma: no cover - only while reporting an error
        return "status"


def _check(status: int, what: str) -> None:
    if status != EB_OK:
        raise EbError(status, what)


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def make_config(L, E, k, H, F, D, M, T, n_shared=0, renorm=1, dtype=DTYPE_BF16, policy=CUMUTIL,
                m=None, residual=1, compute=1, gemm=GEMM_AUTO) -> eb_config:
    if m is None:
        m = max(1, int(round(0.75 * M)))
    return eb_config(L, E, k, H, F, D, M, T, n_shared, int(renorm), dtype, policy, m,
                     int(residual), int(compute), gemm)


def eb_config_check(cfg: eb_config) -> int:
    return load().eb_config_check(ctypes.byref(cfg))


def eb_workspace_size(cfg: eb_config) -> int:
    n = ctypes.c_size_t(0)
    _check(load().eb_workspace_size(ctypes.byref(cfg), ctypes.byref(n)), "eb_workspace_size")
    return n.value


def eb_route(logits, k: int, renorm: bool, idx, gate, hist, status=None, stream=None) -> None:
    """logits [n, E] f32 -> idx [n, k] i32, gate [n, k] f32, hist [E] i32."""
    n, E = logits.shape
    _check(load().eb_route(_ptr(logits), n, E, k, int(renorm), _ptr(idx), _ptr(gate), _ptr(hist),
                           _ptr(status), _stream(stream)), "eb_route")


def eb_loads(hist, D: int, w, stream=None) -> None:
    """hist [M, E] i32 -> w [M, D] i32 (contiguous expert-to-rank map)."""
    M, E = hist.shape
    _check(load().eb_loads(_ptr(hist), M, E, D, _ptr(w), _stream(stream)), "eb_loads")


def eb_loads_mapped(hist, D: int, expert_rank, w, status=None, stream=None) -> None:
    """hist [M, E] i32 -> w [M, D] i32 under the placement expert_rank
    (device [E] i32); status: optional device i32 set on an out-of-range rank."""
    M, E = hist.shape
    _check(load().eb_loads_mapped(_ptr(hist), M, E, D, _ptr(expert_rank), _ptr(w),
                                  _ptr(status) if status is not None else None, _stream(stream)),
           "eb_loads_mapped")


def eb_router(hidden, w_router, scores, status=None, stream=None) -> None:
    """hidden [n, H] bf16 x w_router [E, H] bf16 -> scores [n, E] f32."""
    n, H = hidden.shape
    E = w_router.shape[0]
    _check(load().eb_router(_ptr(hidden), n, H, _ptr(w_router), E, _ptr(scores), _ptr(status),
                            _stream(stream)), "eb_router")


def eb_schedule(w, pending_mask: int, m: int, policy: int, runset, stats=None, stream=None) -> None:
    """w [M, D] i32 -> runset (1-element u32/i32 device tensor), stats [3] i64."""
    M, D = w.shape
    _check(load().eb_schedule(_ptr(w), pending_mask, M, D, m, policy, _ptr(runset), _ptr(stats),
                              _stream(stream)), "eb_schedule")


def eb_route_loads_static(logits, k: int, renorm: bool, D: int, idx, gate, w, status=None,
                          stream=None) -> None:
    """No-allocation routing + loads: logits [n_mb, T, E] f32 -> idx [n_mb, T, k] i32,
    gate [n_mb, T, k] f32, w [n_mb, D] i32.  For callers that cannot allocate
    device memory; the library's fixed 4 MiB device array holds the counts."""
    n_mb, T, E = logits.shape
    _check(load().eb_route_loads_static(_ptr(logits), n_mb, T, E, k, int(renorm), D, _ptr(idx),
                                        _ptr(gate), _ptr(w), _ptr(status), _stream(stream)),
           "eb_route_loads_static")


def eb_selftest_timeout(limit_ns: int, status, stream=None) -> None:
    """Runs the GEMMs' bounded device wait on a barrier nothing arrives on;
    `status` (1-element int32 device tensor) receives EB_ERR_TIMEOUT."""
    _check(load().eb_selftest_timeout(int(limit_ns), _ptr(status), _stream(stream)),
           "eb_selftest_timeout")


class Context:
    """A library context plus the workspace its steps use."""

    def __init__(self, cfg: eb_config, device=None):
        import torch
        self.cfg = cfg
        lib = load()
        if device is not None:
            torch.cuda.set_device(device)
        self.device = torch.device("cuda", torch.cuda.current_device())
        self.ws_bytes = eb_workspace_size(cfg)
        self.workspace = torch.empty(max(self.ws_bytes, 256), dtype=torch.uint8, device=self.device)
        h = ctypes.c_void_p()
        _check(lib.eb_create(ctypes.byref(cfg), ctypes.byref(h)), "eb_create")
        self.handle = h

    def close(self) -> None:
        if getattr(self, "handle", None) is not None and self.handle.value:
            load().eb_destroy(self.handle)
            self.handle = None

    def __del__(self):  # pragma: no cover
        try:
            self.close()
        except Exception:
            pass

    def eb_reset(self, stream=None) -> None:
        _check(load().eb_reset(self.handle, _stream(stream)), "eb_reset")

    def eb_set_router(self, w_router=None, scores=None) -> None:
        """Router weights [L, E, H] bf16 on the device (kept alive by the
        caller): steps then project their routing scores from the hidden
        states, into `scores` [M, L, T, E] f32 if given.  None returns to
        caller-given logits."""
        self._router = (w_router, scores)
        _check(load().eb_set_router(self.handle, _ptr(w_router), _ptr(scores)), "eb_set_router")

    def eb_set_expert_map(self, expert_rank=None) -> None:
        """Placement of the E experts on the D ranks (a sequence of ints), or
        None for the contiguous map."""
        if expert_rank is None:
            _check(load().eb_set_expert_map(self.handle, None), "eb_set_expert_map")
            return
        arr = (ctypes.c_int32 * len(expert_rank))(*[int(r) for r in expert_rank])
        _check(load().eb_set_expert_map(self.handle, ctypes.cast(arr, ctypes.c_void_p)),
               "eb_set_expert_map")

    def eb_moe_step(self, logits, hidden, w_gateup, w_down, stream=None, want_runset=False):
        out = ctypes.c_uint32(0)
        _check(load().eb_moe_step(self.handle, _ptr(logits), _ptr(hidden), _ptr(w_gateup),
                                  _ptr(w_down), _ptr(self.workspace), self.ws_bytes,
                                  _stream(stream), ctypes.byref(out) if want_runset else None),
               "eb_moe_step")
        return out.value if want_runset else None

    def eb_episode(self, logits, hidden, w_gateup, w_down, stream=None) -> int:
        n = ctypes.c_int(0)
        _check(load().eb_episode(self.handle, _ptr(logits), _ptr(hidden), _ptr(w_gateup),
                                 _ptr(w_down), _ptr(self.workspace), self.ws_bytes,
                                 _stream(stream), ctypes.byref(n)), "eb_episode")
        return n.value

    def eb_expert_ffn(self, rows, seg_off, seg_layer, seg_expert, out, w_gateup, w_down,
                      stream=None) -> None:
        """Expert FFN of grouped rows: rows [R, H] (device, cfg dtype), segment
        i = rows [seg_off[i], seg_off[i+1]) for expert seg_expert[i] of layer
        seg_layer[i] (host int sequences); out [R, H] receives every row's
        expert output in the same order.  Synchronous."""
        nseg = len(seg_layer)
        off = (ctypes.c_int32 * (nseg + 1))(*[int(v) for v in seg_off])
        lay = (ctypes.c_int32 * max(nseg, 1))(*[int(v) for v in seg_layer])
        exp = (ctypes.c_int32 * max(nseg, 1))(*[int(v) for v in seg_expert])
        R = int(rows.shape[0])
        _check(load().eb_expert_ffn(self.handle, _ptr(rows), R, ctypes.cast(off, ctypes.c_void_p),
                                    ctypes.cast(lay, ctypes.c_void_p),
                                    ctypes.cast(exp, ctypes.c_void_p), nseg, _ptr(out),
                                    _ptr(w_gateup), _ptr(w_down), _ptr(self.workspace),
                                    self.ws_bytes, _stream(stream)), "eb_expert_ffn")

    def eb_utilization(self):
        a, b, c = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
        _check(load().eb_utilization(self.handle, ctypes.byref(a), ctypes.byref(b),
                                     ctypes.byref(c)), "eb_utilization")
        return a.value, b.value, c.value

    def eb_trace(self, max_steps: Optional[int] = None):
        import numpy as np
        max_steps = self.cfg.M * self.cfg.L if max_steps is None else max_steps
        rows = np.zeros((max_steps, 6), dtype=np.int64)
        layers = np.zeros((max_steps, self.cfg.M), dtype=np.int32)
        n = ctypes.c_int(0)
        _check(load().eb_trace(self.handle, rows.ctypes.data, layers.ctypes.data, max_steps,
                               ctypes.byref(n)), "eb_trace")
        k = min(n.value, max_steps)
        return rows[:k], layers[:k]

    def eb_sync_status(self) -> int:
        return load().eb_sync_status(self.handle)

    def eb_inject_status(self, status: int, stream=None) -> None:
        """Test hook: records `status` in the context's device status word
        (EB_ERR_TIMEOUT also dirties the fused combine's arrival counters)."""
        _check(load().eb_inject_status(self.handle, int(status), _stream(stream)),
               "eb_inject_status")

    def eb_profile(self, enable: bool) -> None:
        _check(load().eb_profile(self.handle, int(enable)), "eb_profile")

    def eb_profile_read(self):
        """{kernel: (milliseconds, launches)} since eb_profile(True)."""
        import numpy as np
        ms = np.zeros(len(PROF_KERNELS), dtype=np.float64)
        n = np.zeros(len(PROF_KERNELS), dtype=np.int64)
        _check(load().eb_profile_read(self.handle, ms.ctypes.data, n.ctypes.data), "eb_profile_read")
        return {k: (float(ms[i]), int(n[i])) for i, k in enumerate(PROF_KERNELS)}

    def eb_launch_count(self) -> int:
        n = ctypes.c_int64(0)
        _check(load().eb_launch_count(self.handle, ctypes.byref(n)), "eb_launch_count")
        return n.value

    def eb_engines(self):
        """(GEMM 1 engine, GEMM 2 engine) as GEMM_* values, after AUTO and the
        shape fallbacks are resolved."""
        g1, g2 = ctypes.c_int(0), ctypes.c_int(0)
        _check(load().eb_engines(self.handle, ctypes.byref(g1), ctypes.byref(g2)), "eb_engines")
        return g1.value, g2.value
