"""Plain-C parts of the oracle (test infrastructure only), built with gcc.

``maxutil`` is the exhaustive MaxUtil of ``oracle/maxutil.c``, for pending
sets too large for the Python enumeration (up to 32 micro-batches).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "maxutil.c")
LIB = os.path.join(HERE, "_native", "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        os.makedirs(os.path.dirname(LIB), exist_ok=True)
        subprocess.run(["gcc", "-O2", "-shared", "-fPIC", "-o", LIB + ".tmp", SRC], check=True)
        os.replace(LIB + ".tmp", LIB)
    return LIB


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _lib.oracle_maxutil.restype = ctypes.c_uint32
        _lib.oracle_maxutil.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                        ctypes.c_int, ctypes.c_int]
    return _lib


def maxutil(pending, w: dict, m: int):
    """Same contract as oracle.schedule.maxutil: sorted list of micro-batch ids."""
    pending = sorted(pending)
    D = len(w[pending[0]])
    rows = np.ascontiguousarray(np.array([w[j] for j in pending], dtype=np.int64))
    ids = np.ascontiguousarray(np.array(pending, dtype=np.int32))
    mask = _load().oracle_maxutil(rows.ctypes.data, ids.ctypes.data, len(pending), D, m)
    return [j for j in range(32) if (mask >> j) & 1]
