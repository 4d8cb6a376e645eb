"""Plain-C parts of the oracle (test infrastructure only), built with gcc.

``maxutil`` is the exhaustive MaxUtil of ``oracle/maxutil.c`` enumerated by
complements, for pending sets too large for the Python enumeration (up to 32
micro-batches); ``maxutil_plain`` is the same definition enumerated forward
over every bitmask (2^n subsets, so pending sets of up to about 24).
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
        _lib.oracle_maxutil_plain.restype = ctypes.c_uint32
        _lib.oracle_maxutil_plain.argtypes = _lib.oracle_maxutil.argtypes
    return _lib


def _call(fn_name, pending, w: dict, m: int):
    pending = sorted(pending)
    D = len(w[pending[0]])
    rows = np.ascontiguousarray(np.array([w[j] for j in pending], dtype=np.int64))
    ids = np.ascontiguousarray(np.array(pending, dtype=np.int32))
    mask = getattr(_load(), fn_name)(rows.ctypes.data, ids.ctypes.data, len(pending), D, m)
    return [j for j in range(32) if (mask >> j) & 1]


def maxutil(pending, w: dict, m: int):
    """Same contract as oracle.schedule.maxutil: sorted list of micro-batch ids
    (enumeration by complements)."""
    return _call("oracle_maxutil", pending, w, m)


def maxutil_plain(pending, w: dict, m: int):
    """The same, enumerating every bitmask forward (2^|pending| subsets)."""
    if len(pending) > 26:
        raise ValueError("the forward enumeration is for pending sets of at most 26")
    return _call("oracle_maxutil_plain", pending, w, m)
