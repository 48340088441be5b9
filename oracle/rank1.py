"""ctypes wrapper of the plain-C float64 rank-1 recursion (O3, ``rank1.c``).

Test infrastructure only (test-suite, smoke check, benchmark CPU-baseline leg).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rank1.c")
_SO = os.path.join(_HERE, "_rank1.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile rank1.c with gcc into oracle/_rank1.so (plain -O2, no fast-math)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared",
                               "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _SO)
    return _SO


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.oracle_dR_rank1.restype = ctypes.c_int
        lib.oracle_dR_rank1.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
            ctypes.c_double, ctypes.c_void_p, ctypes.c_int]
        _lib = lib
    return _lib


def dR_rank1(H: np.ndarray, offsets: np.ndarray, eps2: float,
             nthreads: int | None = None) -> np.ndarray:
    """dR for all positions of all rows (float64), rows packed by ``offsets``."""
    H = np.ascontiguousarray(H, dtype=np.float32)
    offsets = np.ascontiguousarray(offsets, dtype=np.int64)
    N, d = H.shape
    if offsets[-1] != N:
        raise ValueError("offsets[-1] must equal the number of positions")
    out = np.empty(N, dtype=np.float64)
    nt = nthreads or os.cpu_count() or 1
    rc = _load().oracle_dR_rank1(H.ctypes.data, offsets.ctypes.data,
                                 offsets.shape[0] - 1, d, float(d) / eps2,
                                 out.ctypes.data, int(nt))
    if rc != 0:
        raise RuntimeError(f"oracle_dR_rank1 failed ({rc})")
    return out
