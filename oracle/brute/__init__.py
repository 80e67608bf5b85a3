"""ctypes wrapper around the C brute-force enumerator (oracle side, test infrastructure only)."""
import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "brute.c")
_LIB = os.path.join(_HERE, "_brute.so")
_lib = None


def build(force=False):
    """Compile brute.c into _brute.so beside it (gcc -O2 -shared -fPIC)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-shared", "-fPIC", "-o", _LIB, _SRC, "-lm"])
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        f = lib.nq_brute_min_sq_error
        dp = ctypes.POINTER(ctypes.c_double)
        f.argtypes = [dp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                      dp, dp, dp, dp]
        f.restype = ctypes.c_double
        _lib = lib
    return _lib


def min_sq_error(W, r, starts=16, sweeps=500):
    """Optimal squared error of diag(s1) U V^T diag(s2) over all +-1 patterns (r <= 2, size <= 8).

    Returns (err2, U, V, s1, s2).
    """
    W = np.ascontiguousarray(W, dtype=np.float64)
    m, n = W.shape
    U = np.zeros((m, r))
    V = np.zeros((n, r))
    s1 = np.zeros(m)
    s2 = np.zeros(n)
    dp = ctypes.POINTER(ctypes.c_double)
    e = _load().nq_brute_min_sq_error(W.ctypes.data_as(dp), m, n, r, starts, sweeps,
                                      U.ctypes.data_as(dp), V.ctypes.data_as(dp),
                                      s1.ctypes.data_as(dp), s2.ctypes.data_as(dp))
    if e < 0:
        raise ValueError("brute force supports 1 <= m, n <= 8 and r in {1, 2}")
    return e, U, V, s1, s2
