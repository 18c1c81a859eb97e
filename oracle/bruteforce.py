"""ctypes loader for the plain C brute force (bruteforce.c). Test infrastructure only."""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bruteforce.c")
_LIB = os.path.join(_HERE, "_bruteforce.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile bruteforce.c with gcc into oracle/_bruteforce.so (no optimisation tricks)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-shared", "-fPIC", _SRC, "-o", _LIB, "-lm"])
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        p = ctypes.POINTER(ctypes.c_double)
        lib.oracle_bruteforce.argtypes = [p, p, p, p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_int, ctypes.c_double]
        lib.oracle_bruteforce.restype = None
        lib.oracle_bruteforce_rope.argtypes = [p, p, p, p, p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                               ctypes.c_int, ctypes.c_int, ctypes.c_double]
        lib.oracle_bruteforce_rope.restype = None
        _lib = lib
    return _lib


def bruteforce_c(q, k, v, block_len: int, eps: float) -> np.ndarray:
    """Explicit masked N x N evaluation in C. q, k [B,H,N,D]; v [B,H,N,E]; returns o [B,H,N,E]."""
    q = np.ascontiguousarray(q, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    B, H, N, D = q.shape
    E = v.shape[-1]
    o = np.zeros((B, H, N, E), dtype=np.float64)
    p = ctypes.POINTER(ctypes.c_double)
    _load().oracle_bruteforce(q.ctypes.data_as(p), k.ctypes.data_as(p), v.ctypes.data_as(p),
                              o.ctypes.data_as(p), B * H, N, D, E, int(block_len), float(eps))
    return o


def bruteforce_rope_c(q, k, v, block_len: int, eps: float, angles) -> np.ndarray:
    """The rotary form's explicit masked N x N evaluation in C, through relative angles.
    q, k [B,H,N,D] (D even); v [B,H,N,E]; angles [N, D/2]; returns o [B,H,N,E]."""
    q = np.ascontiguousarray(q, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    ang = np.ascontiguousarray(angles, dtype=np.float64)
    B, H, N, D = q.shape
    E = v.shape[-1]
    assert D % 2 == 0 and ang.shape == (N, D // 2)
    o = np.zeros((B, H, N, E), dtype=np.float64)
    p = ctypes.POINTER(ctypes.c_double)
    _load().oracle_bruteforce_rope(q.ctypes.data_as(p), k.ctypes.data_as(p), v.ctypes.data_as(p),
                                   ang.ctypes.data_as(p), o.ctypes.data_as(p), B * H, N, D, E, int(block_len),
                                   float(eps))
    return o
