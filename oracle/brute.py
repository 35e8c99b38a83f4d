"""ctypes wrapper around the long-double triple-loop attention (``brute_attention.c``).

TEST INFRASTRUCTURE ONLY.  ``build()`` compiles the C file with gcc into
``oracle/_brute_attention.so`` (git-ignored); ``brute_attention`` calls it per (b, h).
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "brute_attention.c")
_LIB = os.path.join(_HERE, "_brute_attention.so")
_handle: Optional[ctypes.CDLL] = None


def build(force: bool = False) -> str:
    """Compile the brute-force C oracle (gcc, -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _lib() -> ctypes.CDLL:
    global _handle
    if _handle is None:
        _handle = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        _handle.brute_attention.argtypes = [dp, dp, dp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_double, ctypes.c_int, ctypes.c_int, dp, dp]
        _handle.brute_attention.restype = None
    return _handle


def brute_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float,
                    k0: int = 0, k1: Optional[int] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Same contract as ``oracle.attention`` (no row subset), tiny shapes only (D <= 1024)."""
    B, H, S_q, D = q.shape
    S_kv = k.shape[2]
    if k1 is None:
        k1 = S_kv
    if D > 1024:
        raise ValueError("brute force supports D <= 1024")
    lib = _lib()
    dp = ctypes.POINTER(ctypes.c_double)
    out = np.zeros((B, H, S_q, D), dtype=np.float64)
    lse = np.zeros((B, H, S_q), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            qq = np.ascontiguousarray(q[b, h], dtype=np.float64)
            kk = np.ascontiguousarray(k[b, h], dtype=np.float64)
            vv = np.ascontiguousarray(v[b, h], dtype=np.float64)
            oo = np.zeros((S_q, D), dtype=np.float64)
            ll = np.zeros((S_q,), dtype=np.float64)
            lib.brute_attention(qq.ctypes.data_as(dp), kk.ctypes.data_as(dp), vv.ctypes.data_as(dp),
                                S_q, S_kv, D, float(scale), int(k0), int(k1),
                                oo.ctypes.data_as(dp), ll.ctypes.data_as(dp))
            out[b, h], lse[b, h] = oo, ll
    return out, lse
