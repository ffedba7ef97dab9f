"""Python access to the CPU oracle of the Gated DeltaNet recurrent scan.

TEST INFRASTRUCTURE ONLY: imported by the tests, the package smoke check and
the benchmark's CPU-baseline leg, never by the product path.  It shares no
code with the CUDA library (see ``gdn_oracle.c`` for what it computes and the
readings of the Lily pages it follows).
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import build as _build

_libs = {}
_P = ctypes.c_void_p
_I = ctypes.c_int64


def lib(path: str | None = None):
    path = path or _build.ensure_gdn_built()
    if path not in _libs:
        L = ctypes.CDLL(path)
        L.gdn_oracle_scan.restype = ctypes.c_int
        L.gdn_oracle_scan.argtypes = [_I] * 6 + [_P] * 5 + [ctypes.c_double, _P, _P, _P]
        _libs[path] = L
    return _libs[path]


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def scan(q, k, v, g, beta, scale, S0, L=None):
    """(o float64 [B,T,Hv,dv], S float64 [B,Hv,dv,dk]) of the scan.

    q, k: bf16 bits [B,T,Hk,dk]; v: bf16 bits [B,T,Hv,dv]; g, beta: fp32
    [B,T,Hv]; S0: fp32 [B,Hv,dv,dk]."""
    q, k, v = _c(q, np.uint16), _c(k, np.uint16), _c(v, np.uint16)
    g, beta, S0 = _c(g, np.float32), _c(beta, np.float32), _c(S0, np.float32)
    B, T, Hk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    assert k.shape == q.shape and v.shape[:2] == (B, T) and g.shape == (B, T, Hv) and beta.shape == g.shape
    assert S0.shape == (B, Hv, dv, dk)
    o = np.empty((B, T, Hv, dv), dtype=np.float64)
    S = np.empty((B, Hv, dv, dk), dtype=np.float64)
    st = (L or lib()).gdn_oracle_scan(B, T, Hk, Hv, dk, dv, q.ctypes.data, k.ctypes.data, v.ctypes.data,
                                      g.ctypes.data, beta.ctypes.data, float(scale), S0.ctypes.data,
                                      o.ctypes.data, S.ctypes.data)
    if st:
        raise RuntimeError("gdn oracle scan failed with status %d" % st)
    return o, S
