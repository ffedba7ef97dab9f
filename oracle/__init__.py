"""Python access to the CPU oracle of the MoE expert layer.

TEST INFRASTRUCTURE ONLY: imported by the tests, the package smoke check and
the benchmark's CPU-baseline leg, never by the product path.  It shares no
code with the CUDA library (see ``moe_oracle.c`` for what it computes and the
readings of the Lily pages it follows).
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import build as _build

OK, ERR_ARG, ERR_NONFINITE, ERR_BOUNDS = 0, 1, 5, 7

_libs = {}

_P = ctypes.c_void_p
_I = ctypes.c_int64


def lib(path: str | None = None):
    path = path or _build.ensure_built()
    if path not in _libs:
        L = ctypes.CDLL(path)
        L.moe_oracle_code.restype = ctypes.c_int
        L.moe_oracle_code.argtypes = [_P, _I]
        L.moe_oracle_dequant_one.restype = ctypes.c_double
        L.moe_oracle_dequant_one.argtypes = [_P, _P, _I, _I, _I, _I]
        L.moe_oracle_dequant_matrix.argtypes = [_P, _P, _I, _I, _I, _P]
        L.moe_oracle_router_logits.restype = ctypes.c_int
        L.moe_oracle_router_logits.argtypes = [_I, _P, _I, _I, _P, _P, _P, _I, _P]
        L.moe_oracle_select.restype = ctypes.c_int
        L.moe_oracle_select.argtypes = [_I, _I, _I, _P, _P, _P]
        L.moe_oracle_permute.restype = ctypes.c_int
        L.moe_oracle_permute.argtypes = [_I, _I, _I, _P, _P, _P, _P, _P]
        L.moe_oracle_expert_rows.argtypes = [_I, _I, _I, _I, _P, _P, _P, _P, _I, _P, _P, _P]
        L.moe_oracle_layer.restype = ctypes.c_int
        L.moe_oracle_layer.argtypes = [_I, _I, _I, _I, _I, _I, ctypes.c_int, _P, _P, _P, _P, _I,
                                       _P, _P, _P, _P, _I, _P, _P, _P, _P]
        _libs[path] = L
    return _libs[path]


class OracleError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__("oracle %s failed with status %d" % (what, code))
        self.code = code


def _p(a):
    if a is None:
        return None
    assert isinstance(a, np.ndarray) and a.flags.c_contiguous, type(a)
    return a.ctypes.data


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def code(row_words: np.ndarray, k: int, L=None) -> int:
    row_words = _c(row_words, np.uint32)
    return (L or lib()).moe_oracle_code(_p(row_words), k)


def dequant_one(codes, sb, K, G, n, k, L=None) -> float:
    codes, sb = _c(codes, np.uint32), _c(sb, np.uint16)
    return (L or lib()).moe_oracle_dequant_one(_p(codes), _p(sb), K, G, n, k)


def dequant_matrix(codes, sb, N, K, G, L=None) -> np.ndarray:
    codes, sb = _c(codes, np.uint32), _c(sb, np.uint16)
    W = np.empty((N, K), dtype=np.float64)
    (L or lib()).moe_oracle_dequant_matrix(_p(codes), _p(sb), N, K, G, _p(W))
    return W


def router_logits(x, w_router, bias=None, bias_stride=0, tokens=None, L=None) -> np.ndarray:
    """fp32 logits in the contract order for `tokens` (default: all rows of x)."""
    x, w_router = _c(x, np.uint16), _c(w_router, np.uint16)
    bias = _c(bias, np.float32)
    T, H = x.shape
    E = w_router.shape[0]
    tok = None if tokens is None else _c(tokens, np.int32)
    n = T if tok is None else len(tok)
    out = np.empty((n, E), dtype=np.float32)
    st = (L or lib()).moe_oracle_router_logits(n, _p(tok), H, E, _p(x), _p(w_router), _p(bias),
                                               bias_stride, _p(out))
    if st:
        raise OracleError(st, "router_logits")
    return out


def select(logits, k, L=None):
    """(idx int32 [n, k], w float64 [n, k]) for logits [n, E]."""
    logits = _c(logits, np.float32)
    n, E = logits.shape
    idx = np.empty((n, k), dtype=np.int32)
    w = np.empty((n, k), dtype=np.float64)
    st = (L or lib()).moe_oracle_select(n, E, k, _p(logits), _p(idx), _p(w))
    if st:
        raise OracleError(st, "select")
    return idx, w


def permute(idx, E, L=None):
    """(counts [E], offsets [E+1], row_to_pair [T*k], pair_to_row [T*k])."""
    idx = _c(idx, np.int32)
    T, k = idx.shape
    counts = np.empty(E, dtype=np.int32)
    offsets = np.empty(E + 1, dtype=np.int32)
    r2p = np.empty(T * k, dtype=np.int32)
    p2r = np.empty(T * k, dtype=np.int32)
    st = (L or lib()).moe_oracle_permute(T, E, k, _p(idx), _p(counts), _p(offsets), _p(r2p), _p(p2r))
    if st:
        raise OracleError(st, "permute")
    return counts, offsets, r2p, p2r


def expert_rows(layer, e, x_rows, with_h=False, L=None):
    """Expert e (E = shared) applied to bf16 rows: y [n, H] (and h [n, I])."""
    gu_codes, gu_sb = layer["gu_codes"], layer["gu_sb"]
    d_codes, d_sb = layer["d_codes"], layer["d_sb"]
    H = gu_codes.shape[2] * 8
    I = d_codes.shape[2] * 8
    G = H // gu_sb.shape[2]
    x_rows = _c(x_rows, np.uint16)
    n = x_rows.shape[0]
    y = np.empty((n, H), dtype=np.float64)
    h = np.empty((n, I), dtype=np.float64) if with_h else None
    (L or lib()).moe_oracle_expert_rows(H, I, G, e, _p(gu_codes), _p(gu_sb), _p(d_codes), _p(d_sb),
                                        n, _p(x_rows), _p(h), _p(y))
    return (y, h) if with_h else y


def layer(layer, tokens=None, k=8, has_shared=True, logits_in=None, L=None):
    """Layer output y float64 [n, H] for `tokens` (default all), with idx and w."""
    x = _c(layer["x"], np.uint16)
    T, H = x.shape
    wr = _c(layer["w_router"], np.uint16)
    E = wr.shape[0]
    I = layer["d_codes"].shape[2] * 8
    G = H // layer["gu_sb"].shape[2]
    tok = np.arange(T, dtype=np.int32) if tokens is None else _c(tokens, np.int32)
    n = len(tok)
    bias = _c(layer.get("logit_bias"), np.float32)
    stride = int(layer.get("bias_stride", 0))
    li = _c(logits_in, np.float32)
    y = np.empty((n, H), dtype=np.float64)
    idx = np.empty((n, k), dtype=np.int32)
    w = np.empty((n, k), dtype=np.float64)
    st = (L or lib()).moe_oracle_layer(T, H, I, E, k, G, 1 if has_shared else 0, _p(x), _p(wr), _p(li),
                                       _p(bias), stride, _p(layer["gu_codes"]), _p(layer["gu_sb"]),
                                       _p(layer["d_codes"]), _p(layer["d_sb"]), n, _p(tok), _p(y),
                                       _p(idx), _p(w))
    if st:
        raise OracleError(st, "layer")
    return y, idx, w
