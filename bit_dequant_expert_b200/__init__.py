"""Python binding of libmoe_b200 (one MoE expert layer with groupwise-affine
4-bit weights on B200).

Argument marshalling only: every step of the layer runs in the CUDA library.
The functions carry the C ABI's names (``include/moe_b200.h``); tensors are
passed as torch tensors (their ``data_ptr()``), raw integer addresses or
None (NULL).  ``stream`` defaults to torch's current CUDA stream.

Importing fails loudly when the library has not been built; there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError("libmoe_b200.so is missing; build it with `python bit_dequant_expert_b200/build.py` "
                      "(there is no fallback implementation)")

_lib = ctypes.CDLL(LIB_PATH)

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_WORKSPACE = 3
MOE_ERR_CUDA = 4
MOE_ERR_NONFINITE = 5
MOE_ERR_TIMEOUT = 6
MOE_ERR_BOUNDS = 7

MOE_MODE_SCATTER = 0
MOE_MODE_PAIRS = 1

MOE_PATH_AUTO = 0
MOE_PATH_SIMT = 1
MOE_PATH_GEMV = 2
MOE_PATH_TC = 3
MOE_PATH_TC_GEMV = 4

EXPORTED = (
    "moe_workspace_size", "moe_workspace_init", "moe_route", "moe_permute", "moe_expert_ffn",
    "moe_expert_ffn_path", "moe_combine", "moe_get_device_error", "moe_status_string", "moe_launch_count",
    "moe_permute_static", "moe_decode_layer", "moe_wait_selftest", "moe_gather_rows", "gdn_scan",
    "moe_router_logits",
)

MOE_STATIC_MAX_TOKENS = 16384


class moe_config_t(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("inter", ctypes.c_int32), ("num_experts", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("group_size", ctypes.c_int32), ("has_shared", ctypes.c_int32)]


def config(hidden=2048, inter=512, num_experts=256, top_k=8, group_size=64, has_shared=1) -> moe_config_t:
    return moe_config_t(hidden, inter, num_experts, top_k, group_size, has_shared)


_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_CFG = ctypes.POINTER(moe_config_t)

_lib.moe_workspace_size.restype = ctypes.c_size_t
_lib.moe_workspace_size.argtypes = [_CFG, _I32]
_lib.moe_workspace_init.restype = _I32
_lib.moe_workspace_init.argtypes = [_P, ctypes.c_size_t, _P]
_lib.moe_route.restype = _I32
_lib.moe_route.argtypes = [_CFG, _I32, _P, _P, _P, _P, ctypes.c_int64, _P, _P, _P, _P, ctypes.c_size_t, _P]
_lib.moe_router_logits.restype = _I32
_lib.moe_router_logits.argtypes = [_CFG, _I32, _P, _P, _P, ctypes.c_int64, _P, _P, ctypes.c_size_t, _P]
_lib.moe_permute.restype = _I32
_lib.moe_permute.argtypes = [_CFG, _I32, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
_lib.moe_expert_ffn.restype = _I32
_lib.moe_expert_ffn.argtypes = [_CFG, _I32, _P, _P, _P, _P, _P, _P, _P, _P, _I32, _P, _P, _P, ctypes.c_size_t, _P]
_lib.moe_expert_ffn_path.restype = _I32
_lib.moe_expert_ffn_path.argtypes = [_CFG, _I32, _P, _P, _P, _P, _P, _P, _P, _P, _I32, _P, _P, _P,
                                     ctypes.c_size_t, _I32, _P]
_lib.moe_combine.restype = _I32
_lib.moe_combine.argtypes = [_CFG, _I32, _I32, _P, _P, _P, _P, _P, _P]
_lib.gdn_scan.restype = _I32
_lib.gdn_scan.argtypes = [_I32] * 6 + [_P] * 5 + [ctypes.c_float, _P, _P, _P, _P]
_lib.moe_gather_rows.restype = _I32
_lib.moe_gather_rows.argtypes = [_CFG, _I32, _P, _P, _P, _I32, _I32, _P, _P, _P, ctypes.c_size_t, _P]
_lib.moe_get_device_error.restype = _I32
_lib.moe_get_device_error.argtypes = [_P, _P]
_lib.moe_permute_static.restype = _I32
_lib.moe_permute_static.argtypes = [_CFG, _I32, _P, _P, _P, _P, _P, _P, _P]
_lib.moe_decode_layer.restype = _I32
_lib.moe_decode_layer.argtypes = [_CFG, _I32, _P, _P, _P, ctypes.c_int64, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                  _P, _P, _P, ctypes.c_size_t, _P]
_lib.moe_launch_count.restype = _I32
_lib.moe_launch_count.argtypes = [_CFG, _I32, _I32, _I32]
_lib.moe_status_string.restype = ctypes.c_char_p
_lib.moe_status_string.argtypes = [_I32]
_lib.moe_wait_selftest.restype = _I32
_lib.moe_wait_selftest.argtypes = [_I32, _I32, _I32, ctypes.c_uint64, _P, _P]


class MoeError(RuntimeError):
    def __init__(self, status: int, call: str):
        self.status = status
        super().__init__("%s failed: %s" % (call, moe_status_string(status)))


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _nbytes(t) -> int:
    return t.numel() * t.element_size()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, call: str, raise_on_error: bool) -> int:
    if status != MOE_OK and raise_on_error:
        raise MoeError(status, call)
    return status


def moe_status_string(status: int) -> str:
    return _lib.moe_status_string(status).decode()


def moe_workspace_size(cfg: moe_config_t, max_tokens: int) -> int:
    return int(_lib.moe_workspace_size(ctypes.byref(cfg), max_tokens))


def moe_workspace_init(ws, ws_bytes: int | None = None, stream=None, raise_on_error=True) -> int:
    n = _nbytes(ws) if ws_bytes is None else ws_bytes
    return _check(_lib.moe_workspace_init(_ptr(ws), n, _stream(stream)), "moe_workspace_init", raise_on_error)


def moe_route(cfg, T, x, w_router, logits_in, logit_bias, logit_bias_row_stride, topk_idx, topk_w, counts, ws,
              ws_bytes=None, stream=None, raise_on_error=True) -> int:
    n = _nbytes(ws) if ws_bytes is None else ws_bytes
    st = _lib.moe_route(ctypes.byref(cfg), T, _ptr(x), _ptr(w_router), _ptr(logits_in), _ptr(logit_bias),
                        logit_bias_row_stride, _ptr(topk_idx), _ptr(topk_w), _ptr(counts), _ptr(ws), n,
                        _stream(stream))
    return _check(st, "moe_route", raise_on_error)


def moe_router_logits(cfg, T, x, w_router, logit_bias, logit_bias_row_stride, logits, ws, ws_bytes=None,
                      stream=None, raise_on_error=True) -> int:
    n = _nbytes(ws) if ws_bytes is None else ws_bytes
    st = _lib.moe_router_logits(ctypes.byref(cfg), T, _ptr(x), _ptr(w_router), _ptr(logit_bias),
                                logit_bias_row_stride, _ptr(logits), _ptr(ws), n, _stream(stream))
    return _check(st, "moe_router_logits", raise_on_error)


def moe_permute(cfg, T, topk_idx, counts, offsets, row_to_pair, pair_to_row, ws, ws_bytes=None, stream=None,
                raise_on_error=True) -> int:
    n = _nbytes(ws) if ws_bytes is None else ws_bytes
    st = _lib.moe_permute(ctypes.byref(cfg), T, _ptr(topk_idx), _ptr(counts), _ptr(offsets), _ptr(row_to_pair),
                          _ptr(pair_to_row), _ptr(ws), n, _stream(stream))
    return _check(st, "moe_permute", raise_on_error)


def moe_expert_ffn(cfg, T, x, gu_codes, gu_sb, d_codes, d_sb, offsets, row_to_pair, topk_w, mode, out0, out1, ws,
                   ws_bytes=None, stream=None, raise_on_error=True) -> int:
    n = _nbytes(ws) if ws_bytes is None else ws_bytes
    st = _lib.moe_expert_ffn(ctypes.byref(cfg), T, _ptr(x), _ptr(gu_codes), _ptr(gu_sb), _ptr(d_codes), _ptr(d_sb),
                             _ptr(offsets), _ptr(row_to_pair), _ptr(topk_w), mode, _ptr(out0), _ptr(out1),
                             _ptr(ws), n, _stream(stream))
    return _check(st, "moe_expert_ffn", raise_on_error)


def moe_expert_ffn_path(cfg, T, x, gu_codes, gu_sb, d_codes, d_sb, offsets, row_to_pair, topk_w, mode, out0, out1,
                        ws, path, ws_bytes=None, stream=None, raise_on_error=True) -> int:
    n = _nbytes(ws) if ws_bytes is None else ws_bytes
    st = _lib.moe_expert_ffn_path(ctypes.byref(cfg), T, _ptr(x), _ptr(gu_codes), _ptr(gu_sb), _ptr(d_codes),
                                  _ptr(d_sb), _ptr(offsets), _ptr(row_to_pair), _ptr(topk_w), mode, _ptr(out0),
                                  _ptr(out1), _ptr(ws), n, path, _stream(stream))
    return _check(st, "moe_expert_ffn_path", raise_on_error)


def moe_combine(cfg, T, mode, in0, in1, pair_to_row, topk_w, y, stream=None, raise_on_error=True) -> int:
    st = _lib.moe_combine(ctypes.byref(cfg), T, mode, _ptr(in0), _ptr(in1), _ptr(pair_to_row), _ptr(topk_w), _ptr(y),
                          _stream(stream))
    return _check(st, "moe_combine", raise_on_error)


def moe_gather_rows(cfg, T, x, row_to_pair, topk_w, row_begin, n_rows, rows_out, w_out, ws, ws_bytes=None,
                    stream=None, raise_on_error=True) -> int:
    st = _lib.moe_gather_rows(ctypes.byref(cfg), T, _ptr(x), _ptr(row_to_pair), _ptr(topk_w), row_begin, n_rows,
                              _ptr(rows_out), _ptr(w_out), _ptr(ws), _nbytes(ws) if ws_bytes is None else ws_bytes,
                              _stream(stream))
    return _check(st, "moe_gather_rows", raise_on_error)


def gdn_scan(B, T, Hk, Hv, dk, dv, q, k, v, g, beta, scale, state_in, state_out, o, stream=None,
             raise_on_error=True) -> int:
    """Gated DeltaNet recurrent scan (include/gdn_b200.h)."""
    st = _lib.gdn_scan(B, T, Hk, Hv, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale),
                       _ptr(state_in), _ptr(state_out), _ptr(o), _stream(stream))
    return _check(st, "gdn_scan", raise_on_error)


def moe_decode_layer(cfg, T, x, w_router, logit_bias, logit_bias_row_stride, gu_codes, gu_sb, d_codes, d_sb,
                     topk_idx, topk_w, counts, offsets, row_to_pair, pair_to_row, y_acc, y, ws, ws_bytes=None,
                     stream=None, raise_on_error=True) -> int:
    """The whole layer for T <= 8 tokens in two launches (router, top-k,
    permutation and expert FFNs in one kernel, then the combine)."""
    n = _nbytes(ws) if ws_bytes is None else ws_bytes
    st = _lib.moe_decode_layer(ctypes.byref(cfg), T, _ptr(x), _ptr(w_router), _ptr(logit_bias),
                               logit_bias_row_stride, _ptr(gu_codes), _ptr(gu_sb), _ptr(d_codes), _ptr(d_sb),
                               _ptr(topk_idx), _ptr(topk_w), _ptr(counts), _ptr(offsets), _ptr(row_to_pair),
                               _ptr(pair_to_row), _ptr(y_acc), _ptr(y), _ptr(ws), n, _stream(stream))
    return _check(st, "moe_decode_layer", raise_on_error)


def moe_permute_static(cfg, T, topk_idx, counts, offsets, row_to_pair, pair_to_row, err_out=None, stream=None,
                       raise_on_error=True) -> int:
    """moe_permute without a workspace, for callers that cannot allocate
    device memory (scratch lives in a fixed array inside the library)."""
    st = _lib.moe_permute_static(ctypes.byref(cfg), T, _ptr(topk_idx), _ptr(counts), _ptr(offsets),
                                 _ptr(row_to_pair), _ptr(pair_to_row), _ptr(err_out), _stream(stream))
    return _check(st, "moe_permute_static", raise_on_error)


def moe_launch_count(cfg, T, mode=MOE_MODE_SCATTER, path=MOE_PATH_AUTO) -> int:
    return int(_lib.moe_launch_count(ctypes.byref(cfg), T, mode, path))


def moe_get_device_error(ws, stream=None) -> int:
    return int(_lib.moe_get_device_error(_ptr(ws), _stream(stream)))


def moe_wait_selftest(kind: int, ctas: int, skip_cta: int, limit_ns: int, ws, stream=None,
                      raise_on_error=True) -> int:
    """Makes a bounded device wait expire on purpose (kind 0: an mbarrier
    nothing arrives on; kind 1: a grid barrier of `ctas` CTAs without CTA
    `skip_cta`'s arrival); read the outcome with moe_get_device_error(ws)."""
    st = _lib.moe_wait_selftest(kind, ctas, skip_cta, limit_ns, _ptr(ws), _stream(stream))
    return _check(st, "moe_wait_selftest", raise_on_error)


from .layer import MoELayer  # noqa: E402  (torch-level convenience wrapper)
