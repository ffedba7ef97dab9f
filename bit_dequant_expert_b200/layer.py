"""Torch-level convenience wrapper: device buffers for one MoE layer and the
four library calls in order.  Allocation and marshalling only; the compute is
entirely in libmoe_b200."""
from __future__ import annotations

import numpy as np
import torch

from . import (MOE_MODE_PAIRS, MOE_MODE_SCATTER, MOE_PATH_AUTO, config, moe_combine, moe_decode_layer,
               moe_expert_ffn_path, moe_permute, moe_route, moe_workspace_init, moe_workspace_size)


def to_device(a, device, dtype=None) -> torch.Tensor:
    """numpy uint16 (bf16 bits) / uint32 / float32 / int32 -> device tensor with the same bytes."""
    if isinstance(a, torch.Tensor):
        return a.to(device)
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
    elif a.dtype == np.uint32:
        t = torch.from_numpy(a.view(np.int32))
    else:
        t = torch.from_numpy(a)
    if dtype is not None:
        t = t.to(dtype)
    return t.to(device)


def check_rows(t, name: str, H: int, device: torch.device) -> None:
    """Raises unless t is a contiguous bf16 [n, H] tensor on `device` (any
    index of its type when `device` names none): the library reads it through
    its data pointer alone."""
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor, got %s" % (name, type(t).__name__))
    if t.dtype != torch.bfloat16:
        raise TypeError("%s must be bfloat16, got %s" % (name, t.dtype))
    if t.dim() != 2 or t.shape[1] != H:
        raise ValueError("%s must have shape [T, %d], got %s" % (name, H, tuple(t.shape)))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if t.device.type != device.type or (device.index is not None and t.device.index != device.index):
        raise ValueError("%s is on %s, the layer on %s" % (name, t.device, device))


def check_f32(t, name: str, min_numel: int, device: torch.device) -> None:
    """Raises unless t is a contiguous fp32 tensor of at least min_numel
    elements on `device`."""
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor, got %s" % (name, type(t).__name__))
    if t.dtype != torch.float32:
        raise TypeError("%s must be float32, got %s" % (name, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if t.numel() < min_numel:
        raise ValueError("%s has %d elements, fewer than the %d read" % (name, t.numel(), min_numel))
    if t.device.type != device.type or (device.index is not None and t.device.index != device.index):
        raise ValueError("%s is on %s, the layer on %s" % (name, t.device, device))


_BF16_BITS = (np.dtype(np.uint16), torch.bfloat16, torch.int16)
_CODE_WORDS = (np.dtype(np.uint32), torch.int32, torch.uint32)


def check_weights(weights: dict, group_size: int = 64) -> tuple:
    """(E, H, I) of a packed layer, after checking that every array has the
    shape and element type the library reads it with (bf16 bits for w_router
    and the (scale, bias) pairs, 32-bit words for the codes); raises
    ValueError or TypeError otherwise."""
    for name in ("w_router", "gu_codes", "gu_sb", "d_codes", "d_sb"):
        if name not in weights:
            raise ValueError("weights lack %s" % name)
    gu = weights["gu_codes"]
    if len(gu.shape) != 3:
        raise ValueError("gu_codes must be [E+1, 2I, H/8], got %s" % (tuple(gu.shape),))
    E1, I2, H8 = (int(v) for v in gu.shape)
    E, H, I, G = E1 - 1, 8 * H8, I2 // 2, group_size
    if E < 1 or I2 % 2 or H % G or I % G:
        raise ValueError("gu_codes shape %s gives no layer with groups of %d" % (tuple(gu.shape), G))
    want = {"w_router": (E, H), "gu_codes": (E1, 2 * I, H // 8), "gu_sb": (E1, 2 * I, H // G, 2),
            "d_codes": (E1, H, I // 8), "d_sb": (E1, H, I // G, 2)}
    for name, shape in want.items():
        got = tuple(int(v) for v in weights[name].shape)
        if got != shape:
            raise ValueError("%s must have shape %s, got %s" % (name, shape, got))
        kinds = _CODE_WORDS if name.endswith("codes") else _BF16_BITS
        if weights[name].dtype not in kinds:
            raise TypeError("%s has element type %s" % (name, weights[name].dtype))
    return E, H, I


class MoELayer:
    """One layer's weights resident on the device plus its scratch buffers.

    weights: dict with w_router [E,H] bf16 bits, gu_codes [E+1,2I,H/8] u32,
    gu_sb [E+1,2I,H/G,2] bf16 bits, d_codes [E+1,H,I/8] u32, d_sb
    [E+1,H,I/G,2] bf16 bits (numpy arrays or device tensors).
    """

    def __init__(self, weights: dict, max_tokens: int, device="cuda", mode=MOE_MODE_SCATTER,
                 path=MOE_PATH_AUTO, has_shared=True):
        E, H, I = check_weights(weights)
        E1 = E + 1
        self.cfg = config(hidden=H, inter=I, num_experts=E1 - 1, top_k=8, group_size=64,
                          has_shared=1 if has_shared else 0)
        self.H, self.I, self.E, self.K = H, I, E1 - 1, 8
        self.device = torch.device(device)
        self.mode, self.path = mode, path
        self.max_tokens = max_tokens
        self.w_router = to_device(weights["w_router"], self.device)
        self.gu_codes = to_device(weights["gu_codes"], self.device)
        self.gu_sb = to_device(weights["gu_sb"], self.device)
        self.d_codes = to_device(weights["d_codes"], self.device)
        self.d_sb = to_device(weights["d_sb"], self.device)
        nbytes = moe_workspace_size(self.cfg, max_tokens)
        if nbytes == 0:
            raise ValueError("unsupported layer configuration")
        self.ws = torch.zeros(nbytes, dtype=torch.uint8, device=self.device)
        moe_workspace_init(self.ws)
        T, K, E = max_tokens, self.K, self.E
        dev = self.device
        self.topk_idx = torch.empty(T, K, dtype=torch.int32, device=dev)
        self.topk_w = torch.empty(T, K, dtype=torch.float32, device=dev)
        self.counts = torch.empty(E, dtype=torch.int32, device=dev)
        self.offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
        self.row_to_pair = torch.empty(T * K, dtype=torch.int32, device=dev)
        self.pair_to_row = torch.empty(T * K, dtype=torch.int32, device=dev)
        if mode == MOE_MODE_SCATTER:
            self.out0 = torch.empty(T, H, dtype=torch.float32, device=dev)
            self.out1 = None
        else:
            self.out0 = torch.empty(T * K, H, dtype=torch.bfloat16, device=dev)
            self.out1 = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
        self.y = torch.empty(T, H, dtype=torch.bfloat16, device=dev)

    def route(self, x, T, logit_bias=None, bias_stride=0, logits_in=None, stream=None):
        moe_route(self.cfg, T, x, self.w_router, logits_in, logit_bias, bias_stride, self.topk_idx, self.topk_w,
                  self.counts, self.ws, stream=stream)

    def permute(self, T, stream=None):
        moe_permute(self.cfg, T, self.topk_idx, self.counts, self.offsets, self.row_to_pair, self.pair_to_row,
                    self.ws, stream=stream)

    def expert_ffn(self, x, T, stream=None, path=None):
        moe_expert_ffn_path(self.cfg, T, x, self.gu_codes, self.gu_sb, self.d_codes, self.d_sb, self.offsets,
                            self.row_to_pair, self.topk_w, self.mode, self.out0, self.out1, self.ws,
                            self.path if path is None else path, stream=stream)

    def combine(self, T, stream=None, y_out=None):
        y = self.y if y_out is None else y_out
        moe_combine(self.cfg, T, self.mode, self.out0, self.out1, self.pair_to_row, self.topk_w, y,
                    stream=stream)

    def forward(self, x: torch.Tensor, logit_bias=None, bias_stride=0, logits_in=None, stream=None,
                y_out=None) -> torch.Tensor:
        """y [T, H] bf16 for x [T, H] bf16 (written to y_out if given, else to
        the layer's own output buffer, a view of which is returned)."""
        check_rows(x, "x", self.H, self.device)
        T = x.shape[0]
        if T > self.max_tokens:
            raise ValueError("T=%d exceeds max_tokens=%d" % (T, self.max_tokens))
        if y_out is not None:
            check_rows(y_out, "y_out", self.H, self.device)
            if y_out.shape[0] < T:
                raise ValueError("y_out has %d rows, fewer than the %d tokens" % (y_out.shape[0], T))
        if logit_bias is not None:
            if bias_stride < 0:
                raise ValueError("bias_stride must be >= 0, got %d" % bias_stride)
            check_f32(logit_bias, "logit_bias", (T - 1) * bias_stride + self.E, self.device)
        if logits_in is not None:
            check_f32(logits_in, "logits_in", T * self.E, self.device)
        if self.fused_ok(T) and logits_in is None:
            return self.decode_fused(x, T, logit_bias, bias_stride, stream, y_out)
        self.route(x, T, logit_bias, bias_stride, logits_in, stream)
        self.permute(T, stream)
        self.expert_ffn(x, T, stream)
        self.combine(T, stream, y_out)
        return self.y[:T] if y_out is None else y_out

    def fused_ok(self, T) -> bool:
        """Whether forward() takes the two-launch decode layer for T tokens."""
        return (T <= 8 and self.mode == MOE_MODE_SCATTER and self.path == MOE_PATH_AUTO and self.E == 256
                and self.H in (512, 1024, 2048) and self.I <= 2048)

    def decode_fused(self, x, T, logit_bias=None, bias_stride=0, stream=None, y_out=None) -> torch.Tensor:
        """The layer for T <= 8 tokens in two launches (moe_decode_layer)."""
        y = self.y if y_out is None else y_out
        moe_decode_layer(self.cfg, T, x, self.w_router, logit_bias, bias_stride, self.gu_codes, self.gu_sb,
                         self.d_codes, self.d_sb, self.topk_idx, self.topk_w, self.counts, self.offsets,
                         self.row_to_pair, self.pair_to_row, self.out0, y, self.ws, stream=stream)
        return self.y[:T] if y_out is None else y_out
