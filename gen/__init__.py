"""Seeded synthetic MoE-layer inputs, shared by the oracle and the CUDA path.

Holds no arithmetic of the layer itself: it only draws bits (SplitMix64, see
``moe_gen.c``) and lays them out in the byte formats the layer consumes:

* ``x``          bf16 bits, uint16 [T, H], N(0, 1)
* ``w_router``   bf16 bits, uint16 [E, H], N(0, 0.02)
* ``gu_codes``   uint32 [E+1, 2I, H/8]   gate rows 0..I-1, up rows I..2I-1
* ``gu_sb``      bf16 bits, uint16 [E+1, 2I, H/G, 2]   (scale, bias) per group
* ``d_codes``    uint32 [E+1, H, I/8]
* ``d_sb``       bf16 bits, uint16 [E+1, H, I/G, 2]
* ``logit_bias`` None, float32 [E] (row stride 0) or float32 [T, E]

Expert index E (the last one) is the shared expert.  Codes are uniform on
0..15, scale = bf16(|N(0, 0.02)|) and bias = -8 * scale, as the layer
workloads of the Lily pages' model call for (page 1, "A 35B Model Built for
Local Memory": 256 experts, 8 selected, groupwise-affine 4-bit weights).
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.ensure_built()
        _lib = ctypes.CDLL(path)
        _lib.gen_draw.restype = ctypes.c_uint64
        _lib.gen_draw.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        _lib.gen_key.restype = ctypes.c_uint64
        _lib.gen_key.argtypes = [ctypes.c_uint64] * 3
        _lib.gen_normal_bf16.argtypes = [ctypes.c_uint64, ctypes.c_double, ctypes.c_int,
                                         ctypes.c_void_p, ctypes.c_int64]
        _lib.gen_codes.argtypes = [ctypes.c_uint64, ctypes.c_void_p, ctypes.c_int64]
        _lib.gen_scale_bias.argtypes = [ctypes.c_uint64, ctypes.c_double, ctypes.c_void_p,
                                        ctypes.c_int64]
        _lib.gen_partial_shuffle.argtypes = [ctypes.c_uint64, ctypes.c_int32, ctypes.c_int32,
                                             ctypes.c_void_p, ctypes.c_void_p]
        _lib.gen_uniform_f32.argtypes = [ctypes.c_uint64, ctypes.c_double, ctypes.c_double, ctypes.c_void_p,
                                         ctypes.c_int64]
        _lib.gen_normal_f32.argtypes = [ctypes.c_uint64, ctypes.c_double, ctypes.c_void_p, ctypes.c_int64]
        _lib.gen_unit_bf16.argtypes = [ctypes.c_uint64, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p]
    return _lib


# tensor ids of the key derivation
TID_X, TID_ROUTER, TID_GU_CODES, TID_GU_SB, TID_D_CODES, TID_D_SB, TID_HOT, TID_BIASED = range(1, 9)


@dataclasses.dataclass(frozen=True)
class LayerSpec:
    """Shape and seed of one synthetic MoE layer."""
    T: int
    H: int = 2048
    I: int = 512
    E: int = 256
    k: int = 8
    G: int = 64
    seed: int = 0
    bias: str = "none"   # "none" | "zipf" | "hot"
    layers: int = 1
    name: str = ""

    def with_T(self, T: int) -> "LayerSpec":
        return dataclasses.replace(self, T=T)


CONFIGS = {
    0: LayerSpec(T=8, H=512, I=128, seed=0, name="tiny T=8 H=512 I=128"),
    1: LayerSpec(T=1, seed=1, layers=40, name="decode T=1 H=2048 I=512 x40 layers"),
    2: LayerSpec(T=512, seed=2, bias="zipf", name="prefill T=512 H=2048 I=512 zipf(1.1)"),
    3: LayerSpec(T=2048, seed=3, name="prefill T=2048 H=2048 I=512 uniform"),
    4: LayerSpec(T=16384, seed=4, bias="hot", name="prefill T=16384 H=2048 I=512 hot-8"),
}


def config(i: int) -> LayerSpec:
    return CONFIGS[i]


def _ptr(a: np.ndarray) -> int:
    assert a.flags.c_contiguous
    return a.ctypes.data


def normal_bf16(key: int, std: float, n: int, absval: bool = False) -> np.ndarray:
    out = np.empty(n, dtype=np.uint16)
    lib().gen_normal_bf16(key, std, 1 if absval else 0, _ptr(out), n)
    return out


def key(seed: int, tensor: int, layer: int) -> int:
    return int(lib().gen_key(seed, tensor, layer))


def make_router(spec: LayerSpec, layer: int = 0) -> np.ndarray:
    """Router weights bf16 [E, H] of one layer (the same as make_weights')."""
    return normal_bf16(key(spec.seed, TID_ROUTER, layer), 0.02, spec.E * spec.H).reshape(spec.E, spec.H)


def make_weights(spec: LayerSpec, layer: int = 0) -> dict:
    """Router and expert weights of one layer (E routed experts + 1 shared)."""
    E, H, I, G = spec.E, spec.H, spec.I, spec.G
    s = spec.seed
    w_router = make_router(spec, layer)
    gu_codes = np.empty((E + 1, 2 * I, H // 8), dtype=np.uint32)
    lib().gen_codes(key(s, TID_GU_CODES, layer), _ptr(gu_codes), gu_codes.size)
    gu_sb = np.empty((E + 1, 2 * I, H // G, 2), dtype=np.uint16)
    lib().gen_scale_bias(key(s, TID_GU_SB, layer), 0.02, _ptr(gu_sb), gu_sb.size // 2)
    d_codes = np.empty((E + 1, H, I // 8), dtype=np.uint32)
    lib().gen_codes(key(s, TID_D_CODES, layer), _ptr(d_codes), d_codes.size)
    d_sb = np.empty((E + 1, H, I // G, 2), dtype=np.uint16)
    lib().gen_scale_bias(key(s, TID_D_SB, layer), 0.02, _ptr(d_sb), d_sb.size // 2)
    return dict(w_router=w_router, gu_codes=gu_codes, gu_sb=gu_sb, d_codes=d_codes, d_sb=d_sb)


def make_activations(spec: LayerSpec, layer: int = 0) -> dict:
    """Token activations and the logit bias of one layer.

    x element i is stream element i, so a smaller T is a prefix of a larger one.
    """
    T, H, E = spec.T, spec.H, spec.E
    x = normal_bf16(key(spec.seed, TID_X, layer), 1.0, T * H).reshape(T, H)
    bias, stride = None, 0
    if spec.bias == "zipf":
        # Zipf(s = 1.1) expert popularity: log-weight -1.1 * ln(rank), rank = e + 1.
        bias = np.array([-1.1 * math.log(e + 1) for e in range(E)], dtype=np.float64).astype(np.float32)
        stride = 0
    elif spec.bias == "hot":
        lb = lib()
        hot = np.empty(8, dtype=np.int32)
        scratch = np.empty(E, dtype=np.int32)
        lb.gen_partial_shuffle(key(spec.seed, TID_HOT, 0), E, 8, _ptr(hot), _ptr(scratch))
        nb = T // 2
        biased = np.empty(max(nb, 1), dtype=np.int32)
        scratch_t = np.empty(max(T, 1), dtype=np.int32)
        lb.gen_partial_shuffle(key(spec.seed, TID_BIASED, 0), T, nb, _ptr(biased), _ptr(scratch_t))
        bias = np.zeros((T, E), dtype=np.float32)
        for t in biased[:nb]:
            bias[t, hot] = 8.0
        stride = E
    return dict(x=x, logit_bias=bias, bias_stride=stride)


def make_layer(spec: LayerSpec, layer: int = 0) -> dict:
    d = make_weights(spec, layer)
    d.update(make_activations(spec, layer))
    return d


def hot_experts(spec: LayerSpec) -> np.ndarray:
    hot = np.empty(8, dtype=np.int32)
    scratch = np.empty(spec.E, dtype=np.int32)
    lib().gen_partial_shuffle(key(spec.seed, TID_HOT, 0), spec.E, 8, _ptr(hot), _ptr(scratch))
    return hot


def bf16_to_f32(u16: np.ndarray) -> np.ndarray:
    """View bf16 bit patterns as float32 values (exact widening)."""
    return (np.asarray(u16, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16_bits(f: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bits, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(f, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


# ---------------------------------------------------------------- recurrent-state scan inputs

TID_GDN_Q, TID_GDN_K, TID_GDN_V, TID_GDN_G, TID_GDN_BETA, TID_GDN_S0 = range(20, 26)


@dataclasses.dataclass(frozen=True)
class ScanSpec:
    """Shape and seed of one synthetic Gated DeltaNet scan: B sequences of T
    new tokens, Hk key heads and Hv value heads (Hv a multiple of Hk) of dk
    and dv channels, 30 layers in a decode step."""
    B: int
    T: int
    Hk: int = 16
    Hv: int = 32
    dk: int = 128
    dv: int = 128
    seed: int = 0
    layers: int = 1
    name: str = ""

    def with_T(self, T: int) -> "ScanSpec":
        return dataclasses.replace(self, T=T)

    def with_B(self, B: int) -> "ScanSpec":
        return dataclasses.replace(self, B=B)


SCAN_CONFIGS = {
    0: ScanSpec(B=2, T=17, Hk=2, Hv=4, seed=10, name="tiny B=2 T=17 Hk=2 Hv=4"),
    1: ScanSpec(B=8, T=1, seed=11, layers=30, name="decode B=8 T=1 x30 layers"),
    2: ScanSpec(B=1, T=4, seed=12, layers=30, name="verification B=1 T=4 x30 layers"),
    3: ScanSpec(B=1, T=2048, seed=13, name="prefill B=1 T=2048"),
}


def scan_config(i: int) -> ScanSpec:
    return SCAN_CONFIGS[i]


def uniform_f32(key: int, lo: float, hi: float, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    lib().gen_uniform_f32(key, lo, hi, _ptr(out), n)
    return out


def normal_f32(key: int, std: float, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    lib().gen_normal_f32(key, std, _ptr(out), n)
    return out


def unit_bf16(key: int, nvec: int, dim: int) -> np.ndarray:
    out = np.empty(nvec * dim, dtype=np.uint16)
    lib().gen_unit_bf16(key, nvec, dim, _ptr(out))
    return out.reshape(nvec, dim)


def make_scan(spec: ScanSpec, layer: int = 0) -> dict:
    """Inputs of one scan: q, k unit vectors (bf16 [B,T,Hk,dk]), v ~ N(0,1)
    (bf16 [B,T,Hv,dv]), g (the log of the decay) uniform in [log 0.9, 0) so
    that the decay lies in [0.9, 1) (fp32 [B,T,Hv]), beta uniform in
    [0.05, 0.95) (fp32 [B,T,Hv]), initial state ~ N(0, 0.1) (fp32
    [B,Hv,dv,dk]), and the output scale dk^-1/2."""
    B, T, Hk, Hv, dk, dv, s = spec.B, spec.T, spec.Hk, spec.Hv, spec.dk, spec.dv, spec.seed
    q = unit_bf16(key(s, TID_GDN_Q, layer), B * T * Hk, dk).reshape(B, T, Hk, dk)
    k = unit_bf16(key(s, TID_GDN_K, layer), B * T * Hk, dk).reshape(B, T, Hk, dk)
    v = normal_bf16(key(s, TID_GDN_V, layer), 1.0, B * T * Hv * dv).reshape(B, T, Hv, dv)
    g = uniform_f32(key(s, TID_GDN_G, layer), -0.10536051565782628, 0.0, B * T * Hv).reshape(B, T, Hv)
    beta = uniform_f32(key(s, TID_GDN_BETA, layer), 0.05, 0.95, B * T * Hv).reshape(B, T, Hv)
    S0 = normal_f32(key(s, TID_GDN_S0, layer), 0.1, B * Hv * dv * dk).reshape(B, Hv, dv, dk)
    return dict(q=q, k=k, v=v, g=g, beta=beta, S0=S0, scale=float(dk) ** -0.5)
