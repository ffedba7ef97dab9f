"""Helpers for the GPU parity tests: run the CUDA path through the C ABI on
seeded inputs and compare with the CPU oracle."""
from __future__ import annotations

import numpy as np

import oracle

ROW_REL_TOL = 1e-2       # per token: max_h |y_gpu - y_ref| / max_h |y_ref|
W_ABS_TOL = 2e-6         # routing weights, |w_gpu - w_ref|
W_SUM_TOL = 1e-6         # |sum_k w - 1|


def bf16_tensor_to_f64(t) -> np.ndarray:
    import torch
    return t.detach().to(torch.float32).cpu().numpy().astype(np.float64)


def row_rel_err(y, ref) -> np.ndarray:
    num = np.abs(y - ref).max(axis=1)
    den = np.abs(ref).max(axis=1)
    return num / np.maximum(den, 1e-300)


def run_layer(lay: dict, mode, path, T=None, logits_in=None, max_tokens=None, layer_obj=None):
    """Runs the four calls; returns (outputs dict of numpy arrays, MoELayer)."""
    import torch
    import bit_dequant_expert_b200 as m
    from bit_dequant_expert_b200.layer import MoELayer, to_device
    T = T or lay["x"].shape[0]
    L = layer_obj or MoELayer(lay, max_tokens=max_tokens or T, mode=mode, path=path)
    x = to_device(lay["x"][:T], "cuda")
    bias = lay.get("logit_bias")
    stride = int(lay.get("bias_stride", 0))
    bias_t = None if bias is None else to_device(bias[:T] if stride else bias, "cuda")
    li = None if logits_in is None else to_device(np.ascontiguousarray(logits_in, dtype=np.float32), "cuda")
    y = L.forward(x, logit_bias=bias_t, bias_stride=stride, logits_in=li)
    torch.cuda.synchronize()
    out = dict(
        y=bf16_tensor_to_f64(y),
        idx=L.topk_idx[:T].cpu().numpy(),
        w=L.topk_w[:T].cpu().numpy(),
        counts=L.counts.cpu().numpy(),
        offsets=L.offsets.cpu().numpy(),
        r2p=L.row_to_pair[:T * 8].cpu().numpy(),
        p2r=L.pair_to_row[:T * 8].cpu().numpy(),
        err=m.moe_get_device_error(L.ws),
    )
    return out, L


def check_routing(out, lay, tokens=None, T=None):
    """Bit-exact indices and toleranced weights against the oracle."""
    T = T or lay["x"].shape[0]
    tok = np.arange(T) if tokens is None else np.asarray(tokens)
    li = oracle.router_logits(lay["x"][:T], lay["w_router"], bias=lay.get("logit_bias"),
                              bias_stride=int(lay.get("bias_stride", 0)), tokens=tok.astype(np.int32))
    idx_ref, w_ref = oracle.select(li, 8)
    assert np.array_equal(out["idx"][tok], idx_ref), "routing indices differ"
    assert np.abs(out["w"][tok] - w_ref).max() <= W_ABS_TOL
    assert np.abs(out["w"][tok].astype(np.float64).sum(axis=1) - 1.0).max() <= W_SUM_TOL
    return idx_ref


def check_routing_and_permutation(out, lay, T=None):
    """Every token: indices bit-exact, weights within tolerance, and counts,
    offsets and both row maps bit-exact against the oracle's permutation of
    the oracle's routing."""
    idx_ref = check_routing(out, lay, T=T)
    counts, offsets, r2p, p2r = oracle.permute(idx_ref, 256)
    assert np.array_equal(out["counts"], counts), "counts differ"
    assert np.array_equal(out["offsets"], offsets), "offsets differ"
    assert np.array_equal(out["r2p"], r2p), "row_to_pair differs"
    assert np.array_equal(out["p2r"], p2r), "pair_to_row differs"
    return idx_ref


def spread_tokens(lay, n, seed):
    """n tokens for an output check: the first and last, then as many biased
    (hot-expert) tokens as unbiased ones when the layer has a per-token bias,
    else a uniform draw."""
    T = lay["x"].shape[0]
    rng = np.random.default_rng(seed)
    bias = lay.get("logit_bias")
    if bias is None or not int(lay.get("bias_stride", 0)):
        pick = rng.choice(np.arange(1, T - 1), n - 2, replace=False)
    else:
        biased = np.nonzero(np.asarray(bias).any(axis=1))[0]
        plain = np.setdiff1d(np.arange(T), biased)
        half = (n - 2) // 2
        pick = np.concatenate([rng.choice(biased, half, replace=False),
                               rng.choice(plain, n - 2 - half, replace=False)])
    return np.unique(np.concatenate([[0, T - 1], pick])).astype(np.int64)


def check_permutation_props(out, T, E=256, K=8):
    """Properties that hold at any size, on the device's own routing."""
    idx = out["idx"].reshape(T, K)
    counts, offsets, r2p, p2r = out["counts"], out["offsets"], out["r2p"], out["p2r"]
    assert np.array_equal(counts, np.bincount(idx.ravel(), minlength=E))
    assert offsets[0] == 0 and offsets[E] == T * K and np.array_equal(np.diff(offsets), counts)
    assert np.array_equal(np.sort(r2p), np.arange(T * K))
    assert np.array_equal(p2r[r2p], np.arange(T * K))
    e_of_row = idx.ravel()[r2p]
    t_of_row = r2p // K
    key = e_of_row.astype(np.int64) * (T + 1) + t_of_row
    assert np.all(np.diff(key) > 0), "rows are not ordered by (expert, token)"
    assert np.array_equal(e_of_row, np.repeat(np.arange(E), counts))


def check_output(out, lay, tokens, T=None, logits_in=None, tol=ROW_REL_TOL, has_shared=True):
    T = T or lay["x"].shape[0]
    sub = dict(lay)
    sub["x"] = lay["x"][:T]
    if lay.get("logit_bias") is not None and int(lay.get("bias_stride", 0)):
        sub["logit_bias"] = lay["logit_bias"][:T]
    y_ref, idx_ref, _ = oracle.layer(sub, tokens=np.asarray(tokens, dtype=np.int32), logits_in=logits_in,
                                     has_shared=has_shared)
    err = row_rel_err(out["y"][tokens], y_ref)
    assert err.max() <= tol, "max row-relative error %.3e (token %d)" % (err.max(), int(np.argmax(err)))
    return err
