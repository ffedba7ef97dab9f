"""moe_router_logits against the oracle's contract-order logits, bit for
bit, over shapes that reach both router kernels: the weights-resident tiled
kernel (T >= 64, H a multiple of 256 up to 2048) with one to eight 256-input
stages, ragged 16-token tiles and both bias forms, and the per-warp kernel
(T < 64).  Equal logits make the selection equal; the routing tests check
that separately."""
import numpy as np
import pytest

import gen
import oracle

pytestmark = pytest.mark.gpu


def _logits_gpu(x, w_router, bias=None, stride=0):
    import torch
    import bit_dequant_expert_b200 as m
    from bit_dequant_expert_b200.layer import to_device
    T, H = x.shape
    E = w_router.shape[0]
    cfg = m.config(hidden=H)
    ws = torch.zeros(m.moe_workspace_size(cfg, T), dtype=torch.uint8, device="cuda")
    out = torch.full((T, E), float("nan"), dtype=torch.float32, device="cuda")
    xd, wd = to_device(x, "cuda"), to_device(w_router, "cuda")
    bd = None if bias is None else to_device(np.ascontiguousarray(bias, dtype=np.float32), "cuda")
    m.moe_router_logits(cfg, T, xd, wd, bd, stride, out, ws)
    torch.cuda.synchronize()
    assert m.moe_get_device_error(ws) == m.MOE_OK
    return out.cpu().numpy()


def _check(x, w_router, bias=None, stride=0, tokens=None):
    got = _logits_gpu(x, w_router, bias, stride)
    tok = np.arange(x.shape[0]) if tokens is None else np.asarray(tokens)
    ref = oracle.router_logits(x, w_router, bias=bias, bias_stride=stride, tokens=tok.astype(np.int32))
    sel = got[tok]
    bad = np.argwhere(sel.view(np.uint32) != ref.view(np.uint32))
    assert len(bad) == 0, (len(bad), bad[:4].tolist(), sel[tuple(bad[0])], ref[tuple(bad[0])])


@pytest.mark.parametrize("T,H,bias", [
    (64, 256, "none"),        # one stage, four full token tiles
    (65, 512, "token"),       # a ragged last tile of one token, per-token bias
    (100, 1024, "row"),       # one bias row for every token
    (63, 2048, "none"),       # below the tiled kernel's threshold
    (300, 2048, "token"),
    (2047, 2048, "none"),     # many steps per CTA, ragged tail
])
def test_router_logits_bitexact(T, H, bias):
    spec = gen.LayerSpec(T=T, H=H, seed=11 + T)
    x = gen.make_activations(spec)["x"]
    w = gen.make_router(spec)
    rng = np.random.default_rng(T)
    b, stride = None, 0
    if bias == "token":
        b, stride = (rng.standard_normal((T, 256)) * 0.1).astype(np.float32), 256
    elif bias == "row":
        b = (rng.standard_normal(256) * 0.1).astype(np.float32)
    _check(x, w, b, stride)


@pytest.mark.parametrize("cfg_id", [2, 3])
def test_router_logits_configs(cfg_id):
    spec = gen.config(cfg_id)
    act = gen.make_activations(spec)
    _check(act["x"], gen.make_router(spec), act["logit_bias"], act["bias_stride"])


def test_router_logits_config4_sampled():
    """T = 16384 with the per-token hot bias: 512 tokens spread over both
    halves, computed by the oracle one by one."""
    spec = gen.config(4)
    act = gen.make_activations(spec)
    rng = np.random.default_rng(4)
    tok = np.unique(np.concatenate([[0, spec.T - 1], rng.choice(spec.T, 510, replace=False)]))
    _check(act["x"], gen.make_router(spec), act["logit_bias"], act["bias_stride"], tokens=tok)


def test_router_logits_mixed_magnitudes():
    """Slices of very different sizes: x scaled by 2^(3 (chunk mod 32) - 48),
    so every slice partial has its own exponent and a different addition tree
    or slice order would change the last bits of most logits."""
    T, H = 96, 2048
    spec = gen.LayerSpec(T=T, H=H, seed=5)
    x = gen.bf16_to_f32(gen.make_activations(spec)["x"]).astype(np.float64)
    chunk = np.arange(H) // 8
    x = x * np.exp2(3.0 * (chunk % 32) - 48.0)[None, :]
    xb = gen.f32_to_bf16_bits(x.astype(np.float32)).reshape(T, H)
    _check(xb, gen.make_router(spec))
