"""GPU parity for layer shapes beyond the five synthetic configurations:
decode-layer shapes with 2-16 tokens (speculative decoding's verification
batches, and the crossover to the tensor-core kernel), and layers without the
shared expert on every implementation path.  Collected after the other GPU
tests, so a failure here comes after every other test has run."""
import numpy as np
import pytest

import gen
import oracle
from gpu_util import check_output, check_permutation_props, check_routing, run_layer

pytestmark = pytest.mark.gpu

SCATTER, PAIRS = 0, 1
AUTO, SIMT, GEMV, TC, TC_GEMV = 0, 1, 2, 3, 4


def _decode_shape(T):
    """Layer 3 of the decode seeds (H 2048, I 512) with T tokens."""
    return gen.make_layer(gen.config(1).with_T(T), 3)


@pytest.mark.parametrize("T", [2, 4, 5, 8])
def test_fused_decode_verification_batches(T):
    """2-8 tokens at decode-layer shapes take the fused decode layer; the
    weights it reads are those of the union of the experts the tokens
    select.  Routing, counts and both maps bit-exact; outputs within
    tolerance."""
    lay = _decode_shape(T)
    out, L = run_layer(lay, SCATTER, AUTO)
    assert L.fused_ok(T)
    assert out["err"] == 0
    idx_ref = check_routing(out, lay)
    counts, offsets, r2p, p2r = oracle.permute(idx_ref, 256)
    assert np.array_equal(out["counts"], counts) and np.array_equal(out["offsets"], offsets)
    assert np.array_equal(out["r2p"], r2p) and np.array_equal(out["p2r"], p2r)
    check_output(out, lay, np.arange(T))


def test_decode_shape_past_the_crossover():
    """16 tokens at decode-layer shapes take the four calls with the
    tensor-core expert FFN (scatter mode)."""
    T = 16
    lay = _decode_shape(T)
    out, L = run_layer(lay, SCATTER, AUTO)
    assert not L.fused_ok(T)
    assert out["err"] == 0
    check_routing(out, lay)
    check_permutation_props(out, T)
    check_output(out, lay, np.arange(T))


@pytest.mark.parametrize("path,mode,T", [(AUTO, SCATTER, 1), (AUTO, SCATTER, 6), (GEMV, SCATTER, 3),
                                         (SIMT, SCATTER, 8), (SIMT, PAIRS, 8), (TC, SCATTER, 33),
                                         (TC, PAIRS, 33), (TC_GEMV, SCATTER, 33), (TC_GEMV, SCATTER, 300)])
def test_without_shared_expert(path, mode, T):
    """has_shared = 0: only the routed experts contribute; the matrices at
    index E are never read.  Checked against the oracle without the shared
    expert, with the shared expert's codes set to values that would show if
    they were read.  The split path at T = 33 leaves the tensor-core kernel
    no tile at all (every expert holds at most 8 rows)."""
    from bit_dequant_expert_b200.layer import MoELayer
    lay = dict(gen.make_layer(gen.config(0).with_T(T), 1))
    for name in ("gu_codes", "d_codes"):
        codes = lay[name].copy()
        codes[-1] = 0xFFFFFFFF
        lay[name] = codes
    L = MoELayer(lay, max_tokens=T, mode=mode, path=path, has_shared=False)
    out, _ = run_layer(lay, mode, path, layer_obj=L)
    assert out["err"] == 0
    check_routing(out, lay)
    check_output(out, lay, np.arange(T), has_shared=False)


def _scale_bf16(bits, e):
    """bf16 bits times 2^e, exactly (normal inputs and results)."""
    f = gen.bf16_to_f32(bits).astype(np.float32) * np.float32(2.0 ** e)
    out = gen.f32_to_bf16_bits(f)
    assert np.array_equal(gen.bf16_to_f32(out), f)
    return out


@pytest.mark.parametrize("path,T", [(AUTO, 8), (GEMV, 8), (AUTO, 33)])
def test_routing_with_subnormal_logits(path, T):
    """x and the router matrix scaled by 2^-64 each: every product and every
    logit is subnormal in fp32.  Routing must still match the oracle bit for
    bit, which holds only if neither side flushes subnormals to zero (a flush
    would zero every logit and pick experts 0..7).  T = 8 covers the fused
    decode kernel and the small router, T = 33 the tiled router."""
    lay = dict(gen.make_layer(gen.config(0).with_T(T), 2))
    lay["x"] = _scale_bf16(lay["x"], -64)
    lay["w_router"] = _scale_bf16(lay["w_router"], -64)
    logits = oracle.router_logits(lay["x"], lay["w_router"])
    assert np.all(np.abs(logits) < 2.0 ** -126) and np.all(logits != 0)
    out, _ = run_layer(lay, SCATTER, path)
    assert out["err"] == 0
    idx_ref = check_routing(out, lay)
    assert not np.array_equal(np.sort(idx_ref, axis=1), np.tile(np.arange(8), (T, 1)))


@pytest.mark.parametrize("path,T", [(GEMV, 8), (AUTO, 33)])
def test_given_subnormal_logits_with_ties(path, T):
    """Given logits that are multiples of 2^-140 (subnormal) with mass ties:
    the top 8 by (logit desc, index asc) and their weights match the oracle."""
    rng = np.random.default_rng(T)
    li = (rng.integers(0, 3, size=(T, 256)) * 2.0 ** -140).astype(np.float32)
    lay = gen.make_layer(gen.config(0).with_T(T), 2)
    out, _ = run_layer(lay, SCATTER, path, logits_in=li)
    assert out["err"] == 0
    idx_ref, w_ref = oracle.select(li, 8)
    assert np.array_equal(out["idx"], idx_ref)
    assert np.abs(out["w"] - w_ref).max() <= 2e-6


@pytest.mark.parametrize("path,mode,T", [(AUTO, SCATTER, 8), (GEMV, SCATTER, 3), (SIMT, PAIRS, 8),
                                         (TC, SCATTER, 33), (TC, PAIRS, 33)])
def test_general_scale_and_bias(path, mode, T):
    """(scale, bias) pairs of any sign and with no relation between them (the
    synthetic layers all have positive scales and bias = -8 scale): every path
    must compute scale * q + bias as written."""
    rng = np.random.default_rng(100 + T)
    lay = dict(gen.make_layer(gen.config(0).with_T(T), 4))
    for name in ("gu_sb", "d_sb"):
        sb = np.empty_like(lay[name])
        sb[..., 0] = gen.f32_to_bf16_bits((0.02 * rng.standard_normal(sb.shape[:-1])).astype(np.float32))
        sb[..., 1] = gen.f32_to_bf16_bits((0.05 * rng.standard_normal(sb.shape[:-1])).astype(np.float32))
        lay[name] = sb
    out, _ = run_layer(lay, mode, path)
    assert out["err"] == 0
    check_routing(out, lay)
    check_output(out, lay, np.arange(T))


@pytest.mark.parametrize("mode,T", [(SCATTER, 33), (PAIRS, 100)])
def test_tensor_core_hidden_1024(mode, T):
    """H = 1024, I = 256 on the tensor-core path: 16 (scale, bias) groups per
    gate/up row and 4 per down row, four 64-column blocks of h."""
    lay = gen.make_layer(gen.LayerSpec(T=T, H=1024, I=256, seed=12), 1)
    out, _ = run_layer(lay, mode, TC)
    assert out["err"] == 0
    check_routing(out, lay)
    check_output(out, lay, np.arange(0, T, 3))


@pytest.mark.parametrize("mode", [SCATTER, PAIRS])
def test_one_layer_across_token_counts(mode):
    """One layer object (buffers and workspace for 64 tokens) called with
    token counts that switch between the decode kernel, the fused decode
    layer and the tensor-core path, as a serving loop would: the workspace's
    arrival counter and tickets carry over from call to call, and every call
    matches the oracle on its own tokens (a prefix of the same batch)."""
    from bit_dequant_expert_b200.layer import MoELayer
    lay = gen.make_layer(gen.config(0).with_T(64), 5)
    L = MoELayer(lay, max_tokens=64, mode=mode)
    for T in (5, 33, 1, 8, 64, 2, 8, 17):
        out, _ = run_layer(lay, mode, AUTO, T=T, layer_obj=L)
        assert out["err"] == 0, T
        check_routing(out, lay, T=T)
        check_output(out, lay, np.arange(T), T=T)
