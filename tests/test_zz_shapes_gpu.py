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
AUTO, SIMT, GEMV, TC = 0, 1, 2, 3


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
                                         (TC, PAIRS, 33)])
def test_without_shared_expert(path, mode, T):
    """has_shared = 0: only the routed experts contribute; the matrices at
    index E are never read.  Checked against the oracle without the shared
    expert, with the shared expert's codes set to values that would show if
    they were read."""
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
