"""The split expert-FFN path (MOE_PATH_TC_GEMV, scatter mode): the tensor-core
kernel takes the experts of more than 8 rows and the shared expert, the
decode kernel's row-list launch the experts of 1..8 rows, both adding into the
same y_acc.  Checked against the oracle on sampled tokens (every token when T
is small), against the tensor-core-only path on every token, and for the
automatic choice of it."""
import numpy as np
import pytest

from gpu_util import check_output, check_routing, check_routing_and_permutation, row_rel_err, run_layer
from test_parity_gpu import _sample_tokens, layer_of

pytestmark = pytest.mark.gpu

SCATTER, PAIRS = 0, 1
AUTO, TC, TC_GEMV = 0, 3, 4


def _rows_per_expert(out):
    c = out["counts"][:256]
    return int(((c >= 1) & (c <= 8)).sum()), int((c > 8).sum())


@pytest.mark.parametrize("cfg_id,T", [(0, 9), (0, 33), (0, 300), (3, 33), (3, 300), (3, 1000), (3, 4097)])
def test_split_shapes(cfg_id, T):
    """H 512 / I 128 and H 2048 / I 512 layers: from almost every expert small
    (T = 9, 33) through a mix (300, 1000) to none (4097: the row-list launch
    finds no expert and adds nothing)."""
    lay = layer_of(cfg_id, T=T)
    out, _ = run_layer(lay, SCATTER, TC_GEMV)
    assert out["err"] == 0
    check_routing(out, lay)
    small, big = _rows_per_expert(out)
    if T <= 300:
        assert small > 0
    if T == 4097:
        assert small == 0
    check_output(out, lay, _sample_tokens(T, 24, T + 1))


def test_split_zipf_config():
    """The Zipf-skewed T = 512 layer: experts of 1 to hundreds of rows."""
    lay = layer_of(2)
    T = lay["x"].shape[0]
    out, _ = run_layer(lay, SCATTER, TC_GEMV)
    assert out["err"] == 0
    check_routing_and_permutation(out, lay)
    small, big = _rows_per_expert(out)
    assert small > 10 and big > 10, (small, big)
    check_output(out, lay, _sample_tokens(T, 32, 7))


@pytest.mark.parametrize("cfg_id,T", [(3, 300), (2, 512)])
def test_split_matches_tc_on_every_token(cfg_id, T):
    """Every token of the split path within 2e-2 of the tensor-core-only path
    (two approximations each within 1e-2 of the oracle), so no token's
    small-expert rows are lost or added twice."""
    lay = layer_of(cfg_id, T=T)
    a, _ = run_layer(lay, SCATTER, TC_GEMV)
    b, _ = run_layer(lay, SCATTER, TC)
    assert a["err"] == 0 and b["err"] == 0
    assert np.array_equal(a["idx"], b["idx"])
    assert np.max(row_rel_err(a["y"], b["y"])) < 2e-2


def test_auto_takes_split_for_few_rows_per_expert():
    """MOE_PATH_AUTO splits at H 2048 when the experts hold at most 12 rows on
    average (T * 8 <= 12 * 256), in scatter mode only."""
    import bit_dequant_expert_b200 as m
    cfg = m.config()
    for T, split in ((16, True), (300, True), (384, True), (385, False), (512, False), (2048, False)):
        n_tc = m.moe_launch_count(cfg, T, SCATTER, TC)
        assert m.moe_launch_count(cfg, T, SCATTER, TC_GEMV) == n_tc + 1
        assert m.moe_launch_count(cfg, T, SCATTER, AUTO) == n_tc + (1 if split else 0), T
        assert m.moe_launch_count(cfg, T, PAIRS, AUTO) == m.moe_launch_count(cfg, T, PAIRS, TC)
        assert m.moe_launch_count(cfg, T, PAIRS, TC_GEMV) == -1
    small = m.config(hidden=512, inter=128)
    assert m.moe_launch_count(small, 33, SCATTER, AUTO) == m.moe_launch_count(small, 33, SCATTER, TC)
