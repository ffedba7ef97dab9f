"""moe_permute_static, the entry point for callers that cannot allocate
device memory (a plugin whose host runtime owns every device allocation, a
real-time path that may not call cudaMalloc): it must give exactly the
oracle's permutation, and the results of moe_permute, call after call, with
its scratch in the library's fixed device array.  Collected last so a failure
here comes after every other test has run."""
import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.gpu


def _routing(T, seed):
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.permutation(256)[:8] for _ in range(T)]).astype(np.int32)
    idx[: T // 3] = np.arange(8, 16)          # a skewed share, so counts are uneven
    return idx


def _static(m, cfg, idx, counts=True):
    """One moe_permute_static call on outputs pre-filled with junk; returns
    (offsets, row_to_pair, pair_to_row, err_out) on the host."""
    import torch
    T = idx.shape[0]
    d_idx = torch.from_numpy(idx).cuda()
    d_cnt = torch.from_numpy(np.bincount(idx.ravel(), minlength=256).astype(np.int32)).cuda() if counts else None
    got = [torch.full((n,), -7, dtype=torch.int32, device="cuda") for n in (257, T * 8, T * 8)]
    err = torch.full((1,), 99, dtype=torch.int32, device="cuda")
    m.moe_permute_static(cfg, T, d_idx, d_cnt, got[0], got[1], got[2], err)
    torch.cuda.synchronize()
    return [g.cpu().numpy() for g in got] + [int(err.item())]


def _moe_permute(m, cfg, idx):
    import torch
    T = idx.shape[0]
    d_idx = torch.from_numpy(idx).cuda()
    d_cnt = torch.from_numpy(np.bincount(idx.ravel(), minlength=256).astype(np.int32)).cuda()
    ws = torch.zeros(m.moe_workspace_size(cfg, T), dtype=torch.uint8, device="cuda")
    ref = [torch.empty(n, dtype=torch.int32, device="cuda") for n in (257, T * 8, T * 8)]
    m.moe_permute(cfg, T, d_idx, d_cnt, ref[0], ref[1], ref[2], ws)
    assert m.moe_get_device_error(ws) == m.MOE_OK
    return [r.cpu().numpy() for r in ref]


def _check(m, cfg, idx):
    _, offsets, r2p, p2r = oracle.permute(idx, 256)
    ref = _moe_permute(m, cfg, idx)
    for _ in range(2):                          # two calls in a row share the static scratch
        got = _static(m, cfg, idx)
        assert got[3] == m.MOE_OK
        for a, b, c in zip(got[:3], (offsets, r2p, p2r), ref):
            assert np.array_equal(a, b)         # the oracle's permutation
            assert np.array_equal(a, c)         # and moe_permute's


# T <= 256 takes the single-block kernel (no scratch); larger T the three-kernel path
@pytest.mark.parametrize("T,seed", [(1, 5), (256, 6), (257, 7), (4097, 1), (1000, 2), (16384, 3)])
def test_permute_static_matches_oracle_and_moe_permute(T, seed):
    import bit_dequant_expert_b200 as m
    _check(m, m.config(), _routing(T, seed))


def test_permute_static_changing_sizes_back_to_back():
    """Calls with different token counts one after another on the shared
    array: each result depends only on its own inputs."""
    import bit_dequant_expert_b200 as m
    cfg = m.config()
    for T, seed in ((16384, 11), (300, 12), (4097, 13), (16384, 14), (2, 15)):
        _check(m, cfg, _routing(T, seed))


@pytest.mark.parametrize("T", [4, 1000, 5000])
def test_permute_static_reports_bad_routing(T):
    """A repeated expert within a token, then an index out of range, come back
    as MOE_ERR_BOUNDS in err_out; a clean call afterwards reports MOE_OK."""
    import bit_dequant_expert_b200 as m
    cfg = m.config()
    idx = _routing(T, 21)
    bad = idx.copy()
    bad[T // 2, 5] = bad[T // 2, 2]
    assert _static(m, cfg, bad, counts=False)[3] == m.MOE_ERR_BOUNDS
    bad = idx.copy()
    bad[T - 1, 7] = 300
    assert _static(m, cfg, bad, counts=False)[3] == m.MOE_ERR_BOUNDS
    got = _static(m, cfg, idx)
    assert got[3] == m.MOE_OK
    _, offsets, r2p, p2r = oracle.permute(idx, 256)
    assert np.array_equal(got[0], offsets) and np.array_equal(got[1], r2p) and np.array_equal(got[2], p2r)


def test_permute_static_rejects_oversize():
    import bit_dequant_expert_b200 as m
    cfg = m.config()
    T = m.MOE_STATIC_MAX_TOKENS + 1
    st = m.moe_permute_static(cfg, T, 256, None, 256, 256, 256, None, stream=0, raise_on_error=False)
    assert st == m.MOE_ERR_UNSUPPORTED
