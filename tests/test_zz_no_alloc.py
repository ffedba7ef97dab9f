"""moe_permute_static, the entry point for callers that cannot allocate
device memory (a plugin whose host runtime owns every device allocation, a
real-time path that may not call cudaMalloc): it must give exactly the
results of moe_permute, call after call, with its scratch in the library's
fixed device array.  Collected last so a failure here comes after every
other test has run."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def _routing(T, seed):
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.permutation(256)[:8] for _ in range(T)]).astype(np.int32)
    idx[: T // 3] = np.arange(8, 16)          # a skewed share, so counts are uneven
    return idx


def _permute_both(m, cfg, idx):
    import torch
    T = idx.shape[0]
    d_idx = torch.from_numpy(idx).cuda()
    d_cnt = torch.from_numpy(np.bincount(idx.ravel(), minlength=256).astype(np.int32)).cuda()
    ws = torch.zeros(m.moe_workspace_size(cfg, T), dtype=torch.uint8, device="cuda")
    ref = [torch.empty(n, dtype=torch.int32, device="cuda") for n in (257, T * 8, T * 8)]
    m.moe_permute(cfg, T, d_idx, d_cnt, ref[0], ref[1], ref[2], ws)
    assert m.moe_get_device_error(ws) == m.MOE_OK
    outs = []
    for _ in range(2):                          # two calls in a row share the static scratch
        got = [torch.full((n,), -7, dtype=torch.int32, device="cuda") for n in (257, T * 8, T * 8)]
        err = torch.full((1,), 99, dtype=torch.int32, device="cuda")
        m.moe_permute_static(cfg, T, d_idx, d_cnt, got[0], got[1], got[2], err)
        torch.cuda.synchronize()
        assert int(err.item()) == m.MOE_OK
        outs.append([g.cpu().numpy() for g in got])
    return [r.cpu().numpy() for r in ref], outs


@pytest.mark.parametrize("T,seed", [(4097, 1), (1000, 2), (16384, 3)])
def test_permute_static_matches_moe_permute(T, seed):
    import bit_dequant_expert_b200 as m
    cfg = m.config()
    ref, outs = _permute_both(m, cfg, _routing(T, seed))
    for got in outs:
        for a, b in zip(got, ref):
            assert np.array_equal(a, b)


def test_permute_static_rejects_oversize():
    import bit_dequant_expert_b200 as m
    cfg = m.config()
    T = m.MOE_STATIC_MAX_TOKENS + 1
    st = m.moe_permute_static(cfg, T, 256, None, 256, 256, 256, None, stream=0, raise_on_error=False)
    assert st == m.MOE_ERR_UNSUPPORTED
