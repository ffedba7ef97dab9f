"""Expert parallelism on one GPU: moe_gather_rows bit-exact against the
permutation, the expert-parallel layer (CudaEPOps: shard of the experts with
top_k 1 over received rows, shared expert alone, pairs combine) against the
oracle at one rank, and at 2 and 4 ranks emulated by threads of one process
whose all-to-all is a host-side copy between their tensors (no kernel waits
on another rank's)."""
import threading

import numpy as np
import pytest

import gen
import oracle
from gpu_util import row_rel_err

pytestmark = pytest.mark.gpu


def _x(lay, tokens=None):
    import torch
    x = lay["x"] if tokens is None else lay["x"][tokens]
    return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()


def _ep_run(lay, world, T_per_rank, check_tokens_per_rank):
    """Runs `world` ranks (threads) of the expert-parallel layer over the
    layer's tokens, T_per_rank each; returns the worst row-relative error
    over the checked tokens and the ranks' layers."""
    import torch
    from bit_dequant_expert_b200 import ep
    E = lay["w_router"].shape[0]
    bar = threading.Barrier(world)
    slots = [None] * world

    def exchange_for(rank):
        def a2a(out, inp, out_splits, in_splits):
            torch.cuda.synchronize()
            slots[rank] = (inp, in_splits)
            bar.wait()
            pos = 0
            for s in range(world):
                inp_s, spl = slots[s]
                start, n = sum(spl[:rank]), spl[rank]
                assert n == out_splits[s]
                out[pos:pos + n].copy_(inp_s[start:start + n])
                pos += n
            torch.cuda.synchronize()
            bar.wait()
        return a2a

    layers, outs, errors = [None] * world, [None] * world, []

    def rank_main(rank):
        try:
            ops = ep.CudaEPOps(ep.shard_weights(lay, world, rank), E, world, max_tokens=T_per_rank)
            L = ep.ExpertParallelLayer(ops, E=E, world=world, rank=rank,
                                       exchange=exchange_for(rank) if world > 1 else None)
            toks = np.arange(rank * T_per_rank, (rank + 1) * T_per_rank)
            outs[rank] = L.forward(_x(lay, toks)).float().cpu().numpy().astype(np.float64)
            torch.cuda.synchronize()
            assert ops.device_errors() == [0, 0, 0]
            layers[rank] = L
        except BaseException as exc:   # surfaced below; the barrier is broken so no rank waits forever
            errors.append(exc)
            bar.abort()

    threads = [threading.Thread(target=rank_main, args=(r,)) for r in range(world)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(600)
    if errors:
        raise errors[0]
    worst = 0.0
    rng = np.random.default_rng(7)
    for rank in range(world):
        n = min(check_tokens_per_rank, T_per_rank)
        local = np.sort(rng.choice(T_per_rank, size=n, replace=False))
        toks = (rank * T_per_rank + local).astype(np.int32)
        y_ref, _, _ = oracle.layer(lay, tokens=toks)
        worst = max(worst, float(row_rel_err(outs[rank][local], y_ref).max()))
    return worst, layers


def test_gather_rows_bitexact_and_bounds():
    import torch
    import bit_dequant_expert_b200 as m
    from bit_dequant_expert_b200.layer import MoELayer, to_device
    lay = gen.make_layer(gen.config(3).with_T(300))
    L = MoELayer(lay, max_tokens=300, device="cuda")
    x = to_device(lay["x"], "cuda")
    L.route(x, 300)
    L.permute(300)
    r2p = L.row_to_pair.cpu().numpy()
    w = L.topk_w.cpu().numpy().reshape(-1)
    xb = lay["x"]
    for begin, n in ((0, 2400), (517, 1000), (2399, 1)):
        rows = torch.full((n, 2048), 7.0, dtype=torch.bfloat16, device="cuda")
        wo = torch.full((n,), -1.0, dtype=torch.float32, device="cuda")
        m.moe_gather_rows(L.cfg, 300, x, L.row_to_pair, L.topk_w, begin, n, rows, wo, L.ws)
        got = rows.view(torch.int16).cpu().numpy().view(np.uint16)
        p = r2p[begin:begin + n]
        assert np.array_equal(got, xb[p // 8])
        assert np.array_equal(wo.cpu().numpy(), w[p])
    assert m.moe_get_device_error(L.ws) == m.MOE_OK
    # a pair index out of range: its row comes back zero and the error word says so
    bad = L.row_to_pair.clone()
    bad[3] = 300 * 8
    rows = torch.full((8, 2048), 7.0, dtype=torch.bfloat16, device="cuda")
    m.moe_gather_rows(L.cfg, 300, x, bad, None, 0, 8, rows, None, L.ws)
    got = rows.view(torch.int16).cpu().numpy().view(np.uint16)
    assert not got[3].any() and np.array_equal(got[4], xb[r2p[4] // 8])
    assert m.moe_get_device_error(L.ws) == m.MOE_ERR_BOUNDS
    # host checks: the block must lie inside the permutation
    assert m.moe_gather_rows(L.cfg, 300, x, L.row_to_pair, None, 2000, 401, rows, None, L.ws,
                             raise_on_error=False) == m.MOE_ERR_INVALID_ARG
    assert m.moe_gather_rows(L.cfg, 300, x, L.row_to_pair, None, 0, 0, None, None, L.ws,
                             raise_on_error=False) == m.MOE_OK


@pytest.mark.parametrize("cfg_i,T,check", [(0, 8, 8), (3, 2048, 48)])
def test_expert_parallel_one_rank_matches_oracle(cfg_i, T, check):
    lay = gen.make_layer(gen.config(cfg_i).with_T(T))
    worst, layers = _ep_run(lay, 1, T, check)
    assert worst <= 1e-2, worst
    assert layers[0].last["send"] == [8 * T]


@pytest.mark.parametrize("cfg_i,world,T,check", [(0, 2, 8, 8), (3, 2, 512, 24), (3, 4, 256, 16)])
def test_expert_parallel_emulated_ranks_match_oracle(cfg_i, world, T, check):
    lay = gen.make_layer(gen.config(cfg_i).with_T(T * world))
    worst, layers = _ep_run(lay, world, T, check)
    assert worst <= 1e-2, worst
    for a in range(world):
        assert sum(layers[a].last["send"]) == 8 * T
        for b in range(world):
            assert layers[a].last["send"][b] == layers[b].last["recv"][a]


def test_expert_shard_call_with_top1_matches_oracle_rows():
    """The shard's grouped call alone: 128 local experts, every row its own
    token (top_k 1), rows interleaved so row_to_pair is not the identity;
    scatter mode gives w * expert(row) at each row's own position."""
    import torch
    import bit_dequant_expert_b200 as m
    from bit_dequant_expert_b200 import ep
    from bit_dequant_expert_b200.layer import to_device
    lay = gen.make_layer(gen.config(3).with_T(64))
    sh = ep.shard_weights(lay, 2, 1)            # experts 128..255, shared last
    rng = np.random.default_rng(3)
    counts = np.zeros((2, 128), dtype=np.int64)
    counts[:, rng.choice(128, 12, replace=False)] = rng.integers(1, 9, size=(2, 12))
    R = int(counts.sum())
    offsets, r2p = ep.local_rows(counts)
    xr = lay["x"][rng.integers(0, 64, size=R)]
    w = rng.uniform(0.05, 0.5, size=R).astype(np.float32)
    cfg = m.config(num_experts=128, top_k=1, has_shared=0)
    ws = torch.zeros(m.moe_workspace_size(cfg, R), dtype=torch.uint8, device="cuda")
    m.moe_workspace_init(ws)
    y = torch.empty(R, 2048, dtype=torch.float32, device="cuda")
    for path in (m.MOE_PATH_TC, m.MOE_PATH_SIMT):
        m.moe_expert_ffn_path(cfg, R, to_device(xr, "cuda"), to_device(sh["gu_codes"], "cuda"),
                              to_device(sh["gu_sb"], "cuda"), to_device(sh["d_codes"], "cuda"),
                              to_device(sh["d_sb"], "cuda"), to_device(offsets, "cuda"), to_device(r2p, "cuda"),
                              to_device(w, "cuda"), m.MOE_MODE_SCATTER, y, None, ws, path)
        got = y.cpu().numpy().astype(np.float64)
        assert m.moe_get_device_error(ws) == m.MOE_OK
        ref = np.empty_like(got)
        for e in range(128):
            rows = r2p[offsets[e]:offsets[e + 1]]
            if len(rows):
                ref[rows] = w[rows, None] * oracle.expert_rows(lay, 128 + e, xr[rows])
        assert row_rel_err(got, ref).max() <= 1e-2
