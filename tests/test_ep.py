"""Expert parallelism on CPU ranks: the exchange bookkeeping of
bit_dequant_expert_b200.ep (send splits, the received-row map, the two
all-to-alls and the return order) run over gloo with world sizes 2 and 4, its
compute steps done by the oracle; every rank's layer output must match the
oracle's single-process layer for the same tokens."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from bit_dequant_expert_b200 import ep  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _bf16(u16: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).view(torch.bfloat16)


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _round_bf16(f64: np.ndarray) -> torch.Tensor:
    import gen
    return _bf16(gen.f32_to_bf16_bits(np.asarray(f64, dtype=np.float32)))


class OracleOps:
    """The five compute steps of one rank, by the oracle, on CPU tensors."""

    def __init__(self, lay: dict, world: int, rank: int):
        self.lay, self.E = lay, lay["w_router"].shape[0]
        self.lo, self.hi = ep.expert_range(self.E, world, rank)

    def route(self, x):
        import oracle
        xb = _bits(x)
        logits = oracle.router_logits(xb, self.lay["w_router"])
        idx, w = oracle.select(logits, 8)
        counts, offsets, r2p, p2r = oracle.permute(idx, self.E)
        return {"counts": torch.from_numpy(counts.astype(np.int32)), "offsets": offsets, "row_to_pair": r2p,
                "pair_to_row": p2r, "topk_w": w.astype(np.float32).reshape(-1), "T": xb.shape[0]}

    def gather(self, x, r, begin, n):
        p = r["row_to_pair"][begin:begin + n]
        return x[torch.from_numpy(p // 8).long()].contiguous(), torch.from_numpy(r["topk_w"][p])

    def experts(self, xr, offsets, r2p, wr, recv_counts):
        import oracle
        xb, w = _bits(xr), wr.numpy()
        out = np.zeros((xb.shape[0], xb.shape[1]), dtype=np.float64)
        for e in range(self.hi - self.lo):
            rows = r2p[offsets[e]:offsets[e + 1]]
            if len(rows):
                out[rows] = w[rows, None] * oracle.expert_rows(self.lay, self.lo + e, xb[rows])
        return _round_bf16(out)

    def shared(self, x):
        import oracle
        return _round_bf16(oracle.expert_rows(self.lay, self.E, _bits(x)))

    def combine(self, yr, ys, r):
        rows = yr.float().numpy().astype(np.float64)[r["pair_to_row"]].reshape(r["T"], 8, -1)
        return rows.sum(axis=1) + ys.float().numpy()


def _rank_main(rank, world, port, T_per_rank, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import gen
    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        spec = gen.config(0).with_T(T_per_rank * world)
        lay = gen.make_layer(spec)
        mine = np.arange(rank * T_per_rank, (rank + 1) * T_per_rank)
        layer = ep.ExpertParallelLayer(OracleOps(lay, world, rank), E=256)
        y = layer.forward(_bf16(lay["x"][mine]))
        y_ref, _, _ = oracle.layer(lay, tokens=mine.astype(np.int32))
        rel = np.abs(y - y_ref).max(axis=1) / np.abs(y_ref).max(axis=1)
        out[rank] = (float(rel.max()), layer.last["send"], layer.last["recv"])
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,T", [(2, 8), (4, 5)])
def test_expert_parallel_layer_matches_oracle(world, T):
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, T, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(300)
        codes = [p.exitcode for p in procs]
        res = dict(out)
    assert codes == [0] * world, codes
    for r in range(world):
        rel, send, recv = res[r]
        assert rel <= 1e-2, (r, rel)
        assert sum(send) == 8 * T   # every pair of the rank's tokens leaves once
    # what rank a sent to rank b is what rank b received from rank a
    for a in range(world):
        for b in range(world):
            assert res[a][1][b] == res[b][2][a]


def _local_rows_brute(c):
    N, El = c.shape
    starts, pos = {}, 0
    for s in range(N):
        for e in range(El):
            starts[(s, e)] = pos
            pos += c[s, e]
    r2p, offsets = [], [0]
    for e in range(El):
        for s in range(N):
            r2p += list(range(starts[(s, e)], starts[(s, e)] + c[s, e]))
        offsets.append(len(r2p))
    return np.array(offsets), np.array(r2p, dtype=np.int64)


@pytest.mark.parametrize("N,El,seed", [(2, 128, 0), (4, 64, 1), (8, 32, 2), (3, 5, 3), (1, 256, 4)])
def test_local_rows_brute_force(N, El, seed):
    rng = np.random.default_rng(seed)
    c = rng.integers(0, 6, size=(N, El))
    c[rng.random((N, El)) < 0.3] = 0        # experts some ranks send nothing to
    off, r2p = ep.local_rows(c)
    off_b, r2p_b = _local_rows_brute(c)
    assert np.array_equal(off, off_b) and np.array_equal(r2p, r2p_b)
    assert np.array_equal(np.sort(r2p), np.arange(c.sum()))   # a permutation of the received rows


def test_local_rows_empty_and_send_splits():
    off, r2p = ep.local_rows(np.zeros((2, 4), dtype=np.int64))
    assert off.tolist() == [0] * 5 and r2p.size == 0
    counts = np.arange(8)
    assert ep.send_splits(counts, 2) == [0 + 1 + 2 + 3, 4 + 5 + 6 + 7]
    assert ep.send_splits(counts, 1) == [28]


def test_expert_range_and_shard():
    assert ep.expert_range(256, 4, 3) == (192, 256)
    with pytest.raises(ValueError):
        ep.expert_range(256, 3, 0)
    w = {"w_router": np.zeros((8, 2)), "gu_codes": np.arange(9)[:, None], "gu_sb": np.arange(9)[:, None],
         "d_codes": np.arange(9)[:, None], "d_sb": np.arange(9)[:, None]}
    s = ep.shard_weights(w, 2, 1)
    assert s["gu_codes"][:, 0].tolist() == [4, 5, 6, 7, 8]   # experts 4..7, then the shared one (index 8)
