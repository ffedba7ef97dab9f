"""Expert parallelism for the MoE layer over N ranks, one process per GPU.

Rank q holds the routed experts [q E/N, (q+1) E/N), a replica of the shared
expert and a replica of the router.  One layer call on rank q, for its own
tokens x [T, H]:

  1. route + permute its tokens over all E experts (the four-call path's first
     two calls).  The permutation is expert-major, so the rows bound for rank
     d are the contiguous block offsets[d E/N] .. offsets[(d+1) E/N].
  2. exchange per-expert row counts (all-to-all of [N, E/N] integers), then
     gather the permuted rows with their routing weights (moe_gather_rows) and
     exchange them (all-to-all with those counts as splits).  Received rows sit
     in (source rank, local expert, row) order.
  3. run the local experts over the received rows in one grouped call: every
     row is its own token with one pair (top_k = 1), and row_to_pair maps the
     expert-major order of the call onto the received order, so nothing is
     moved; the scatter mode writes w * y of each row at its received position.
  4. send the weighted rows back (all-to-all with the splits reversed); they
     arrive in the sender's permuted row order.
  5. the shared expert over its own tokens, then the pairs combine with unit
     weights adds the returned rows of each token to it.

The pages describe one GPU (Lily runs on a single Mac, "Perplexity's Lily
brings fast local AI to Apple silicon Macs", "The Numbers and Their Test
Conditions"); this sharding follows the layer's structure: a token's eight
routed experts are independent until the weighted sum ("Perplexity built an
inference engine for one model, one chip", second paragraph).

The compute steps run through an `ops` object: `CudaEPOps` calls the CUDA
library; a test can substitute another implementation of the same five
methods to check the exchange logic here on CPU ranks.  Collectives go
through torch.distributed (NCCL on GPUs); tensors cross as 32-bit words.
"""
from __future__ import annotations

import numpy as np
import torch

__all__ = ["expert_range", "shard_weights", "send_splits", "local_rows", "ExpertParallelLayer", "CudaEPOps"]


def expert_range(E: int, world: int, rank: int) -> tuple[int, int]:
    """[lo, hi) of the routed experts rank `rank` holds; E must divide evenly."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank %d of %d" % (rank, world))
    if E % world:
        raise ValueError("%d experts do not split evenly over %d ranks" % (E, world))
    n = E // world
    return rank * n, (rank + 1) * n


def shard_weights(weights: dict, world: int, rank: int) -> dict:
    """This rank's packed expert matrices: its routed experts in order, then
    the shared expert (index E of the full arrays) last; the router is kept
    whole."""
    E = int(weights["w_router"].shape[0])
    lo, hi = expert_range(E, world, rank)
    keep = list(range(lo, hi)) + [E]
    out = {"w_router": weights["w_router"]}
    for name in ("gu_codes", "gu_sb", "d_codes", "d_sb"):
        a = weights[name]
        out[name] = np.ascontiguousarray(a[keep]) if isinstance(a, np.ndarray) else a[keep].contiguous()
    return out


def send_splits(counts: np.ndarray, world: int) -> list[int]:
    """Rows this rank sends to each rank: its per-expert counts summed over
    each rank's block of experts."""
    counts = np.asarray(counts, dtype=np.int64)
    return [int(v) for v in counts.reshape(world, -1).sum(axis=1)]


def local_rows(recv_counts: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """(offsets [El+1], row_to_pair [R]) of the grouped call over received rows.

    recv_counts [N, El]: rows of each local expert received from each rank.
    Received rows are ordered (source, expert, row); the call's rows are
    ordered (expert, source, row), and row_to_pair[r] is the received
    position of call row r."""
    c = np.asarray(recv_counts, dtype=np.int64)
    N, El = c.shape
    per_src = c.sum(axis=1)
    src_start = np.concatenate([[0], np.cumsum(per_src)[:-1]])                      # [N]
    recv_start = src_start[:, None] + np.cumsum(c, axis=1) - c                       # [N, El]: chunk (s, e)
    lengths = c.T.reshape(-1)                                                        # chunks in (e, s) order
    starts = recv_start.T.reshape(-1)
    call_start = np.cumsum(lengths) - lengths
    R = int(lengths.sum())
    r2p = np.repeat(starts - call_start, lengths) + np.arange(R, dtype=np.int64)
    per_expert = c.sum(axis=0)
    offsets = np.concatenate([[0], np.cumsum(per_expert)])
    return offsets.astype(np.int32), r2p.astype(np.int32)


def _words(t: torch.Tensor) -> torch.Tensor:
    """bf16 [n, H] rows as int32 [n, H/2] words (the collectives' element type)."""
    return t.view(torch.int32)


class ExpertParallelLayer:
    """One MoE layer sharded by experts over the ranks of `group`.

    ops: the compute backend (CudaEPOps for this rank's GPU).  E routed
    experts in total, top 8, shared expert replicated.  forward(x) takes this
    rank's tokens and returns their layer output; every rank of the group must
    call it the same number of times (the exchanges are collective)."""

    def __init__(self, ops, E: int = 256, top_k: int = 8, group=None, world=None, rank=None, exchange=None):
        import torch.distributed as dist
        self.ops, self.E, self.K, self.group = ops, E, top_k, group
        on = dist.is_available() and dist.is_initialized()
        self.world = world if world is not None else (dist.get_world_size(group) if on else 1)
        self.rank = rank if rank is not None else (dist.get_rank(group) if on else 0)
        self.exchange = exchange   # optional all-to-all stand-in: (out, inp, out_splits, in_splits)
        self.lo, self.hi = expert_range(E, self.world, self.rank)
        self.El = self.hi - self.lo
        self.last = {}   # bookkeeping of the last call, for tests and the bench

    def _a2a(self, out: torch.Tensor, inp: torch.Tensor, out_splits, in_splits) -> None:
        if self.exchange is not None:
            self.exchange(out, inp, list(out_splits), list(in_splits))
            return
        if self.world == 1:
            out.copy_(inp)
            return
        import torch.distributed as dist
        dist.all_to_all_single(out, inp, list(out_splits), list(in_splits), group=self.group)

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        ops, K, N, El = self.ops, self.K, self.world, self.El
        T, H = int(x.shape[0]), int(x.shape[1])
        dev = x.device
        r = ops.route(x)
        counts = r["counts"].to("cpu", torch.int64).numpy()
        send = send_splits(counts, N)
        # 2. per-expert counts, then the rows and their weights
        cnt_out = r["counts"].to(torch.int32).contiguous()
        cnt_in = torch.empty(N * El, dtype=torch.int32, device=cnt_out.device)
        self._a2a(cnt_in, cnt_out, [El] * N, [El] * N)
        recv_counts = cnt_in.to("cpu", torch.int64).numpy().reshape(N, El)
        recv = [int(v) for v in recv_counts.sum(axis=1)]
        R = sum(recv)
        xs, ws = ops.gather(x, r, 0, T * K)
        xr = torch.empty(R, H, dtype=torch.bfloat16, device=dev)
        wr = torch.empty(R, dtype=torch.float32, device=dev)
        self._a2a(_words(xr), _words(xs), recv, send)
        self._a2a(wr, ws, recv, send)
        # 3. the local experts over the received rows
        offsets, r2p = local_rows(recv_counts)
        yl = ops.experts(xr, offsets, r2p, wr, recv_counts)
        # 4. back to the senders, in their permuted row order
        yr = torch.empty(T * K, H, dtype=torch.bfloat16, device=dev)
        self._a2a(_words(yr), _words(yl), send, recv)
        # 5. shared expert + the returned rows of each token
        ys = ops.shared(x)
        self.last = {"send": send, "recv": recv, "recv_counts": recv_counts, "offsets": offsets, "row_to_pair": r2p}
        return ops.combine(yr, ys, r)


class CudaEPOps:
    """The five compute steps of ExpertParallelLayer on this rank's GPU,
    through the CUDA library: route/permute/gather/combine with the full
    configuration (E experts, top 8, shared), the local experts with E/N
    experts and top_k 1, the shared expert as a call with no routed rows."""

    def __init__(self, weights_local: dict, E: int, world: int, max_tokens: int, device="cuda"):
        from . import config, moe_workspace_init, moe_workspace_size
        from .layer import to_device
        El = int(weights_local["gu_codes"].shape[0]) - 1
        if El * world != E:
            raise ValueError("shard holds %d experts, expected %d / %d" % (El, E, world))
        if not 1 <= max_tokens <= 8192:
            raise ValueError("max_tokens must be in 1..8192 (a source rank's rows fill one expert call)")
        H = int(weights_local["gu_codes"].shape[2]) * 8
        I = int(weights_local["gu_codes"].shape[1]) // 2
        if tuple(weights_local["w_router"].shape) != (E, H):
            raise ValueError("w_router must be [%d, %d]" % (E, H))
        full = weights_local
        self.dev = torch.device(device)
        self.H, self.I, self.E, self.El, self.T_max = H, I, E, El, max_tokens
        self.cfg = config(hidden=H, inter=I, num_experts=E, top_k=8, has_shared=1)
        self.cfg_loc = config(hidden=H, inter=I, num_experts=El, top_k=1, has_shared=0)
        self.cfg_sh = config(hidden=H, inter=I, num_experts=El, top_k=1, has_shared=1)
        self.w_router = to_device(full["w_router"], self.dev)
        self.gu_codes = to_device(full["gu_codes"], self.dev)
        self.gu_sb = to_device(full["gu_sb"], self.dev)
        self.d_codes = to_device(full["d_codes"], self.dev)
        self.d_sb = to_device(full["d_sb"], self.dev)
        # the received rows of one call: at most every pair of every rank
        self.R_max = min(65536, 8 * max_tokens * world)
        self.ws = torch.zeros(moe_workspace_size(self.cfg, max_tokens), dtype=torch.uint8, device=self.dev)
        self.ws_loc = torch.zeros(moe_workspace_size(self.cfg_loc, self.R_max), dtype=torch.uint8, device=self.dev)
        self.ws_sh = torch.zeros(moe_workspace_size(self.cfg_sh, max_tokens), dtype=torch.uint8, device=self.dev)
        for w in (self.ws, self.ws_loc, self.ws_sh):
            if w.numel() == 0:
                raise ValueError("unsupported layer configuration")
            moe_workspace_init(w)
        T, dev = max_tokens, self.dev
        self.topk_idx = torch.empty(T, 8, dtype=torch.int32, device=dev)
        self.topk_w = torch.empty(T, 8, dtype=torch.float32, device=dev)
        self.counts = torch.empty(E, dtype=torch.int32, device=dev)
        self.offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
        self.row_to_pair = torch.empty(T * 8, dtype=torch.int32, device=dev)
        self.pair_to_row = torch.empty(T * 8, dtype=torch.int32, device=dev)
        self.ones = torch.ones(T * 8, dtype=torch.float32, device=dev)
        self.sh_offsets = torch.zeros(El + 1, dtype=torch.int32, device=dev)
        self.sh_dummy_i = torch.zeros(T, dtype=torch.int32, device=dev)
        self.sh_dummy_w = torch.zeros(T, dtype=torch.float32, device=dev)
        self.sh_rows = torch.empty(T, H, dtype=torch.bfloat16, device=dev)

    def route(self, x):
        from . import moe_permute, moe_route
        T = x.shape[0]
        moe_route(self.cfg, T, x, self.w_router, None, None, 0, self.topk_idx, self.topk_w, self.counts, self.ws)
        moe_permute(self.cfg, T, self.topk_idx, self.counts, self.offsets, self.row_to_pair, self.pair_to_row,
                    self.ws)
        return {"counts": self.counts, "offsets": self.offsets, "row_to_pair": self.row_to_pair,
                "pair_to_row": self.pair_to_row, "topk_idx": self.topk_idx[:T], "topk_w": self.topk_w[:T], "T": T}

    def gather(self, x, r, begin, n):
        from . import moe_gather_rows
        rows = torch.empty(n, self.H, dtype=torch.bfloat16, device=self.dev)
        w = torch.empty(n, dtype=torch.float32, device=self.dev)
        moe_gather_rows(self.cfg, r["T"], x, self.row_to_pair, self.topk_w, begin, n, rows, w, self.ws)
        return rows, w

    def _experts_call(self, xr, offsets, r2p, wr, y_acc, yl):
        from . import MOE_MODE_SCATTER, moe_combine, moe_expert_ffn
        R = xr.shape[0]
        d_off = torch.from_numpy(offsets).to(self.dev)
        d_r2p = torch.from_numpy(r2p).to(self.dev)
        moe_expert_ffn(self.cfg_loc, R, xr, self.gu_codes, self.gu_sb, self.d_codes, self.d_sb, d_off, d_r2p, wr,
                       MOE_MODE_SCATTER, y_acc, None, self.ws_loc)
        moe_combine(self.cfg_loc, R, MOE_MODE_SCATTER, y_acc, None, None, None, yl)

    def experts(self, xr, offsets, r2p, wr, recv_counts):
        R = int(xr.shape[0])
        yl = torch.empty(R, self.H, dtype=torch.bfloat16, device=self.dev)
        if R == 0:
            return yl
        if R <= self.R_max:
            y_acc = torch.empty(R, self.H, dtype=torch.float32, device=self.dev)
            self._experts_call(xr, offsets, r2p, wr, y_acc, yl)
            return yl
        # more rows than one call takes: one call per source rank's block (each <= 8 T_max rows)
        start = 0
        for c in np.asarray(recv_counts):
            n = int(c.sum())
            if n:
                off = np.concatenate([[0], np.cumsum(c)]).astype(np.int32)
                y_acc = torch.empty(n, self.H, dtype=torch.float32, device=self.dev)
                self._experts_call(xr[start:start + n], off, np.arange(n, dtype=np.int32), wr[start:start + n],
                                   y_acc, yl[start:start + n])
            start += n
        return yl

    def shared(self, x):
        from . import MOE_MODE_PAIRS, moe_expert_ffn
        T = x.shape[0]
        ys = torch.empty(T, self.H, dtype=torch.bfloat16, device=self.dev)
        moe_expert_ffn(self.cfg_sh, T, x, self.gu_codes, self.gu_sb, self.d_codes, self.d_sb, self.sh_offsets,
                       self.sh_dummy_i, self.sh_dummy_w, MOE_MODE_PAIRS, self.sh_rows, ys, self.ws_sh)
        return ys

    def combine(self, yr, ys, r):
        from . import MOE_MODE_PAIRS, moe_combine
        T = r["T"]
        y = torch.empty(T, self.H, dtype=torch.bfloat16, device=self.dev)
        moe_combine(self.cfg, T, MOE_MODE_PAIRS, yr, ys, self.pair_to_row, self.ones, y)
        return y

    def device_errors(self) -> list[int]:
        from . import moe_get_device_error
        return [moe_get_device_error(w) for w in (self.ws, self.ws_loc, self.ws_sh)]
