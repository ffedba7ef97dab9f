"""gdn_scan (the register-resident Gated DeltaNet scan) against the CPU
oracle, element by element.

Tolerances, from the arithmetic: the kernel works in fp32 and rounds o to
bf16.  o: each [dv] output vector within 1e-2 of its largest oracle element
(bf16 rounding is 2^-9 relative; the rest is fp32 drift).  State: within
1e-3 of the head's largest oracle element; fp32 rounding of 128-term dot
products adds ~sqrt(128) * 2^-24 relative per token, and the update
S (a (I - beta k k^T)) with a <= 1, ||k|| = 1, beta in (0, 1) does not
amplify earlier errors, so after T = 2048 tokens the expected drift is
~sqrt(2048 * 128) * 6e-8 = 3e-5: the bound leaves a 30x margin."""
import numpy as np
import pytest

import gen
import oracle.gdn as G

pytestmark = pytest.mark.gpu

O_TOL = 1e-2
S_TOL = 1e-3


def _dev(a):
    import torch
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(a).cuda()


def _run(d, in_place=False):
    import torch
    import bit_dequant_expert_b200 as m
    B, T, Hk, dk = d["q"].shape
    Hv, dv = d["v"].shape[2], d["v"].shape[3]
    q, k, v, g, beta = (_dev(d[n]) for n in ("q", "k", "v", "g", "beta"))
    s_in = _dev(d["S0"])
    s_out = s_in if in_place else torch.full_like(s_in, float("nan"))
    o = torch.full((B, T, Hv, dv), float("nan"), dtype=torch.bfloat16, device="cuda")
    m.gdn_scan(B, T, Hk, Hv, dk, dv, q, k, v, g, beta, d["scale"], s_in, s_out, o)
    torch.cuda.synchronize()
    return o.float().cpu().numpy().astype(np.float64), s_out.cpu().numpy().astype(np.float64)


def _check(d, o, S):
    o_ref, S_ref = G.scan(d["q"], d["k"], d["v"], d["g"], d["beta"], d["scale"], d["S0"])
    assert np.isfinite(o).all() and np.isfinite(S).all()
    o_err = np.abs(o - o_ref).max(axis=-1) / np.abs(o_ref).max(axis=-1)
    s_err = np.abs(S - S_ref).max(axis=(-2, -1)) / np.abs(S_ref).max(axis=(-2, -1))
    assert o_err.max() <= O_TOL, o_err.max()
    assert s_err.max() <= S_TOL, s_err.max()
    return o_err.max(), s_err.max()


@pytest.mark.parametrize("cfg_i,B,T", [
    (0, None, None),          # tiny, T = 17: one whole chunk of 16 tokens and a ragged tail
    (0, 1, 1), (0, 3, 16), (0, 2, 33),
    (1, 8, 1),                # decode: 8 sequences, one token, 16 key / 32 value heads
    (1, 8, 4), (1, 5, 16),    # enough (sequence, head, row block) items for the item-walking kernel
    (2, None, None),          # verification: one sequence, 4 tokens
    (3, None, None),          # prefill: one sequence of 2048 tokens
])
def test_gdn_scan_matches_oracle(cfg_i, B, T):
    spec = gen.scan_config(cfg_i)
    if B is not None:
        spec = spec.with_B(B).with_T(T)
    d = gen.make_scan(spec)
    o, S = _run(d)
    _check(d, o, S)


def test_gdn_scan_in_place_state_and_chained_calls():
    """state_out may be state_in; two calls of 9 then 8 tokens equal one call
    of 17 (the state carries everything between calls)."""
    import torch
    import bit_dequant_expert_b200 as m
    d = gen.make_scan(gen.scan_config(0))
    o_full, S_full = _run(d)
    _check(d, o_full, S_full)
    B, T, Hk, dk = d["q"].shape
    Hv, dv = d["v"].shape[2], d["v"].shape[3]
    state = _dev(d["S0"])
    outs = []
    for lo, hi in ((0, 9), (9, 17)):
        part = {n: np.ascontiguousarray(d[n][:, lo:hi]) for n in ("q", "k", "v", "g", "beta")}
        o = torch.empty((B, hi - lo, Hv, dv), dtype=torch.bfloat16, device="cuda")
        m.gdn_scan(B, hi - lo, Hk, Hv, dk, dv, *(_dev(part[n]) for n in ("q", "k", "v", "g", "beta")),
                   d["scale"], state, state, o)
        outs.append(o.float().cpu().numpy())
    torch.cuda.synchronize()
    o_two = np.concatenate(outs, axis=1).astype(np.float64)
    _check(d, o_two, state.cpu().numpy().astype(np.float64))
    # the split changes nothing: same arithmetic in the same order
    assert np.array_equal(o_two, o_full)


def test_gdn_scan_edge_values():
    """beta = 0 (nothing written) and g = 0 (no decay): the state comes back
    bit-identical, and o is scale * S0 q."""
    spec = gen.scan_config(0)
    d = gen.make_scan(spec)
    d["beta"] = np.zeros_like(d["beta"])
    d["g"] = np.zeros_like(d["g"])
    o, S = _run(d)
    assert np.array_equal(S, d["S0"].astype(np.float64))
    _check(d, o, S)


def test_gdn_scan_item_walk_in_place():
    """Decode shape (every CTA walks several items, prefetching the next
    one's state): state_out may be state_in."""
    d = gen.make_scan(gen.scan_config(1).with_B(7).with_T(2))
    o, S = _run(d, in_place=True)
    _check(d, o, S)
