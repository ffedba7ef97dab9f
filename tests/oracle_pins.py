"""Checks that pin the CPU oracle to facts other than itself.

Every check takes a loaded oracle library (so the mutation tests can run the
same checks against deliberately broken copies) and raises AssertionError on
a mismatch.  The facts come from hand-worked fixtures under tests/golden/,
closed forms of special layers, brute force on tiny inputs, and invariants of
the definitions on the Lily pages ("A 35B Model Built for Local Memory":
256 experts, 8 selected, groupwise affine 4-bit weights; "Perplexity built an
inference engine for one model, one chip", second paragraph: one shared
expert sees every token).
"""
from __future__ import annotations

import math
import os

import numpy as np

import gen
import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line.split()


def bf16_bits(v: float) -> int:
    """bf16 bit pattern of a value that bf16 represents exactly."""
    b = int(gen.f32_to_bf16_bits(np.array([v], dtype=np.float32))[0])
    assert float(gen.bf16_to_f32(np.array([b], dtype=np.uint16))[0]) == v, v
    return b


# ----------------------------------------------------------------- dequant


def check_dequant_golden(L):
    K, G = 128, 64
    for s, b, q, want in _rows("dequant_cases.txt"):
        s, b, q, want = float(s), float(b), int(q), float(want)
        for n in (0, 2):            # a later row: row offsets of codes and (scale, bias)
            for k in (q % 8, 64 + 8 + 3, 127):   # group 0 and group 1, several nibble slots
                codes = np.zeros((3, K // 8), dtype=np.uint32)
                sb = np.zeros((3, K // G, 2), dtype=np.uint16)
                # fill every other group and row with a decoy (scale 1, bias 100)
                sb[:, :, 0] = bf16_bits(1.0)
                sb[:, :, 1] = bf16_bits(100.0)
                codes[:] = 0x99999999
                codes[n, k // 8] = (0x99999999 & ~(0xF << (4 * (k % 8)))) | (q << (4 * (k % 8)))
                sb[n, k // G] = (bf16_bits(s), bf16_bits(b))
                got = oracle.dequant_one(codes, sb, K, G, n, k, L=L)
                assert got == want, (s, b, q, n, k, got, want)


def check_nibble_order(L):
    for word, k, want in _rows("nibble_cases.txt"):
        row = np.array([int(word, 16), 0], dtype=np.uint32)
        got = oracle.code(row, int(k), L=L)
        assert got == int(want), (word, k, got, want)
    # word index: input k = 8m + j lives in word m
    row = np.array([0x0, 0x00000050, 0x0], dtype=np.uint32)
    assert oracle.code(row, 8, L=L) == 0 and oracle.code(row, 9, L=L) == 5
    assert oracle.code(row, 1, L=L) == 0 and oracle.code(row, 17, L=L) == 0


def check_dequant_matrix_affine(L):
    """Matrix decode agrees with codes placed one at a time (q -> s*q + b)."""
    rng = np.random.default_rng(5)
    N, K, G = 4, 128, 64
    q = rng.integers(0, 16, size=(N, K))
    codes = np.zeros((N, K // 8), dtype=np.uint32)
    for n in range(N):
        for k in range(K):
            codes[n, k // 8] |= np.uint32(int(q[n, k]) << (4 * (k % 8)))
    scales = [0.5, 0.25, 2.0, 0.125, 1.0, 4.0, 0.0625, 8.0]
    sb = np.zeros((N, K // G, 2), dtype=np.uint16)
    for n in range(N):
        for g in range(K // G):
            s = scales[(n * 2 + g) % 8]
            sb[n, g] = (bf16_bits(s), bf16_bits(-3.0 * s))
    W = oracle.dequant_matrix(codes, sb, N, K, G, L=L)
    for n in range(N):
        for k in range(K):
            s = scales[(n * 2 + k // G) % 8]
            assert W[n, k] == s * q[n, k] - 3.0 * s, (n, k)


# ------------------------------------------------------------- router order


def check_router_order_golden(L):
    H, E = 512, 3
    for name, want, bias, *prods in _rows("router_order_cases.txt"):
        x = np.zeros((1, H), dtype=np.uint16)
        wr = np.zeros((E, H), dtype=np.uint16)
        for p in prods:
            h, xv, wv = p.split(":")
            x[0, int(h)] = bf16_bits(float(xv))
            wr[1, int(h)] = bf16_bits(float(wv))   # expert 1; experts 0 and 2 stay zero
        b = np.array([0.0, float(bias), 0.0], dtype=np.float32)
        got = oracle.router_logits(x, wr, bias=b, bias_stride=0, L=L)
        assert got[0, 1] == np.float32(want), (name, got[0, 1], want)
        assert got[0, 0] == 0.0 and got[0, 2] == 0.0, name


def check_router_error_bound(L):
    """fp32 contract-order logits stay within the textbook bound of the exact sum.

    Each slice sums H/32 exact products with one rounding per step, then 5
    butterfly levels: |l32 - l_exact| <= (H/32 + 5) * 2^-24 * sum |x w|.
    """
    rng = np.random.default_rng(11)
    T, H, E = 5, 2048, 16
    x = gen.f32_to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    wr = gen.f32_to_bf16_bits((0.02 * rng.standard_normal((E, H))).astype(np.float32))
    xf = gen.bf16_to_f32(x).astype(np.float64)
    wf = gen.bf16_to_f32(wr).astype(np.float64)
    got = oracle.router_logits(x, wr, L=L)
    for t in range(T):
        for e in range(E):
            prods = xf[t] * wf[e]            # exact in fp64 (8-bit x 8-bit significands)
            exact = math.fsum(prods)
            bound = (H / 32 + 5) * 2.0 ** -24 * np.abs(prods).sum()
            assert abs(float(got[t, e]) - exact) <= bound, (t, e, got[t, e], exact)
    # a per-token bias row is added to its own token
    bias = rng.standard_normal((T, E)).astype(np.float32)
    gotb = oracle.router_logits(x, wr, bias=bias, bias_stride=E, L=L)
    assert np.array_equal(gotb, (got + bias).astype(np.float32))
    # selected tokens give the same rows as the full batch
    sub = oracle.router_logits(x, wr, bias=bias, bias_stride=E, tokens=np.array([3, 1]), L=L)
    assert np.array_equal(sub, gotb[[3, 1]])


def check_router_subnormal(L):
    """Subnormal products and partial sums are kept, not flushed to zero.

    With x_h = 2^-70 (1 + (h mod 128)/128) and w_h = 2^-70 over H = 256
    inputs, every product 2^-140 (1 + (h mod 128)/128) is an exact fp32
    subnormal, every partial sum stays an exact multiple of 2^-149 below
    2^-126, and the logit is sum_h of them = 383 * 2^-140 exactly; a flush of
    subnormals to zero anywhere would give 0.
    """
    H, E = 256, 2
    x = np.array([[bf16_bits(2.0 ** -70 * (1 + (h % 128) / 128)) for h in range(H)]], dtype=np.uint16)
    wr = np.zeros((E, H), dtype=np.uint16)
    wr[1, :] = bf16_bits(2.0 ** -70)
    got = oracle.router_logits(x, wr, L=L)
    want = np.float32(383 * 2.0 ** -140)
    assert 0 < want < np.float32(2.0 ** -126)
    assert got[0, 1] == want, (got[0, 1], want)
    assert got[0, 0] == 0.0


# ---------------------------------------------------------------- selection


def _brute_topk(row, k):
    order = sorted(range(len(row)), key=lambda e: (-float(row[e]), e))
    return order[:k]


def check_select_example(L):
    row = np.array([[0.5, 2, 2, -1, 2, 0, 1, 2]], dtype=np.float32)
    idx, w = oracle.select(row, 3, L=L)
    assert idx[0].tolist() == [1, 2, 4], idx
    assert abs(w[0].sum() - 1.0) < 1e-15 and np.allclose(w[0], 1.0 / 3.0, rtol=0, atol=1e-15)


def check_select_bruteforce(L):
    rng = np.random.default_rng(7)
    for trial in range(300):
        E = int(rng.integers(2, 13))
        k = int(rng.integers(1, min(4, E) + 1))
        n = 3
        if trial % 2:
            logits = rng.integers(0, 3, size=(n, E)).astype(np.float32)   # mass ties
        else:
            logits = rng.standard_normal((n, E)).astype(np.float32)
        idx, w = oracle.select(logits, k, L=L)
        for t in range(n):
            assert idx[t].tolist() == _brute_topk(logits[t], k), (logits[t], idx[t])
            # renormalised weights = softmax over the selected logits (fp64)
            sel = logits[t, idx[t]].astype(np.float64)
            ref = np.exp(sel - sel.max())
            ref /= ref.sum()
            assert np.allclose(w[t], ref, rtol=0, atol=1e-15), (w[t], ref)
            assert abs(w[t].sum() - 1.0) < 1e-15


def check_select_ties_and_zero(L):
    # all equal: indices 0..7 and weights exactly 1/8
    idx, w = oracle.select(np.zeros((1, 256), dtype=np.float32), 8, L=L)
    assert idx[0].tolist() == list(range(8)) and np.all(w[0] == 0.125)
    # -0.0 and +0.0 tie, lowest index wins whichever sign it carries
    for a, b in ((-0.0, 0.0), (0.0, -0.0)):
        row = np.full((1, 6), -1.0, dtype=np.float32)
        row[0, 2], row[0, 4] = a, b
        idx, _ = oracle.select(row, 2, L=L)
        assert idx[0].tolist() == [2, 4], (a, b, idx)
    # two levels: one logit ln2 above seven equal ones -> 2/9 and 1/9
    row = np.full((1, 256), -30.0, dtype=np.float32)
    row[0, 10:17] = 1.0
    row[0, 200] = np.float32(1.0 + math.log(2.0))
    idx, w = oracle.select(row, 8, L=L)
    assert idx[0].tolist() == [200] + list(range(10, 17))
    ratio = math.exp(float(row[0, 200]) - 1.0)     # exp of the fp32 gap, exactly as rounded
    assert abs(w[0, 0] - ratio / (ratio + 7)) < 1e-15
    assert np.allclose(w[0, 1:], 1.0 / (ratio + 7), rtol=0, atol=1e-15)


def check_select_nonfinite(L):
    for bad in (np.nan, np.inf, -np.inf):
        row = np.zeros((2, 16), dtype=np.float32)
        row[1, 5] = bad
        try:
            oracle.select(row, 4, L=L)
        except oracle.OracleError as err:
            assert err.code == oracle.ERR_NONFINITE
        else:
            raise AssertionError("non-finite logit accepted")


# ----------------------------------------------------------------- permute


def check_permute_invariants(L):
    rng = np.random.default_rng(3)
    for T, E, k in ((1, 256, 8), (37, 16, 4), (300, 256, 8), (64, 8, 8)):
        idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
        counts, offsets, r2p, p2r = oracle.permute(idx, E, L=L)
        assert counts.sum() == T * k
        assert np.array_equal(counts, np.bincount(idx.ravel(), minlength=E))
        assert offsets[0] == 0 and offsets[E] == T * k and np.all(np.diff(offsets) == counts)
        assert np.array_equal(np.sort(r2p), np.arange(T * k))
        assert np.array_equal(p2r[r2p], np.arange(T * k))
        # brute force: rows ordered by (expert, token)
        pairs = sorted(range(T * k), key=lambda p: (int(idx.ravel()[p]), p // k))
        assert r2p.tolist() == pairs
    # a token may not pick one expert twice, and indices must be in range
    for bad in (np.array([[1, 1]], dtype=np.int32), np.array([[0, 9]], dtype=np.int32)):
        try:
            oracle.permute(bad, 8, L=L)
        except oracle.OracleError as err:
            assert err.code == oracle.ERR_BOUNDS
        else:
            raise AssertionError("bad routing accepted")


# -------------------------------------------------------------- layer forms


def _probe_layer(T, H, I, E, G, rng, probes, down_val, bias_fill=None):
    """A layer whose experts are sparse probes.

    probes[e] = (j, k_gate, k_up, o): gate row j reads input k_gate with
    weight 1, up row I+j reads input k_up with weight 1, down row o reads h_j
    with weight down_val[e]; every other weight is 0 (scale 0, bias 0).
    """
    x = gen.f32_to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32) * 0.5)
    wr = gen.f32_to_bf16_bits((0.02 * rng.standard_normal((E, H))).astype(np.float32))
    gu_codes = np.zeros((E + 1, 2 * I, H // 8), dtype=np.uint32)
    gu_sb = np.zeros((E + 1, 2 * I, H // G, 2), dtype=np.uint16)
    d_codes = np.zeros((E + 1, H, I // 8), dtype=np.uint32)
    d_sb = np.zeros((E + 1, H, I // G, 2), dtype=np.uint16)
    one = bf16_bits(1.0)
    for e, (j, kg, ku, o) in probes.items():
        gu_codes[e, j, kg // 8] |= np.uint32(1 << (4 * (kg % 8)))
        gu_sb[e, j, kg // G] = (one, 0)
        gu_codes[e, I + j, ku // 8] |= np.uint32(1 << (4 * (ku % 8)))
        gu_sb[e, I + j, ku // G] = (one, 0)
        d_codes[e, o, j // 8] |= np.uint32(1 << (4 * (j % 8)))
        d_sb[e, o, j // G] = (bf16_bits(down_val[e]), 0)
    return dict(x=x, w_router=wr, gu_codes=gu_codes, gu_sb=gu_sb, d_codes=d_codes, d_sb=d_sb,
                logit_bias=None, bias_stride=0)


def _silu(z):
    return z / (1.0 + math.exp(-z))


def check_layer_probe(L):
    """Sparse probes pin gate vs up, input/output indexing, the down transpose,
    the routed weights and the shared expert:
    y[t, o] = sum over selected/shared e probing o of c_e * w_e * silu(x[kg]) * x[ku]."""
    rng = np.random.default_rng(21)
    T, H, I, E, G, k = 6, 256, 128, 16, 64, 4
    probes, vals = {}, {}
    for e in range(E + 1):
        j = int(rng.integers(0, I))
        kg, ku = (int(v) for v in rng.choice(H, 2, replace=False))
        o = int(rng.integers(0, H))
        probes[e] = (j, kg, ku, o)
        vals[e] = float(e + 1)          # exact small integers
    lay = _probe_layer(T, H, I, E, G, rng, probes, vals)
    y, idx, w = oracle.layer(lay, k=k, L=L)
    xf = gen.bf16_to_f32(lay["x"]).astype(np.float64)
    for t in range(T):
        ref = np.zeros(H)
        slots = [(int(idx[t, s]), w[t, s]) for s in range(k)] + [(E, 1.0)]
        for e, we in slots:
            j, kg, ku, o = probes[e]
            ref[o] += we * vals[e] * _silu(xf[t, kg]) * xf[t, ku]
        assert np.allclose(y[t], ref, rtol=1e-13, atol=1e-300), (t, np.abs(y[t] - ref).max())
    # routing of the layer is the routing of its own logits
    li = oracle.router_logits(lay["x"], lay["w_router"], L=L)
    idx2, w2 = oracle.select(li, k, L=L)
    assert np.array_equal(idx, idx2) and np.array_equal(w, w2)


def check_layer_constant(L):
    """Every scale 0: each weight equals its group's bias.  With gate bias bg,
    up bias bu and down bias bd everywhere, and S_t = sum_h x[t, h],
    y[t, :] = 2 * I * bd * silu(bg * S_t) * bu * S_t  (routed weights sum to
    one, plus the shared expert)."""
    rng = np.random.default_rng(13)
    T, H, I, E, G = 5, 256, 128, 16, 64
    bg, bu, bd = 0.03125, -0.0625, 0.5
    x = gen.f32_to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32) * 0.25)
    wr = gen.f32_to_bf16_bits((0.02 * rng.standard_normal((E, H))).astype(np.float32))
    gu_codes = rng.integers(0, 2 ** 32, size=(E + 1, 2 * I, H // 8), dtype=np.uint32)
    d_codes = rng.integers(0, 2 ** 32, size=(E + 1, H, I // 8), dtype=np.uint32)
    gu_sb = np.zeros((E + 1, 2 * I, H // G, 2), dtype=np.uint16)
    gu_sb[:, :I, :, 1] = bf16_bits(bg)
    gu_sb[:, I:, :, 1] = bf16_bits(bu)
    d_sb = np.zeros((E + 1, H, I // G, 2), dtype=np.uint16)
    d_sb[:, :, :, 1] = bf16_bits(bd)
    lay = dict(x=x, w_router=wr, gu_codes=gu_codes, gu_sb=gu_sb, d_codes=d_codes, d_sb=d_sb,
               logit_bias=None, bias_stride=0)
    y, _, _ = oracle.layer(lay, k=8, L=L)
    xf = gen.bf16_to_f32(x).astype(np.float64)
    for t in range(T):
        S = math.fsum(xf[t])
        want = 2 * I * bd * _silu(bg * S) * bu * S
        assert np.allclose(y[t], want, rtol=1e-12, atol=1e-300), (t, y[t, :3], want)


def check_layer_equivariance(L):
    """Tokens do not mix: a token's output does not depend on the batch."""
    spec = gen.LayerSpec(T=6, H=256, I=128, seed=9)
    lay = gen.make_layer(spec)
    y, idx, w = oracle.layer(lay, L=L)
    perm = np.array([4, 0, 5, 2, 1, 3], dtype=np.int32)
    y2, idx2, w2 = oracle.layer(lay, tokens=perm, L=L)
    assert np.array_equal(y2, y[perm]) and np.array_equal(idx2, idx[perm])
    lay3 = dict(lay, x=np.ascontiguousarray(lay["x"][perm]))
    y3, _, _ = oracle.layer(lay3, L=L)
    assert np.allclose(y3, y[perm], rtol=1e-14, atol=1e-300)


def check_layer_bias_routes(L):
    """A large logit bias on a hot set sends the token to exactly that set."""
    spec = gen.LayerSpec(T=4, H=256, I=128, seed=17)
    lay = gen.make_layer(spec)
    hot = [3, 250, 17, 99, 5, 128, 64, 200]
    bias = np.zeros((4, 256), dtype=np.float32)
    bias[1, hot] = 50.0
    lay["logit_bias"], lay["bias_stride"] = bias, 256
    _, idx, _ = oracle.layer(lay, L=L)
    assert sorted(idx[1].tolist()) == sorted(hot)
    # a [E] bias row (stride 0) applies to every token
    lay["logit_bias"], lay["bias_stride"] = bias[1].copy(), 0
    _, idx, _ = oracle.layer(lay, L=L)
    for t in range(4):
        assert sorted(idx[t].tolist()) == sorted(hot)


ALL_CHECKS = [
    check_dequant_golden,
    check_nibble_order,
    check_dequant_matrix_affine,
    check_router_order_golden,
    check_router_error_bound,
    check_router_subnormal,
    check_select_example,
    check_select_bruteforce,
    check_select_ties_and_zero,
    check_select_nonfinite,
    check_permute_invariants,
    check_layer_probe,
    check_layer_constant,
    check_layer_equivariance,
    check_layer_bias_routes,
]
