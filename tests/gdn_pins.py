"""Pins of the recurrent-scan oracle (oracle/gdn_oracle.c) to facts that do
not come from the oracle itself.  Each check takes an oracle library handle,
so the same checks run against planted mutants (test_gdn_oracle.py).

  pure decay       beta = 0 (or k = 0): nothing is written, S_T = (prod a) S0
                   and o_t = scale (prod_{s<=t} a_s) S0 q_t;
  single write     S0 = 0, one token: S = beta v k^T, o = scale beta (k.q) v;
  delta retrieval  a = 1, beta = 1 and exactly orthonormal keys (rows of a
                   Hadamard matrix / 2, exact in bf16): each write makes the
                   state recall v for k exactly, and after dk writes the
                   state is sum_j v_j k_j^T whatever S0 was;
  matrix form      the same recurrence evaluated as products of dk x dk
                   matrices, S <- S (a (I - beta k k^T)) + beta v k^T, in
                   numpy fp64, with query/key heads shared by value heads;
  no tokens        T = 0 leaves the state unchanged.
"""
import numpy as np

import gen
import oracle.gdn as G


def _bits(f):
    return gen.f32_to_bf16_bits(np.asarray(f, dtype=np.float32))


def _vals(b):
    return gen.bf16_to_f32(b).astype(np.float64)


def _random(rng, B, T, Hk, Hv, dk, dv):
    q = _bits(rng.normal(size=(B, T, Hk, dk)) * 0.5)
    k = _bits(rng.normal(size=(B, T, Hk, dk)) * 0.5)
    v = _bits(rng.normal(size=(B, T, Hv, dv)))
    g = rng.uniform(-0.3, 0.0, size=(B, T, Hv)).astype(np.float32)
    beta = rng.uniform(0.05, 0.95, size=(B, T, Hv)).astype(np.float32)
    S0 = rng.normal(size=(B, Hv, dv, dk)).astype(np.float32)
    return q, k, v, g, beta, S0


def check_pure_decay(L):
    rng = np.random.default_rng(1)
    q, k, v, g, beta, S0 = _random(rng, 1, 5, 1, 2, 8, 6)
    for zero_beta in (True, False):
        b2 = np.zeros_like(beta) if zero_beta else beta
        k2 = k if zero_beta else np.zeros_like(k)
        o, S = G.scan(q, k2, v, g, b2, 0.7, S0, L=L)
        decay = np.cumprod(np.exp(g.astype(np.float64)), axis=1)          # [B, T, Hv]
        S_ref = decay[0, -1][:, None, None] * S0[0].astype(np.float64)
        assert np.allclose(S[0], S_ref, rtol=1e-12, atol=1e-14)
        for t in range(5):
            o_ref = 0.7 * decay[0, t][:, None] * np.einsum("hij,j->hi", S0[0].astype(np.float64), _vals(q[0, t, 0]))
            assert np.allclose(o[0, t], o_ref, rtol=1e-12, atol=1e-14)


def check_single_write(L):
    rng = np.random.default_rng(2)
    q, k, v, g, beta, S0 = _random(rng, 1, 1, 1, 3, 8, 5)
    S0 = np.zeros_like(S0)
    o, S = G.scan(q, k, v, g, beta, 1.3, S0, L=L)
    kk, qq = _vals(k[0, 0, 0]), _vals(q[0, 0, 0])
    for h in range(3):
        vv = _vals(v[0, 0, h])
        bt = float(beta[0, 0, h])
        assert np.allclose(S[0, h], bt * np.outer(vv, kk), rtol=1e-12, atol=1e-15)
        assert np.allclose(o[0, 0, h], 1.3 * bt * np.dot(kk, qq) * vv, rtol=1e-12, atol=1e-15)


def check_delta_retrieval(L):
    Hd = np.array([[1, 1, 1, 1], [1, -1, 1, -1], [1, 1, -1, -1], [1, -1, -1, 1]], dtype=np.float64) / 2.0
    rng = np.random.default_rng(3)
    T, dk, dv = 4, 4, 3
    k = _bits(Hd[None, :, None, :])                                        # [1, T, 1, dk], orthonormal rows
    q = k.copy()
    v = _bits(rng.normal(size=(1, T, 1, dv)))
    g = np.zeros((1, T, 1), dtype=np.float32)
    beta = np.ones((1, T, 1), dtype=np.float32)
    S0 = rng.normal(size=(1, 1, dv, dk)).astype(np.float32)
    o, S = G.scan(q, k, v, g, beta, 1.0, S0, L=L)
    V = _vals(v[0, :, 0])                                                  # [T, dv]
    # every write: reading with the key just written returns its value
    for t in range(T):
        assert np.allclose(o[0, t, 0], V[t], rtol=0, atol=1e-12)
    # after dk orthonormal writes the state is sum_j v_j k_j^T, S0 forgotten
    assert np.allclose(S[0, 0], V.T @ Hd, rtol=0, atol=1e-12)


def check_matrix_form(L):
    rng = np.random.default_rng(4)
    B, T, Hk, Hv, dk, dv = 2, 6, 2, 4, 8, 5
    q, k, v, g, beta, S0 = _random(rng, B, T, Hk, Hv, dk, dv)
    o, S = G.scan(q, k, v, g, beta, 0.35, S0, L=L)
    for b in range(B):
        for h in range(Hv):
            hk = h // (Hv // Hk)
            M = S0[b, h].astype(np.float64)
            for t in range(T):
                kk, qq, vv = _vals(k[b, t, hk]), _vals(q[b, t, hk]), _vals(v[b, t, h])
                a, bt = np.exp(float(g[b, t, h])), float(beta[b, t, h])
                M = M @ (a * (np.eye(dk) - bt * np.outer(kk, kk))) + bt * np.outer(vv, kk)
                assert np.allclose(o[b, t, h], 0.35 * (M @ qq), rtol=1e-10, atol=1e-12)
            assert np.allclose(S[b, h], M, rtol=1e-10, atol=1e-12)


def check_no_tokens(L):
    rng = np.random.default_rng(5)
    q, k, v, g, beta, S0 = _random(rng, 2, 0, 1, 2, 4, 4)
    o, S = G.scan(q, k, v, g, beta, 1.0, S0, L=L)
    assert o.size == 0 and np.array_equal(S, S0.astype(np.float64))


ALL_CHECKS = [check_pure_decay, check_single_write, check_delta_retrieval, check_matrix_form, check_no_tokens]
