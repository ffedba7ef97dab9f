"""The seeded input generator: published SplitMix64 vectors, determinism and
the distributions the layer workloads call for."""
import math

import numpy as np

import gen


def test_splitmix64_published_vectors():
    # SplitMix64 (Steele, Lea & Flood 2014) from state 1234567: the widely
    # published first five outputs, and the first output from state 0.
    L = gen.lib()
    want = [6457827717110365317, 3203168211198807973, 9817491932198370423,
            4593380528125082431, 16408922859458223821]
    assert [L.gen_draw(1234567, i) for i in range(5)] == want
    assert L.gen_draw(0, 0) == 0xE220A8397B1DCDAF


def test_deterministic_and_prefix():
    spec = gen.LayerSpec(T=16, H=256, I=128, seed=5)
    a = gen.make_layer(spec)
    b = gen.make_layer(spec)
    for name in ("x", "w_router", "gu_codes", "gu_sb", "d_codes", "d_sb"):
        assert np.array_equal(a[name], b[name]), name
    small = gen.make_activations(spec.with_T(3))
    assert np.array_equal(small["x"], a["x"][:3])
    other = gen.make_layer(spec, layer=1)
    assert not np.array_equal(other["gu_codes"], a["gu_codes"])


def test_distributions():
    spec = gen.LayerSpec(T=64, H=512, I=128, seed=0)
    lay = gen.make_layer(spec)
    x = gen.bf16_to_f32(lay["x"]).astype(np.float64)
    assert abs(x.mean()) < 0.02 and abs(x.std() - 1.0) < 0.02
    wr = gen.bf16_to_f32(lay["w_router"]).astype(np.float64)
    assert abs(wr.std() - 0.02) < 0.001
    codes = lay["gu_codes"]
    nib = np.stack([(codes >> (4 * j)) & 0xF for j in range(8)], axis=-1).ravel()
    hist = np.bincount(nib, minlength=16) / nib.size
    assert np.all(np.abs(hist - 1 / 16) < 0.002)
    sb = lay["gu_sb"]
    s = gen.bf16_to_f32(sb[..., 0]).astype(np.float64)
    b = gen.bf16_to_f32(sb[..., 1]).astype(np.float64)
    assert np.all(s >= 0) and np.array_equal(b, -8.0 * s)
    # |N(0, 0.02)| has mean 0.02 * sqrt(2 / pi)
    assert abs(s.mean() - 0.02 * math.sqrt(2 / math.pi)) < 0.0005


def test_config_biases():
    z = gen.make_activations(gen.config(2).with_T(4))
    assert z["bias_stride"] == 0 and z["logit_bias"].shape == (256,)
    assert z["logit_bias"][0] == 0.0 and abs(z["logit_bias"][9] + 1.1 * math.log(10)) < 1e-6
    spec = gen.config(4).with_T(64)
    h = gen.make_activations(spec)
    bias = h["logit_bias"]
    assert bias.shape == (64, 256) and h["bias_stride"] == 256
    hot = gen.hot_experts(spec)
    assert len(set(hot.tolist())) == 8
    rows = np.nonzero(bias.any(axis=1))[0]
    assert len(rows) == 32
    assert np.all(bias[rows][:, hot] == 8.0) and bias.sum() == 32 * 8 * 8.0
