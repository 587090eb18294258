"""The seeded input generator: determinism, distribution and layout."""
import math

import numpy as np


def test_splitmix64_stream_definition(synth_mod):
    lib = synth_mod.lib()
    # output i of SplitMix64 is mix(key + (i+1) * gamma); mix(0) = 0 and the
    # stream of key 0 at i = -1 mod 2^64 therefore yields 0.
    gamma = 0x9E3779B97F4A7C15
    assert lib.synth_splitmix64_at(0, (2**64 - 1)) == 0
    # consecutive outputs of one key follow the additive gamma walk
    a = lib.synth_splitmix64_at(12345, 3)
    b = lib.synth_splitmix64_at((12345 + gamma) % 2**64, 2)
    assert a == b


def test_bf16_rounding_nearest_even(synth_mod):
    lib = synth_mod.lib()
    assert lib.synth_f64_to_bf16(1.0) == 0x3F80
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: rounds to the even mantissa (1.0)
    assert lib.synth_f64_to_bf16(1.0 + 2.0 ** -8) == 0x3F80
    # 1 + 3 * 2^-8 is a tie between 1+2^-7 (odd) and 1+2^-6 (even): rounds up
    assert lib.synth_f64_to_bf16(1.0 + 3 * 2.0 ** -8) == 0x3F82
    assert lib.synth_f64_to_bf16(-2.5) == 0xC020


def test_normals_are_standard(synth_mod):
    x = synth_mod.make_tensor(2, 0, 1, 4, 4096, 64, pos_weight=0.0, noise_weight=1.0)
    f = synth_mod.bf16_bits_to_f32(x).astype(np.float64)
    assert abs(f.mean()) < 0.01 and abs(f.std() - 1.0) < 0.01
    # ~4.6% outside 2 sigma for a normal
    assert 0.04 < (np.abs(f) > 2).mean() < 0.052


def test_deterministic_and_streams_differ(synth_mod):
    w = synth_mod.WORKLOADS["tiny"]
    q1, k1, v1 = synth_mod.make_qkv(w, seed=0)
    q2, k2, v2 = synth_mod.make_qkv(w, seed=0)
    assert np.array_equal(q1, q2) and np.array_equal(k1, k2) and np.array_equal(v1, v2)
    q3, _, _ = synth_mod.make_qkv(w, seed=1)
    assert not np.array_equal(q1, q3)
    assert not np.array_equal(q1, k1)


def test_embedding_layout(synth_mod):
    d = 64
    e = synth_mod.embedding(d, 3, 5, 7)
    # pairs are (sin, cos) of one angle
    np.testing.assert_allclose(e[0::2] ** 2 + e[1::2] ** 2, 1.0, atol=1e-14)
    # pair 0 is axis t with omega 1, pair 1 axis h, pair 2 axis w
    assert abs(e[0] - math.sin(3.0)) < 1e-15 and abs(e[2] - math.sin(5.0)) < 1e-15
    assert abs(e[4] - math.sin(7.0)) < 1e-15


def test_tile_major_token_order(synth_mod):
    """Q = e(t,h,w) with no noise: token s of tile tau must carry the embedding of
    its (t,h,w) coordinate in tile-major order."""
    grid = (2, 3, 4)     # tile grid -> token grid 8 x 12 x 16
    S = 64 * 24
    x = synth_mod.make_tensor(0, 0, 1, 1, S, 16, grid=grid, pos_weight=1.0, noise_weight=0.0)
    f = synth_mod.bf16_bits_to_f32(x)[0, 0]
    for s in (0, 1, 5, 63, 64, 100, 64 * 23 + 17):
        tile, u = divmod(s, 64)
        tt, th, tw = tile // 12, (tile // 4) % 3, tile % 4
        ut, uh, uw = u // 16, (u // 4) % 4, u % 4
        e = synth_mod.embedding(16, 4 * tt + ut, 4 * th + uh, 4 * tw + uw).astype(np.float32)
        np.testing.assert_allclose(f[s], e, atol=1e-2)


def test_bernoulli_mask(synth_mod):
    m = synth_mod.make_bernoulli_mask(0, 3, 100, 0.3)
    assert m.shape == (3, 100, 100)
    assert (m[:, np.arange(100), np.arange(100)] == 1).all()
    off = m.copy()
    off[:, np.arange(100), np.arange(100)] = 0
    assert abs(off.sum() / (3 * 100 * 99) - 0.3) < 0.01
    assert synth_mod.make_bernoulli_mask(0, 3, 100, 1.0).min() == 1
