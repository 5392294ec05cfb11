"""Pins of the oracle's per-channel gated pooling (the per-channel variant of
softmax-gated pooling with a learned positional bias): closed forms for
uniform gates, a bias that picks one slot in one channel only, the reduction
to the scalar gate when the bias is the same in every channel, the gate
reading each channel of the key alone, weights summing to one per channel.
CPU only."""
import numpy as np

import oracle as O


def _tokens(D):
    # token p carries p + 0.01 c in channel c
    return lambda p: float(p) + 0.01 * np.arange(D)


def test_uniform_gates_give_the_window_mean_per_channel():
    D = 5
    src = _tokens(D)
    (out,), w = O.pool_entries_per_channel(src, [src], np.zeros(D), np.zeros((8, D)), 8, 4,
                                           range(6))
    c = 0.01 * np.arange(D)
    # entry 0 sees positions 0..3 (left edge), entry j >= 1 sees 4j-4 .. 4j+3
    assert np.allclose(out[0], 1.5 + c, rtol=0, atol=1e-14)
    for j in range(1, 6):
        assert np.allclose(out[j], 4 * j - 0.5 + c, rtol=0, atol=1e-13)
    assert w.shape == (6, 8, D)
    assert np.allclose(w[0][:, 0], [0, 0, 0, 0, 0.25, 0.25, 0.25, 0.25])
    # HCA: 128 tokens, window = stride
    (out,), _ = O.pool_entries_per_channel(src, [src], np.zeros(D), np.zeros((128, D)), 128, 128,
                                           range(3))
    for j in range(3):
        assert np.allclose(out[j], 128 * j + 63.5 + c, rtol=0, atol=1e-12)


def test_bias_picks_one_slot_in_one_channel_only():
    D, r_star, c_star = 4, 6, 2
    src = _tokens(D)
    b = np.zeros((8, D))
    b[r_star, c_star] = 60.0                 # e^-60 leaves the other slots out
    (out,), w = O.pool_entries_per_channel(src, [src], np.zeros(D), b, 8, 4, [3])
    pos = O.pool_positions(3, 8, 4)
    assert np.isclose(out[0][c_star], pos[r_star] + 0.01 * c_star, rtol=0, atol=1e-12)
    for c in range(D):
        if c != c_star:                      # the other channels keep the mean
            assert np.isclose(out[0][c], pos.mean() + 0.01 * c, rtol=0, atol=1e-12)
    assert np.isclose(w[0][r_star, c_star], 1.0, atol=1e-20)


def test_same_bias_in_every_channel_is_the_scalar_gate():
    rng = np.random.default_rng(11)
    D, pool, stride = 6, 8, 4
    X = rng.standard_normal((64, D))
    src = lambda p: X[p]
    b = rng.standard_normal(pool)
    (pc,), wpc = O.pool_entries_per_channel(src, [src], np.zeros(D), np.repeat(b[:, None], D, 1),
                                            pool, stride, range(10))
    (sc,), wsc = O.pool_entries(src, [src], np.zeros(D), b, pool, stride, range(10))
    assert np.allclose(pc, sc, rtol=0, atol=1e-14)
    assert np.allclose(wpc, np.repeat(wsc[:, :, None], D, 2), rtol=0, atol=1e-15)


def test_the_gate_reads_its_own_channel_of_the_key():
    # channel 1's weight is large; the key is large in channel 1 at one slot
    # only: channel 1 takes that slot (and so does the value's channel 1),
    # the other channels (weight 0) keep the mean; the value itself never
    # moves the gate
    D, pool, stride, j = 3, 8, 4, 2
    pos = O.pool_positions(j, pool, stride)
    hot = int(pos[5])
    K = lambda p: np.array([1.0, 100.0 if p == hot else 0.0, -1.0])
    V = lambda p: np.array([p, 2.0 * p, 1000.0 if p == pos[0] else 3.0])
    w = np.array([0.0, 1.0, 0.0])
    (k, v), a = O.pool_entries_per_channel(K, [K, V], w, np.zeros((pool, D)), pool, stride, [j])
    assert np.isclose(v[0][1], 2.0 * hot, rtol=0, atol=1e-9)
    assert np.isclose(v[0][0], pos.mean(), rtol=0, atol=1e-12)
    assert np.isclose(v[0][2], (1000.0 + 7 * 3.0) / 8, rtol=0, atol=1e-12)
    assert np.isclose(k[0][1], 100.0, rtol=0, atol=1e-9)
    assert np.allclose(a[0][:, 0], 1 / 8) and np.allclose(a[0][:, 2], 1 / 8)


def test_weights_sum_to_one_per_channel_and_convexity():
    rng = np.random.default_rng(12)
    D, pool, stride = 7, 8, 4
    X = rng.standard_normal((80, D)) * 3
    src = lambda p: X[p]
    (out,), w = O.pool_entries_per_channel(src, [src], rng.standard_normal(D),
                                           rng.standard_normal((pool, D)), pool, stride,
                                           range(20))
    assert np.allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-14)
    assert np.all(w >= 0)
    for j in range(20):
        p = O.pool_positions(j, pool, stride)
        p = p[p >= 0]
        assert np.all(out[j] <= X[p].max(axis=0) + 1e-12)
        assert np.all(out[j] >= X[p].min(axis=0) - 1e-12)
