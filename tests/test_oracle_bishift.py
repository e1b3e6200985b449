"""Pins of the oracle's bidirectional shift for sparse (MAE) inputs.

"Vision-RWKV Backbone" (MAE pre-training) says only that Q-Shift becomes a
bidirectional shift.  The reading pinned here: Q-Shift's two groups that move
along the token row stay ([0, g) from token w - s, [g, 2g) from w + s, zero past
the ends), every other channel passes through unchanged.
"""
import numpy as np


def test_hand_worked_row(oracle_mod):
    # one row of 4 tokens, C = 8, gamma = 1/4 -> g = 2; token t, channel c = 10 t + c
    x = np.array([[[10 * t + c for c in range(8)] for t in range(4)]], dtype=np.float64)
    out = oracle_mod.bishift(x, 1, 4, 1, 0.25)[0]
    want = np.array([
        [0, 0, 12, 13, 4, 5, 6, 7],       # t = 0: [0,2) from t-1 (none), [2,4) from t+1
        [0, 1, 22, 23, 14, 15, 16, 17],
        [10, 11, 32, 33, 24, 25, 26, 27],
        [20, 21, 0, 0, 34, 35, 36, 37],   # t = 3: [2,4) from t+1 (none)
    ], dtype=np.float64)
    np.testing.assert_array_equal(out, want)


def test_relation_to_qshift_on_one_row(oracle_mod):
    # on an H = 1 grid Q-Shift's row groups match; its vertical groups read
    # outside the grid (zero) where the bidirectional shift passes x through
    rng = np.random.default_rng(0)
    x = rng.standard_normal((2, 9, 24))
    a = oracle_mod.bishift(x, 1, 9, 2, 0.25)
    q = oracle_mod.qshift(x, 1, 9, 2, 0.25)
    g = 6
    np.testing.assert_array_equal(a[..., :2 * g], q[..., :2 * g])
    assert np.all(q[..., 2 * g:4 * g] == 0.0)
    np.testing.assert_array_equal(a[..., 2 * g:], x[..., 2 * g:])


def test_mu_interpolation_and_f32_order(oracle_mod):
    rng = np.random.default_rng(1)
    x = rng.standard_normal((1, 12, 16))
    mu = rng.uniform(0, 1, 16)
    xs = oracle_mod.bishift(x, 2, 6, 1, 0.25)
    np.testing.assert_allclose(oracle_mod.bishift(x, 2, 6, 1, 0.25, mu), mu * x + (1 - mu) * xs,
                               rtol=1e-15)
    f32 = oracle_mod.bishift_f32(x, 2, 6, 1, 0.25, mu)
    np.testing.assert_allclose(f32, mu * x + (1 - mu) * xs, rtol=1e-6, atol=1e-6)
    # the rows of a 2 x 6 grid shift independently
    np.testing.assert_array_equal(xs[0, 6, :4], np.zeros(4))  # row 1, w = 0: [0, g) from w-1


def test_hand_worked_row_listing_bounds(oracle_mod):
    # C = 6, gamma = 1/4: the listing's first two bounds are int(1.5) = 1 and
    # int(3.0) = 3, so channel 0 comes from t-1, channels 1-2 from t+1, and
    # channels 3-5 pass through.  Token t, channel c = 10 t + c.
    x = np.array([[[10 * t + c for c in range(6)] for t in range(3)]], dtype=np.float64)
    out = oracle_mod.bishift(x, 1, 3, 1, 0.25)[0]
    want = np.array([
        [0, 11, 12, 3, 4, 5],
        [0, 21, 22, 13, 14, 15],
        [10, 0, 0, 23, 24, 25],
    ], dtype=np.float64)
    np.testing.assert_array_equal(out, want)
