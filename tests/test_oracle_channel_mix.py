"""Pins of the oracle's channel-mix path (eq. 3-4 without projections:
sigma(QS_R(x)) * max(QS_K(x), 0)^2) against hand-worked values and limits.

Sources: "Vision-RWKV Backbone", Overall Architecture, eq. 3-4 (R_c, K_c from
Q-Shift, V_c = SquaredReLU(K_c), O_c = sigma(R_c) (.) V_c) and Quad-Directional
Token Shift, eq. 9.
"""
import numpy as np


def test_hand_worked_single_token_grid(oracle_mod):
    # a 1x1 grid: every shifted group reads outside the grid (zero), so with
    # mu the mixes are mu * x.  gamma = 0.2, C = 6: the listing's bounds are
    # int(1.2) = 1, int(2.4) = 2, int(3.6) = 3, int(4.8) = 4, so channels 4, 5
    # copy x.  x = [2, -1, 3, 0.5, -2, 1.5]
    x = np.array([[[2.0, -1.0, 3.0, 0.5, -2.0, 1.5]]])
    mu_r = np.array([0.5, 0.5, 0.0, 1.0, 0.3, 0.9])
    mu_k = np.array([1.0, 1.0, 0.5, 0.25, 0.7, 0.1])
    out = oracle_mod.channel_mix(x, 1, 1, 1, 0.2, mu_r, mu_k)[0, 0]
    sig = lambda z: 1.0 / (1.0 + np.exp(-z))
    want = [
        sig(1.0) * 2.0 ** 2,      # r = 0.5*2,   k = 1.0*2
        sig(-0.5) * 0.0,          # k = -1 -> relu 0
        sig(0.0) * 1.5 ** 2,      # r = 0,       k = 0.5*3
        sig(0.5) * 0.125 ** 2,    # r = 1*0.5,   k = 0.25*0.5
        sig(-2.0) * 0.0,          # copied channel: r = k = -2
        sig(1.5) * 1.5 ** 2,      # copied channel: r = k = 1.5
    ]
    np.testing.assert_allclose(out, want, rtol=1e-14)
    # at gamma = 1/4 the bounds are 1, 3, 4, 6: channels 4, 5 move (from h+1,
    # outside the grid), so r = mu_r x and k = mu_k x there as well
    out = oracle_mod.channel_mix(x, 1, 1, 1, 0.25, mu_r, mu_k)[0, 0]
    np.testing.assert_allclose(out[:4], want[:4], rtol=1e-14)
    np.testing.assert_allclose(out[4:], [0.0, sig(0.9 * 1.5) * (0.1 * 1.5) ** 2], rtol=1e-14)


def test_negative_inputs_give_zero(oracle_mod):
    rng = np.random.default_rng(0)
    x = -np.abs(rng.standard_normal((2, 20, 8))) - 0.1
    out = oracle_mod.channel_mix(x, 4, 5, 1, 0.25, rng.uniform(0, 1, 8), rng.uniform(0, 1, 8))
    assert np.all(out == 0.0)


def test_gate_limits_and_square(oracle_mod):
    # mu = 1 everywhere: r = k = x, so out = sigma(x) * relu(x)^2
    rng = np.random.default_rng(1)
    x = rng.standard_normal((1, 12, 16)) * 3
    out = oracle_mod.channel_mix(x, 3, 4, 1, 0.25, np.ones(16), np.ones(16))
    kp = np.maximum(x, 0.0)
    assert np.all(out <= kp ** 2 + 1e-15) and np.all(out >= 0.5 * kp ** 2 - 1e-15)
    big = oracle_mod.channel_mix(np.full((1, 4, 4), 40.0), 2, 2, 1, 0.25, np.ones(4), np.ones(4))
    np.testing.assert_allclose(big, 1600.0, rtol=1e-15)
