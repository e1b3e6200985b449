"""Pins of the oracle's spatial-mix block (Q-Shift, R/K/V projections, Bi-WKV,
sigma gate, W_O, LayerNorm; "Vision-RWKV Backbone", Overall Architecture,
eq. 1-2 with eq. 5 and eq. 9).

- LayerNorm is checked against torch.nn.functional.layer_norm and against its
  defining properties (zero mean, unit biased variance before the affine).
- With identity projections and an identity LayerNorm affine the block
  reduces to LayerNorm of the spatial-mix core, which is pinned on its own.
- Projections are linear: scaling W_V scales V, which leaves wkv's ratio
  structure intact (wkv is linear in v), so O scales and LayerNorm removes
  the scale.
"""
import numpy as np
import torch

from linear_complexity_vision_b200 import synth


def _block_inputs(B=2, H=3, W=4, C=8, seed=3):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((B, H * W, C))
    ws = [rng.standard_normal((C, C)) / np.sqrt(C) for _ in range(4)]
    w = rng.uniform(-3, 3, C)
    u = rng.standard_normal(C)
    mus = [rng.uniform(0, 1, C) for _ in range(3)]
    g = 1 + 0.1 * rng.standard_normal(C)
    b = 0.1 * rng.standard_normal(C)
    return x, ws, w, u, mus, g, b


def test_layer_norm_matches_torch(oracle_mod):
    rng = np.random.default_rng(0)
    y = rng.standard_normal((3, 5, 16)) * 4 + 2
    g = rng.standard_normal(16)
    b = rng.standard_normal(16)
    want = torch.nn.functional.layer_norm(torch.from_numpy(y), (16,), torch.from_numpy(g),
                                          torch.from_numpy(b), eps=1e-5).numpy()
    np.testing.assert_allclose(oracle_mod.layer_norm(y, g, b), want, rtol=1e-12, atol=1e-12)


def test_layer_norm_moments(oracle_mod):
    rng = np.random.default_rng(1)
    y = rng.standard_normal((4, 32)) * 10 - 3
    z = oracle_mod.layer_norm(y, np.ones(32), np.zeros(32), eps=0.0)
    np.testing.assert_allclose(z.mean(axis=-1), 0.0, atol=1e-12)
    np.testing.assert_allclose((z ** 2).mean(axis=-1), 1.0, rtol=1e-12)


def test_identity_projections_reduce_to_core(oracle_mod):
    x, _, w, u, mus, _, _ = _block_inputs()
    C = x.shape[2]
    eye = np.eye(C)
    got = oracle_mod.spatial_mix_block(x, eye, eye, eye, eye, w, u, *mus, np.ones(C), np.zeros(C),
                                       3, 4, method="direct")
    core = oracle_mod.spatial_core(x, x, x, w, u, 3, 4, 1, 0.25, *mus, method="direct")
    np.testing.assert_allclose(got, oracle_mod.layer_norm(core, np.ones(C), np.zeros(C)),
                               rtol=1e-12, atol=1e-12)


def test_scaling_w_o_is_removed_by_layer_norm(oracle_mod):
    x, ws, w, u, mus, g, b = _block_inputs(seed=5)
    a = oracle_mod.spatial_mix_block(x, *ws, w, u, *mus, g, b, 3, 4, eps=0.0)
    ws2 = list(ws)
    ws2[3] = ws[3] * 7.5
    c = oracle_mod.spatial_mix_block(x, *ws2, w, u, *mus, g, b, 3, 4, eps=0.0)
    np.testing.assert_allclose(a, c, rtol=1e-10, atol=1e-12)


def test_projection_is_applied_after_the_shift(oracle_mod):
    # a channel permutation P as W_K = W_V = P (and W_R = P): the block equals
    # the core run on x with the permutation applied after Q-Shift, i.e. on
    # the shifted inputs permuted -- not on a permuted x shifted afterwards
    x, _, w, u, mus, _, _ = _block_inputs(seed=7)
    C = x.shape[2]
    perm = np.roll(np.arange(C), 3)
    P = np.eye(C)[:, perm]  # x @ P == x[..., perm]
    got = oracle_mod.spatial_mix_block(x, P, P, P, np.eye(C), w[perm], u[perm], *mus,
                                       np.ones(C), np.zeros(C), 3, 4, method="direct")
    xr, xk, xv = (oracle_mod.qshift(x, 3, 4, 1, 0.25, m)[..., perm] for m in mus)
    core = oracle_mod.gate(xr, oracle_mod.biwkv_direct(xk, xv, w[perm], u[perm]))
    np.testing.assert_allclose(got, oracle_mod.layer_norm(core, np.ones(C), np.zeros(C)),
                               rtol=1e-12, atol=1e-12)


def test_bf16_rounding_option_stays_close(oracle_mod):
    x, ws, w, u, mus, g, b = _block_inputs(B=1, H=6, W=6, C=16, seed=9)
    a = oracle_mod.spatial_mix_block(x, *ws, w, u, *mus, g, b, 6, 6)
    c = oracle_mod.spatial_mix_block(x, *ws, w, u, *mus, g, b, 6, 6, round_like_bf16=True)
    assert np.max(np.abs(a - c)) < 0.1 and np.max(np.abs(a - c)) > 0.0
