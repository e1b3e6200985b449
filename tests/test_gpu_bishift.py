"""GPU parity of the bidirectional shift for sparse (MAE) inputs
(vrwkv_qshift_params.mode = VRWKV_QSHIFT_BIDIR, vrwkv_bishift) against the
oracle's reading of "Vision-RWKV Backbone" (MAE pre-training): the two row
groups of Q-Shift shift along the token row, every other channel passes
through.  A sparse input is one row of its visible tokens (H = 1).

The shift is bit-exact (same float32 operation order as Q-Shift); the fused
core and the channel mix on bidirectionally shifted inputs use the tolerances
of their Q-Shift tests."""
import zlib

import numpy as np
import pytest

from linear_complexity_vision_b200 import synth
from helpers import TOL, biwkv_scale, scaled_error, to_device, to_numpy, vec_f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def vk():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import linear_complexity_vision_b200 as vk
    vk.load_library()
    return vk


def _x(B, H, W, C, salt):
    seed = 20300000 + zlib.crc32(repr((B, H, W, C, salt)).encode()) % 100000
    return seed, synth.draw(seed, "x", (B, H * W, C), ("normal", 1.0))


SHIFT_CASES = [
    (2, 1, 49, 64, 1),     # 49 visible tokens of a 14 x 14 grid (MAE keeps 25 %)
    (1, 1, 196, 384, 1),   # all 196 tokens as one row
    (2, 1, 13, 24, 2),     # g = 6 (vectors straddle groups), shift 2
    (1, 1, 7, 13, 1),      # odd C: scalar kernel
    (2, 4, 9, 32, 1),      # H > 1: each row shifts on its own
    (1, 1, 5, 64, 9),      # shift past the row: the row groups empty
]


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("use_mu", [True, False])
@pytest.mark.parametrize("B,H,W,C,s", SHIFT_CASES)
def test_bishift_bit_exact(vk, oracle_mod, dt, use_mu, B, H, W, C, s):
    seed, x = _x(B, H, W, C, "shift")
    mu = synth.draw(seed, "mu_k", (C,), ("uniform", 0.0, 1.0))
    xt, xd = to_device(x, dt)
    mut, mud = vec_f32(mu)
    got = vk.bishift(xt, H, W, s, 0.25, mu=mut if use_mu else None)
    want = oracle_mod.bishift_f32(xd.astype(np.float32), H, W, s, 0.25,
                                  mu=mud.astype(np.float32) if use_mu else None,
                                  round_bf16=(dt == "bf16"))
    np.testing.assert_array_equal(to_numpy(got), want.astype(np.float64))


@pytest.mark.parametrize("dt,B,H,W,C", [
    ("f32", 2, 1, 49, 64),
    ("bf16", 2, 1, 196, 96),
    ("bf16", 1, 1, 1024, 32),    # one row spanning four CTAs
    ("bf16", 2, 16, 64, 64),     # H > 1 on the TMA path (group size 16)
])
def test_spatial_gate_bidir(vk, oracle_mod, dt, B, H, W, C):
    seed, x = _x(B, H, W, C, "gate")
    w = synth.draw(seed, "w", (C,), ("uniform", -5.0, 5.0))
    u = synth.draw(seed, "u", (C,), ("normal", 1.0))
    mus = [synth.draw(seed, n, (C,), ("uniform", 0.0, 1.0)) for n in ("mu_r", "mu_k", "mu_v")]
    xt, xd = to_device(x, dt)
    wt, wd = vec_f32(w)
    ut, ud = vec_f32(u)
    mt, md = zip(*[vec_f32(m) for m in mus])
    qs = vk.QShift(H, W, 1, 0.25, *mt, mode=1)
    got = to_numpy(vk.spatial_gate(xt, xt, xt, wt, ut, qs=qs))
    vk.device_status()
    r, k, v = (oracle_mod.bishift(xd, H, W, 1, 0.25, m) for m in md)
    want = oracle_mod.gate(r, oracle_mod.biwkv_direct(k, v, wd, ud))
    scale = oracle_mod.gate(r, biwkv_scale(oracle_mod, k, v, wd, ud))
    err = scaled_error(got, want, scale)
    assert err <= TOL[dt], f"scaled error {err:.3e}"


def test_channel_mix_bidir(vk, oracle_mod):
    seed, x = _x(2, 1, 64, 64, "cm")
    mus = [synth.draw(seed, n, (64,), ("uniform", 0.0, 1.0)) for n in ("mu_r", "mu_k")]
    xt, xd = to_device(x, "f32")
    mt, md = zip(*[vec_f32(m) for m in mus])
    got = to_numpy(vk.channel_mix(xt, vk.QShift(1, 64, 1, 0.25, mt[0], mt[1], None, mode=1)))
    r = oracle_mod.bishift(xd, 1, 64, 1, 0.25, md[0])
    k = oracle_mod.bishift(xd, 1, 64, 1, 0.25, md[1])
    want = 1.0 / (1.0 + np.exp(-r)) * np.maximum(k, 0.0) ** 2
    np.testing.assert_allclose(got, want, rtol=1e-5, atol=1e-6)


def test_mode_is_validated(vk):
    import torch
    x = torch.zeros(1, 16, 16, device="cuda")
    with pytest.raises(vk.VrwkvError):
        vk.spatial_gate(x, x, x, x[0, 0], x[0, 0], qs=vk.QShift(4, 4, mode=7))


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("B,H,W,C,s,gamma", [
    (2, 1, 11, 10, 1, 0.25),   # bounds 2, 5: channel groups [0,2) [2,5)
    (1, 1, 20, 26, 2, 0.25),   # bounds 6, 13
    (1, 2, 16, 64, 1, 0.125),  # bounds 8, 16 (vector kernel)
])
def test_bishift_listing_bounds(vk, oracle_mod, dt, B, H, W, C, s, gamma):
    seed, x = _x(B, H, W, C, "bounds")
    mu = synth.draw(seed, "mu_k", (C,), ("uniform", 0.0, 1.0))
    xt, xd = to_device(x, dt)
    mut, mud = vec_f32(mu)
    got = vk.bishift(xt, H, W, s, gamma, mu=mut)
    want = oracle_mod.bishift_f32(xd.astype(np.float32), H, W, s, gamma,
                                  mu=mud.astype(np.float32), round_bf16=(dt == "bf16"))
    np.testing.assert_array_equal(to_numpy(got), want.astype(np.float64))
