"""GPU parity of the channel-mix elementwise path (vrwkv_channel_mix) against
the float64 oracle, element by element on the same seeded inputs:
out = sigma(QS_R(x)) * max(QS_K(x), 0)^2 ("Vision-RWKV Backbone", Overall
Architecture, eq. 3-4 with identity projections; Q-Shift of eq. 9).

Error metric.  k = x_shift + mu_k*(x - x_shift) can cancel to ~0, so a plain
relative error is ill-posed.  In float32 the mix x_shift + mu*(x - x_shift)
is off by at most a few ulps of m_* = (|mu_*| + |1 - mu_*|)(|x| + |x_shift|),
and sigma(r) moves by sigma(r)(1 - sigma(r)) times the error of r, so the error
of every element is divided by
    S = sigma(r) * m_k^2 * (1 + m_r),
which bounds |out| and the propagated rounding: hardware exp2 and reciprocal
and the float32 steps keep the error within ~10 float32 ulps of S, and one
rounding to bfloat16 at the store adds at most 2^-9 S.  Tolerances: 1e-5
(float32 I/O), 4e-3 (bfloat16 I/O).
"""
import zlib

import numpy as np
import pytest

from linear_complexity_vision_b200 import synth
from helpers import to_device, to_numpy, torch_dtype, vec_f32

pytestmark = pytest.mark.gpu

CM_TOL = {"f32": 1e-5, "bf16": 4e-3}


@pytest.fixture(scope="module")
def vk():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import linear_complexity_vision_b200 as vk
    vk.load_library()
    return vk


def _sigmoid(z):
    """1/(1+e^-z) without cancellation for z << 0: e^z/(1+e^z) there."""
    e = np.exp(-np.abs(z))
    return np.where(z >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def _scale(oracle, xd, H, W, s, gamma, mu_r, mu_k):
    """S = sigma(QS_R(x)) * m_k^2 * (1 + m_r) in float64 (see the module doc)."""
    xs = oracle.qshift(xd, H, W, s, gamma)
    r = xs if mu_r is None else oracle.qshift(xd, H, W, s, gamma, mu=mu_r)
    mag = np.abs(xd) + np.abs(xs)

    def m(mu):
        return mag if mu is None else (np.abs(mu) + np.abs(1.0 - mu)) * mag
    mk = m(mu_k)
    return _sigmoid(r) * mk * mk * (1.0 + m(mu_r))


def _check(vk, oracle, x, dt, H, W, s, gamma, mu_r, mu_k, use_qs=True, offset=0):
    import torch
    B, T, C = x.shape
    xt, xd = to_device(x, dt)
    if offset:
        buf = torch.empty(xt.numel() + offset, dtype=torch_dtype(dt), device="cuda")
        xs = buf[offset:].view(B, T, C)
        xs.copy_(xt)
        xt = xs
        obuf = torch.empty_like(buf)
        out = obuf[offset:].view(B, T, C)
    else:
        out = None
    mr = mk = None
    mrd = mkd = None
    if mu_r is not None:
        mr, mrd = vec_f32(mu_r)
    if mu_k is not None:
        mk, mkd = vec_f32(mu_k)
    qs = vk.QShift(H, W, s, gamma, mu_r=mr, mu_k=mk) if use_qs else None
    got = to_numpy(vk.channel_mix(xt, qs, out=out))
    vk.device_status()
    if use_qs:
        want = oracle.channel_mix(xd, H, W, s, gamma, mrd, mkd)
        scale = _scale(oracle, xd, H, W, s, gamma, mrd, mkd)
    else:
        # QS is the identity: sigma(x) * relu(x)^2
        want = _sigmoid(xd) * np.maximum(xd, 0.0) ** 2
        scale = _sigmoid(xd) * xd * xd * (1.0 + np.abs(xd))
    err = float(np.max(np.abs(got - want) / np.maximum(scale, 1e-30)))
    assert np.all(np.isfinite(got))
    assert err <= CM_TOL[dt], f"scaled error {err:.3e} > {CM_TOL[dt]}"
    return got


CASES = [
    # B, H, W, C, s, gamma
    (2, 14, 14, 384, 1, 0.25),    # the 224^2 grid
    (3, 5, 7, 64, 1, 0.25),       # ragged rows: 105 rows over the CTAs
    (1, 1, 1, 64, 1, 0.25),       # a single token
    (1, 1, 9, 32, 1, 0.25),       # H = 1
    (1, 9, 1, 32, 1, 0.25),       # W = 1
    (2, 6, 6, 64, 2, 0.25),       # shift 2
    (1, 3, 3, 64, 4, 0.25),       # shift beyond the grid: empty groups
    (2, 6, 6, 64, 0, 0.25),       # shift 0
    (1, 6, 6, 64, 1, 0.0),        # gamma 0: every channel copied
    (2, 8, 8, 13, 1, 0.25),       # odd C: scalar kernel
    (1, 8, 8, 40, 1, 0.25),       # g = 10: vectors straddle groups (scalar kernel)
    (1, 4, 4, 4160, 1, 0.25),     # 520 bf16 / 1040 f32 vectors: split channel chunks
    (8, 64, 64, 1024, 1, 0.25),   # the 1024^2 grid at C = 1024 (full size)
    # the listing's bounds int(C*gamma*j) where C*gamma is not an integer
    (2, 5, 6, 10, 1, 0.25),       # bounds 2, 5, 7, 10 (scalar kernel)
    (1, 8, 8, 64, 1, 0.125),      # bounds 8, 16, 24, 32: vector kernel, 32.. copied
    (1, 6, 6, 50, 2, 0.145),      # double rounding: last bound 28
]


def _inputs(B, H, W, C, salt):
    seed = 20270000 + zlib.crc32(repr((B, H, W, C, salt)).encode()) % 100000
    x = synth.draw(seed, "x", (B, H * W, C), ("normal", 1.0))
    mu_r = synth.draw(seed, "mu_r", (C,), ("uniform", 0.0, 1.0))
    mu_k = synth.draw(seed, "mu_k", (C,), ("uniform", 0.0, 1.0))
    return x, mu_r, mu_k


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("B,H,W,C,s,gamma", CASES)
def test_channel_mix_parity(vk, oracle_mod, dt, B, H, W, C, s, gamma):
    x, mu_r, mu_k = _inputs(B, H, W, C, "cm")
    _check(vk, oracle_mod, x, dt, H, W, s, gamma, mu_r, mu_k)


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("which", ["none", "r", "k"])
def test_channel_mix_without_mu(vk, oracle_mod, dt, which):
    B, H, W, C = 2, 7, 9, 64
    x, mu_r, mu_k = _inputs(B, H, W, C, which)
    _check(vk, oracle_mod, x, dt, H, W, 1, 0.25,
           None if which in ("none", "r") else mu_r,
           None if which in ("none", "k") else mu_k)


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("C", [64, 13])
def test_channel_mix_identity_shift(vk, oracle_mod, dt, C):
    x, _, _ = _inputs(2, 5, 6, C, "id")
    _check(vk, oracle_mod, x, dt, 5, 6, 1, 0.25, None, None, use_qs=False)


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_channel_mix_unaligned(vk, oracle_mod, dt):
    # element-aligned but not 16-byte aligned tensors take the scalar kernel
    x, mu_r, mu_k = _inputs(2, 5, 6, 64, "unaligned")
    _check(vk, oracle_mod, x, dt, 5, 6, 1, 0.25, mu_r, mu_k, offset=1)
    assert vk.load_library().vrwkv_last_kernel().decode() == "channel_mix_scalar_kernel"


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_channel_mix_extremes(vk, oracle_mod, dt):
    # large |x|: sigma saturates to 0 and 1; negative k gives exact zeros
    B, H, W, C = 1, 6, 6, 64
    x, mu_r, mu_k = _inputs(B, H, W, C, "ext")
    x = x * 40.0
    got = _check(vk, oracle_mod, x, dt, H, W, 1, 0.25, mu_r, mu_k)
    _, xd = to_device(x, dt)
    k = oracle_mod.qshift(xd, H, W, 1, 0.25, mu=vec_f32(mu_k, device="cpu")[1])
    assert np.all(got[k < -1e-3] == 0.0)


def test_channel_mix_fast_path_and_deterministic(vk, oracle_mod):
    x, mu_r, mu_k = _inputs(2, 14, 14, 384, "det")
    a = _check(vk, oracle_mod, x, "bf16", 14, 14, 1, 0.25, mu_r, mu_k)
    assert vk.load_library().vrwkv_last_kernel().decode() == "channel_mix_vec_kernel"
    b = _check(vk, oracle_mod, x, "bf16", 14, 14, 1, 0.25, mu_r, mu_k)
    np.testing.assert_array_equal(a, b)


def test_channel_mix_invalid(vk):
    import torch
    x = torch.zeros(1, 4, 16, device="cuda")
    with pytest.raises(vk.VrwkvError):
        vk.channel_mix(x, vk.QShift(3, 2))       # H*W != T
    with pytest.raises(vk.VrwkvError):
        vk.channel_mix(x, vk.QShift(2, 2, gamma=0.3))
    with pytest.raises(vk.VrwkvError):
        vk.channel_mix(x, out=x)                 # output overlaps the input
