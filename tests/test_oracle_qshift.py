"""Pins of the oracle's Q-Shift against hand-worked grids and invariants.

Sources: "Vision-RWKV Backbone", Quad-Directional Token Shift, eq. 9; the
q_shift listing on "LinXin's Blog" (Vision-RWKV entry).
"""
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load_fixture(name):
    params, rows = {}, []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            if parts[0].isalpha() or "_" in parts[0]:
                params[parts[0]] = float(parts[1])
            else:
                rows.append([float(p) for p in parts])
    return params, np.array(rows)


def _coded_input(H, W, C):
    h = np.arange(H)[:, None, None]
    w = np.arange(W)[None, :, None]
    c = np.arange(C)[None, None, :]
    x = 100.0 * c + 10.0 * h + w + 1.0
    return x.reshape(1, H * W, C)


@pytest.mark.parametrize("name", ["qshift_H2_W3_C8_s1.txt",
                                  "qshift_H3_W4_C10_s2.txt",
                                  "qshift_H3_W3_C13_s1.txt",
                                  "qshift_H2_W4_C6_s1.txt",
                                  "qshift_H3_W3_C10_s1_g02.txt"])
def test_qshift_hand_worked(oracle_mod, name):
    p, expected = _load_fixture(name)
    H, W, C, s = int(p["H"]), int(p["W"]), int(p["C"]), int(p["shift_pixel"])
    x = _coded_input(H, W, C)
    out = oracle_mod.qshift(x, H, W, s, p["gamma"])
    np.testing.assert_array_equal(out[0], expected)
    out32 = oracle_mod.qshift_f32(x.astype(np.float32), H, W, s, p["gamma"])
    np.testing.assert_array_equal(out32[0], expected.astype(np.float32))


def _source_code_input(B, H, W, C):
    """x encodes its own pixel: value = 1 + 1000*b + 10*h + w (any channel)."""
    b = np.arange(B)[:, None, None, None]
    h = np.arange(H)[None, :, None, None]
    w = np.arange(W)[None, None, :, None]
    x = 1.0 + 1000.0 * b + 10.0 * h + w + 0.0 * np.arange(C)
    return x.reshape(B, H * W, C)


def _listing_bounds(C, gamma):
    """The listing's slice bounds, evaluated by Python exactly as it prints
    them: int(C*gamma), int(C*gamma*2), int(C*gamma*3), int(C*gamma*4)."""
    return [0, int(C*gamma), int(C*gamma*2), int(C*gamma*3), int(C*gamma*4)]


def _listing_group(c, bounds):
    for j in range(4):
        if bounds[j] <= c < bounds[j + 1]:
            return j
    return 4


# C*gamma integral and not: 2.5 (C=10), 3.25 (C=13), 1.5 (C=6), 5.5 (C=22),
# 1.4 (C=7); at C=50, gamma=0.145 the double evaluation truncates the last
# bound to 28 where exact arithmetic gives 29
@pytest.mark.parametrize("H,W,C,s,gamma", [(5, 7, 12, 1, 0.25), (6, 4, 16, 2, 0.25),
                                           (3, 3, 9, 1, 0.25), (7, 5, 20, 3, 0.2),
                                           (4, 5, 10, 1, 0.25), (3, 6, 13, 2, 0.25),
                                           (5, 3, 6, 1, 0.25), (4, 4, 22, 1, 0.25),
                                           (3, 5, 50, 1, 0.145), (4, 3, 7, 1, 0.2)])
def test_qshift_every_value_comes_from_its_neighbour(oracle_mod, H, W, C, s, gamma):
    B = 2
    x = _source_code_input(B, H, W, C)
    out = oracle_mod.qshift(x, H, W, s, gamma).reshape(B, H, W, C)
    bounds = _listing_bounds(C, gamma)
    offsets = {0: (0, -s), 1: (0, s), 2: (-s, 0), 3: (s, 0)}
    for bb in range(B):
        for h in range(H):
            for w in range(W):
                for c in range(C):
                    dh, dw = offsets.get(_listing_group(c, bounds), (0, 0))
                    sh, sw = h + dh, w + dw
                    if 0 <= sh < H and 0 <= sw < W:
                        want = 1.0 + 1000.0 * bb + 10.0 * sh + sw
                    else:
                        want = 0.0
                    assert out[bb, h, w, c] == want, (bb, h, w, c)


def test_qshift_bounds_in_double_follow_python(oracle_mod):
    # 50 * 0.145 * 4 is 28.999999999999996 in double: the listing's last bound
    # is 28, one short of the exact 29, so channels 28 and 29 are copied
    assert _listing_bounds(50, 0.145) == [0, 7, 14, 21, 28]
    H, W, C = 3, 4, 50
    x = _source_code_input(1, H, W, C)
    out = oracle_mod.qshift(x, H, W, 1, 0.145).reshape(H, W, C)
    xr = x.reshape(H, W, C)
    np.testing.assert_array_equal(out[..., 28:], xr[..., 28:])
    # channel 27 belongs to the fourth group (from h+1): the last row reads 0
    assert np.all(out[H - 1, :, 27] == 0)
    np.testing.assert_array_equal(out[:H - 1, :, 27], xr[1:, :, 27])


@pytest.mark.parametrize("gamma", [0.25, 0.2, 0.15, 0.125, 0.1, 0.05])
def test_qshift_copies_exactly_the_channels_from_4_gamma_C(oracle_mod, gamma):
    """The untouched channels are those >= int(C*gamma*4) (the listing's last
    assignment): at gamma = 1/4 none, since int(C*0.25*4) = C."""
    H, W, s = 4, 5, 1
    for C in range(1, 41):
        x = _source_code_input(1, H, W, C)
        # every shifted value differs from x somewhere (interior reads move)
        out = oracle_mod.qshift(x, H, W, s, gamma)
        copied = [c for c in range(C) if np.array_equal(out[..., c], x[..., c])]
        assert copied == list(range(int(C * gamma * 4), C)), (C, gamma)
        if gamma == 0.25:
            assert copied == []


def test_qshift_zero_borders_and_copied_channels(oracle_mod):
    rng = np.random.default_rng(1)
    B, H, W, C, s = 2, 6, 5, 22, 2
    x = rng.standard_normal((B, H * W, C)) + 3.0  # no exact zeros
    out = oracle_mod.qshift(x, H, W, s, 0.25).reshape(B, H, W, C)
    xr = x.reshape(B, H, W, C)
    b0, b1, b2, b3, b4 = _listing_bounds(C, 0.25)  # 0, 5, 11, 16, 22
    assert (b1, b2, b3, b4) == (5, 11, 16, 22)
    assert np.all(out[:, :, :s, b0:b1] == 0)              # from w-s
    assert np.all(out[:, :, W - s:, b1:b2] == 0)          # from w+s
    assert np.all(out[:, :s, :, b2:b3] == 0)              # from h-s
    assert np.all(out[:, H - s:, :, b3:b4] == 0)          # from h+s
    np.testing.assert_array_equal(out[..., b4:], xr[..., b4:])
    # interior values are non-zero
    assert np.all(out[:, :, s:, b0:b1] != 0)
    assert np.all(out[:, :, :W - s, b1:b2] != 0)
    assert np.all(out[:, s:, :, b2:b3] != 0)
    assert np.all(out[:, :H - s, :, b3:b4] != 0)


def test_qshift_shift_then_unshift_is_identity_inside(oracle_mod):
    rng = np.random.default_rng(2)
    H, W, C, s = 7, 9, 8, 2
    x = rng.standard_normal((1, H * W, C))
    y = oracle_mod.qshift(x, H, W, s, 0.25)
    # group 0 (from w-s) followed by group 1 (from w+s) restores x where both
    # reads stay inside the grid: swap channel groups 0<->1 and 2<->3.
    g = 2
    perm = np.r_[np.arange(g, 2 * g), np.arange(0, g),
                 np.arange(3 * g, 4 * g), np.arange(2 * g, 3 * g)]
    z = oracle_mod.qshift(y[:, :, perm], H, W, s, 0.25)[:, :, np.argsort(perm)]
    xr, zr = x.reshape(H, W, C), z.reshape(H, W, C)
    np.testing.assert_array_equal(zr[:, : W - s, 0:g], xr[:, : W - s, 0:g])
    np.testing.assert_array_equal(zr[:, s:, g:2 * g], xr[:, s:, g:2 * g])
    np.testing.assert_array_equal(zr[: H - s, :, 2 * g:3 * g], xr[: H - s, :, 2 * g:3 * g])
    np.testing.assert_array_equal(zr[s:, :, 3 * g:4 * g], xr[s:, :, 3 * g:4 * g])


def test_qshift_mu_endpoints(oracle_mod):
    rng = np.random.default_rng(3)
    H, W, C = 4, 5, 12
    x = rng.standard_normal((2, H * W, C))
    xd = oracle_mod.qshift(x, H, W, 1, 0.25)
    np.testing.assert_array_equal(oracle_mod.qshift(x, H, W, 1, 0.25, mu=np.ones(C)), x)
    np.testing.assert_array_equal(oracle_mod.qshift(x, H, W, 1, 0.25, mu=np.zeros(C)), xd)
    mu = rng.uniform(0, 1, C)
    mixed = oracle_mod.qshift(x, H, W, 1, 0.25, mu=mu)
    # an interpolation stays between its two end points
    lo, hi = np.minimum(x, xd), np.maximum(x, xd)
    assert np.all(mixed >= lo - 1e-15) and np.all(mixed <= hi + 1e-15)


def test_qshift_eq9_order_is_a_group_permutation(oracle_mod):
    rng = np.random.default_rng(4)
    H, W, C = 5, 6, 16
    field = rng.standard_normal((1, H * W, 1))
    x = np.repeat(field, C, axis=2)  # same picture in every channel
    a = oracle_mod.qshift(x, H, W, 1, 0.25)
    b = oracle_mod.qshift(x, H, W, 1, 0.25, eq9_order=True)
    g = C // 4
    # eq. 9: groups (h-1, h+1, w-1, w+1); listing: (w-s, w+s, h-s, h+s)
    for eq_grp, code_grp in enumerate((2, 3, 0, 1)):
        np.testing.assert_array_equal(b[..., eq_grp * g:(eq_grp + 1) * g],
                                      a[..., code_grp * g:(code_grp + 1) * g])


def test_qshift_degenerate_shifts(oracle_mod):
    rng = np.random.default_rng(5)
    H, W, C = 3, 4, 8
    x = rng.standard_normal((1, H * W, C)) + 5.0
    # shift 0 copies every channel
    np.testing.assert_array_equal(oracle_mod.qshift(x, H, W, 0, 0.25), x)
    # a shift at or beyond the grid extent empties the moved groups
    out = oracle_mod.qshift(x, H, W, 4, 0.25)
    assert np.all(out[..., :8] == 0)
    out = oracle_mod.qshift(x, H, W, 3, 0.25)  # >= H only
    assert np.all(out[..., 4:8] == 0)
    assert np.all(out[..., 0:4].reshape(H, W, 4)[:, 0, :2] == 0)
    # gamma = 0.1 at C = 8: the bounds are int(0.8) = 0, int(1.6) = 1,
    # int(2.4) = 2, int(3.2) = 3, so the first group is empty, channels 0, 1, 2
    # move (w+1, h-1, h+1) and channels 3.. are copied
    out = oracle_mod.qshift(x, H, W, 1, 0.1).reshape(H, W, C)
    xr = x.reshape(H, W, C)
    np.testing.assert_array_equal(out[:, :W - 1, 0], xr[:, 1:, 0])
    np.testing.assert_array_equal(out[1:, :, 1], xr[:H - 1, :, 1])
    np.testing.assert_array_equal(out[:H - 1, :, 2], xr[1:, :, 2])
    np.testing.assert_array_equal(out[..., 3:], xr[..., 3:])
    # gamma = 0 copies every channel
    np.testing.assert_array_equal(oracle_mod.qshift(x, H, W, 1, 0.0), x)


def test_qshift_f32_matches_f64_within_rounding(oracle_mod):
    rng = np.random.default_rng(6)
    H, W, C = 6, 6, 24
    x = rng.standard_normal((2, H * W, C)).astype(np.float32)
    mu = rng.uniform(0, 1, C).astype(np.float32)
    a = oracle_mod.qshift_f32(x, H, W, 1, 0.25, mu=mu)
    b = oracle_mod.qshift(x.astype(np.float64), H, W, 1, 0.25, mu=mu.astype(np.float64))
    np.testing.assert_allclose(a, b, rtol=0, atol=4 * np.finfo(np.float32).eps * 8)
    # without mu the binary32 path is a pure copy
    np.testing.assert_array_equal(oracle_mod.qshift_f32(x, H, W, 1, 0.25),
                                  oracle_mod.qshift(x.astype(np.float64), H, W, 1, 0.25))


def test_round_bf16_matches_torch(oracle_mod):
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(7)
    a = np.concatenate([
        rng.standard_normal(10000).astype(np.float32) * 10,
        # exact ties between two bfloat16 neighbours (low 16 bits = 0x8000)
        (np.arange(1, 200, dtype=np.uint32) << 16 | 0x8000).view(np.float32),
        np.array([0.0, -0.0, 1e-40, -3e38, np.inf, -np.inf], dtype=np.float32)])
    ours = oracle_mod.round_bf16(a)
    ref = torch.from_numpy(a).to(torch.bfloat16).to(torch.float32).numpy()
    np.testing.assert_array_equal(ours, ref)
