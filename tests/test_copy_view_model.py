"""Models, in numpy, of the two copy geometries the TMA kernels rely on,
checked against the oracle and against plain indexing (no GPU).

1. Q-Shift through the flat token view.  Where the image view cannot serve
   (W not a multiple of 8 or above 256), a shifted tile is the plain tile's
   boxes displaced by the group's token offset (-s, +s, -s*W, +s*W), loaded
   with zero fill outside [0, T); for the horizontal groups the first or last
   min(s, W) tokens of every image row are then cleared.  This model applies
   that rule to every channel group and compares it with the oracle's Q-Shift
   ("Vision-RWKV Backbone", Quad-Directional Token Shift, eq. 9; the q_shift
   listing of "LinXin's Blog"), with mu = 0 (the shifted tokens alone).

2. The residue-major views.  A tile is 8 sub-tiles, sub-tile i row m holding
   token 8 m + i of the CTA.  One TMA box fills the whole tile from the view
   (C, T/8, 8, B) with strides (8 C, C, T C) elements -- the residue axis
   outermost in the box -- or, with Q-Shift, from the image view
   (C, W/8, H, 8, B) with strides (8 C, W C, C, H W C).  The model builds the
   box with numpy strides (a box fills shared memory innermost dimension
   first) and checks it against the layout the kernels read.
"""
import numpy as np
import pytest

import oracle


def _flat_shift_model(x, H, W, s, gamma):
    """The kernels' flat-view Q-Shift (mu = 0) of x (B, T, C)."""
    B, T, C = x.shape
    b = [int(C * gamma * (j + 1)) for j in range(4)]
    out = np.empty_like(x)
    t = np.arange(T)
    w = t % W
    for c in range(C):
        grp = sum(c >= bj for bj in b)
        if grp >= 4:
            out[:, :, c] = x[:, :, c]
            continue
        dt = [-s, s, -s * W, s * W][grp]
        src = t + dt
        ok = (src >= 0) & (src < T)             # the TMA's zero fill outside [0, T)
        col = np.zeros((B, T))
        col[:, ok] = x[:, src[ok], c]
        sw = min(s, W)
        if grp == 0:
            col[:, w < sw] = 0.0                # row-wrapped: source left of the row
        elif grp == 1:
            col[:, w >= W - sw] = 0.0           # row-wrapped: source right of the row
        out[:, :, c] = col
    return out


@pytest.mark.parametrize("H,W,s", [(14, 14, 1), (3, 11, 2), (5, 7, 3), (4, 4, 5), (2, 300, 3),
                                   (6, 1, 1), (1, 9, 1), (10, 13, 4), (8, 64, 70)])
@pytest.mark.parametrize("gamma", [0.25, 0.125])
def test_flat_view_rule_is_q_shift(H, W, s, gamma):
    rng = np.random.default_rng(H * 1000 + W * 10 + s)
    C = 16
    x = rng.standard_normal((2, H * W, C))
    want = oracle.qshift(x, H, W, s, gamma, mu=np.zeros(C))
    np.testing.assert_array_equal(_flat_shift_model(x, H, W, s, gamma), want)


def test_flat_view_rule_fails_without_the_row_clearing():
    # the displaced boxes alone carry tokens across image rows: the clearing
    # step is what makes them eq. 9
    H, W, s = 6, 10, 1
    rng = np.random.default_rng(5)
    x = rng.standard_normal((1, H * W, 4))
    want = oracle.qshift(x, H, W, s, 0.25, mu=np.zeros(4))
    t = np.arange(H * W)
    shifted = np.zeros(H * W)
    shifted[1:] = x[0, :-1, 0]               # group 0: source t - 1
    assert not np.array_equal(shifted, want[0, :, 0])


def _box(base, strides, box, start):
    """Elements a TMA box of the given extents reads, innermost first, from a
    view with element strides; out-of-range coordinates read as zero."""
    dims, ext = box
    out = np.zeros(tuple(reversed(ext)), dtype=base.dtype)
    for idx in np.ndindex(*reversed(ext)):
        coord = [start[d] + idx[len(ext) - 1 - d] for d in range(len(ext))]
        if all(0 <= coord[d] < dims[d] for d in range(len(ext))):
            off = sum(coord[d] * strides[d] for d in range(len(ext)))
            out[idx] = base[off]
    return out


@pytest.mark.parametrize("T,t0", [(2048, 1024), (1280, 1024), (1000, 0)])
def test_residue_major_token_view(T, t0):
    C, c0, B, b, TC = 24, 8, 2, 1, 1024
    x = np.arange(B * T * C, dtype=np.int64)   # element = its own flat index
    dims = (C, T // 8, 8, B)
    strides = (1, 8 * C, C, T * C)
    box = _box(x, strides, (dims, (8, TC // 8, 8, 1)), (c0, t0 // 8, 0, b))
    # shared memory: [b][i][m][c] -> sub-tile i, row m holds token t0 + 8 m + i
    for i in range(8):
        for m in range(TC // 8):
            t = t0 + 8 * m + i
            want = [(b * T + t) * C + c0 + c for c in range(8)] if t < (T // 8) * 8 else [0] * 8
            assert list(box[0, i, m, :]) == want


@pytest.mark.parametrize("H,W,r0,rows", [(64, 64, 16, 16), (40, 32, 32, 32), (32, 128, 8, 8)])
def test_residue_major_image_view(H, W, r0, rows):
    C, c0, B, b = 16, 8, 2, 1
    T = H * W
    x = np.arange(B * T * C, dtype=np.int64)
    dims = (C, W // 8, H, 8, B)
    strides = (1, 8 * C, W * C, C, T * C)
    box = _box(x, strides, (dims, (8, W // 8, rows, 8, 1)), (c0, 0, r0, 0, b))
    # [b][i][h][m'][c] -> sub-tile i, row (h - r0) W / 8 + m' holds token h W + 8 m' + i
    for i in range(8):
        for hh in range(rows):
            for mp in range(W // 8):
                h = r0 + hh
                want = [(b * T + h * W + 8 * mp + i) * C + c0 + c for c in range(8)] if h < H else [0] * 8
                assert list(box[0, i, hh, mp, :]) == want
                # the same element at the flat token of the sub-tile row
                tl = hh * W + 8 * mp + i
                assert tl % 8 == i and tl // 8 == hh * (W // 8) + mp
