"""GPU parity of the Bi-WKV backward kernel (vrwkv_biwkv_bwd) against the
float64 oracle (the chain rule of eq. 5 of "Vision-RWKV Backbone", Linear
Complexity Bidirectional Attention, pinned by finite differences of the
forward oracle), on the same seeded inputs.

Error metric.  Every gradient is a sum of signed terms; its error is divided
by the sum of the absolute values of those terms (computed by the oracle), the
scale that float32 rounding error is proportional to.  Tolerances: 1e-4 for
float32 I/O; 2e-2 for dk and dv with bfloat16 I/O (one rounding at the
store), 1e-4 for dw and du in either (float32 outputs).  Small cases compare
every element; large ones every element of a seeded sample of columns.
"""
import zlib

import numpy as np
import pytest

from linear_complexity_vision_b200 import synth
from helpers import to_device, to_numpy, torch_dtype, vec_f32

pytestmark = pytest.mark.gpu

TOL_KV = {"f32": 1e-4, "bf16": 2e-2}
TOL_WU = 1e-4


@pytest.fixture(scope="module")
def vk():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import linear_complexity_vision_b200 as vk
    vk.load_library()
    return vk


@pytest.fixture(params=["tm", "8tok"])
def bwd_path(request, monkeypatch):
    """The default backward (the 16-token tensor-memory kernel where the
    inputs arrive by TMA and gk, gv are 16-byte aligned) and the 8-token
    kernel (VRWKV_BWD_TM=0)."""
    if request.param == "8tok":
        monkeypatch.setenv("VRWKV_BWD_TM", "0")
    else:
        monkeypatch.delenv("VRWKV_BWD_TM", raising=False)
    return request.param


def _inputs(B, T, C, dt, salt, kstd=1.0, w=("uniform", -5.0, 5.0)):
    seed = 20280000 + zlib.crc32(repr((B, T, C, dt, salt)).encode()) % 100000
    k = synth.draw(seed, "k", (B, T, C), ("normal", kstd))
    v = synth.draw(seed, "v", (B, T, C), ("normal", 1.0))
    g = synth.draw(seed, "x", (B, T, C), ("normal", 1.0))  # upstream gradient
    ww = synth.draw(seed, "w", (C,), w)
    u = synth.draw(seed, "u", (C,), ("normal", 1.0))
    return k, v, g, ww, u


def _run(vk, k, v, g, w, u, dt, offset=0):
    import torch
    B, T, C = k.shape
    dev = []
    host = []
    for a in (k, v, g):
        t, h = to_device(a, dt)
        if offset:
            buf = torch.empty(t.numel() + offset, dtype=torch_dtype(dt), device="cuda")
            s = buf[offset:].view(B, T, C)
            s.copy_(t)
            t = s
        dev.append(t)
        host.append(h)
    wt, wd = vec_f32(w)
    ut, ud = vec_f32(u)
    out = vk.biwkv_bwd(dev[0], dev[1], wt, ut, dev[2])
    vk.device_status()
    res = [to_numpy(x) for x in out[:4]] + [out[4].cpu().numpy(), out[5].cpu().numpy()]
    return res, host, wd, ud


def _check(vk, oracle, k, v, g, w, u, dt, cols=None, offset=0):
    B, T, C = k.shape
    (gk, gv, gw, gu, gwt, gut), (kd, vd, gd), wd, ud = _run(vk, k, v, g, w, u, dt, offset)
    if cols is None:
        cols = np.arange(B * C)
    ok, ov, ow, ou, (sk, sv, sw, su) = oracle.biwkv_bwd_columns(kd, vd, wd, ud, gd, cols,
                                                               with_scale=True)
    bb, cc = np.divmod(cols, C)
    tiny = 1e-30
    e_k = np.max(np.abs(gk[bb, :, cc] - ok) / np.maximum(sk, tiny))
    e_v = np.max(np.abs(gv[bb, :, cc] - ov) / np.maximum(sv, tiny))
    e_w = np.max(np.abs(gw[bb, cc] - ow) / np.maximum(sw, tiny))
    e_u = np.max(np.abs(gu[bb, cc] - ou) / np.maximum(su, tiny))
    assert np.all(np.isfinite(gk)) and np.all(np.isfinite(gv))
    assert e_k <= TOL_KV[dt], f"dk scaled error {e_k:.3e}"
    assert e_v <= TOL_KV[dt], f"dv scaled error {e_v:.3e}"
    assert e_w <= TOL_WU, f"dw scaled error {e_w:.3e}"
    assert e_u <= TOL_WU, f"du scaled error {e_u:.3e}"
    # the batch totals are the per-row parts summed in order
    np.testing.assert_allclose(gwt, gw.sum(axis=0, dtype=np.float64), rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(gut, gu.sum(axis=0, dtype=np.float64), rtol=1e-5, atol=1e-6)
    return gk, gv, gw, gu


SMALL = [
    # B, T, C
    (2, 1, 16),     # T = 1
    (2, 2, 16),     # T = 2: w drops out
    (1, 7, 5),      # ragged chunk, C odd (scalar loads)
    (3, 33, 17),    # C = 17: a half-filled channel slab
    (2, 196, 32),   # the 14 x 14 grid
    (1, 255, 16),
    (2, 256, 16),   # one full CTA
    (2, 257, 16),   # one token into a second CTA
    (1, 513, 40),   # three CTAs, ragged tail
    (1, 1000, 16),
]


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("B,T,C", SMALL)
def test_bwd_parity_small(vk, oracle_mod, dt, B, T, C, bwd_path):
    k, v, g, w, u = _inputs(B, T, C, dt, "small")
    _check(vk, oracle_mod, k, v, g, w, u, dt)


@pytest.mark.parametrize("dt,B,T,C", [("bf16", 4, 4096, 768), ("f32", 1, 4096, 64),
                                      ("bf16", 2, 3000, 48), ("f32", 8, 196, 384)])
def test_bwd_parity_large_sampled(vk, oracle_mod, dt, B, T, C, bwd_path):
    # the 64 x 64 grid at C = 768 (bf16) is the backward of the
    # biwkv_B4_T4096_C768_bf16 workload; every element of 24 sampled columns
    k, v, g, w, u = _inputs(B, T, C, dt, "large", kstd=2.0, w=("uniform", -8.0, 8.0))
    rng = np.random.default_rng(zlib.crc32(repr((dt, B, T, C)).encode()))
    cols = rng.choice(B * C, size=min(24, B * C), replace=False)
    _check(vk, oracle_mod, k, v, g, w, u, dt, cols=np.sort(cols))


@pytest.mark.parametrize("w_kind", ["zero", "huge_positive", "strong_negative"])
def test_bwd_decay_extremes(vk, oracle_mod, w_kind, bwd_path):
    T = 720
    d = {"zero": ("uniform", 0.0, 0.0), "huge_positive": ("uniform", 60.0 * T, 60.0 * T),
         "strong_negative": ("uniform", -20.0, -10.0)}[w_kind]
    k, v, g, w, u = _inputs(1, T, 32, "f32", w_kind, w=d)
    _check(vk, oracle_mod, k, v, g, w, u, "f32")


def test_bwd_shift_invariance_in_k(vk, oracle_mod, bwd_path):
    # adding 80 to every k would overflow e^k in float32 without the
    # maximum renormalisation; the gradients must not change
    k, v, g, w, u = _inputs(2, 600, 32, "f32", "shift")
    a = _check(vk, oracle_mod, k, v, g, w, u, "f32")
    b = _check(vk, oracle_mod, k + 80.0, v, g, w, u, "f32")
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, rtol=2e-4, atol=2e-5)


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_bwd_unaligned(vk, oracle_mod, dt, bwd_path):
    # element-aligned tensors that are not pair-aligned take scalar loads
    k, v, g, w, u = _inputs(2, 300, 32, dt, "unaligned")
    _check(vk, oracle_mod, k, v, g, w, u, dt, offset=1)


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("B,T,C", [(2, 1000, 16), (1, 4096, 24), (2, 257, 8)])
def test_bwd_tma_store_path(vk, oracle_mod, monkeypatch, dt, B, T, C):
    # the optional TMA-store output path (VRWKV_BWD_TMA_STORE=1) against the
    # oracle: full CTAs, a ragged last CTA and a single short column
    monkeypatch.setenv("VRWKV_BWD_TMA_STORE", "1")
    monkeypatch.setenv("VRWKV_BWD_TM", "0")  # an option of the 8-token kernel
    k, v, g, w, u = _inputs(B, T, C, dt, "tma_store")
    _check(vk, oracle_mod, k, v, g, w, u, dt)


def test_bwd_deterministic(vk, oracle_mod, bwd_path):
    k, v, g, w, u = _inputs(2, 1024, 64, "bf16", "det")
    a, _, _, _ = _run(vk, k, v, g, w, u, "bf16")
    b, _, _, _ = _run(vk, k, v, g, w, u, "bf16")
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)
    want = "biwkv_bwd_tm_kernel" if bwd_path == "tm" else "biwkv_bwd_kernel"
    assert vk.load_library().vrwkv_last_kernel().decode() == want


def test_bwd_matches_autograd_of_forward_kernel_shape(vk, oracle_mod):
    # consistency between the two CUDA entry points: for a linear loss
    # L = sum(gy * wkv), a small step along dv changes L by <dv, step>
    import torch
    B, T, C = 1, 300, 32
    k, v, g, w, u = _inputs(B, T, C, "f32", "consistency")
    kt, _ = to_device(k, "f32")
    vt, _ = to_device(v, "f32")
    gt, _ = to_device(g, "f32")
    wt, _ = vec_f32(w)
    ut, _ = vec_f32(u)
    _, gv, _, _, _, _ = vk.biwkv_bwd(kt, vt, wt, ut, gt)
    step = torch.from_numpy(synth.draw(5, "v", (B, T, C), ("normal", 1.0))).float().cuda()
    h = 1e-2
    lp = torch.sum(gt.double() * vk.biwkv_fwd(kt, vt + h * step, wt, ut).double())
    lm = torch.sum(gt.double() * vk.biwkv_fwd(kt, vt - h * step, wt, ut).double())
    fd = float((lp - lm) / (2 * h))
    an = float(torch.sum(gv.double() * step.double()))
    assert abs(fd - an) <= 1e-3 * max(1.0, abs(an))
