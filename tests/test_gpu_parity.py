"""GPU parity: the CUDA path through the C ABI against the float64 oracle,
element by element, on the same seeded inputs.

Q-Shift must be bit-exact.  Bi-WKV and the gated core must stay within a
scaled error (see helpers.py) of 1e-4 for float32 I/O and 2e-2 for bfloat16
I/O.  Small cases compare every element with eq. 5 evaluated directly; large
cases compare every element with the RNN form (eq. 6-7, itself pinned to
eq. 5 by the CPU tests) and a seeded sample of elements with eq. 5 directly.
"""
import zlib

import numpy as np
import pytest

from linear_complexity_vision_b200 import synth
from helpers import (TOL, plain_relative_error, biwkv_scale, scaled_error, to_device, to_numpy, torch_dtype,
                     vec_f32)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def vk():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import linear_complexity_vision_b200 as vk
    vk.load_library()
    return vk


# ---------------------------------------------------------------------------
# Q-Shift: bit-exact
# ---------------------------------------------------------------------------
QS_CASES = [
    (2, 14, 14, 384, 1, 0.25),   # the 224^2 grid
    (3, 5, 7, 13, 1, 0.25),      # odd C: scalar path
    (1, 4, 6, 40, 2, 0.25),      # shift 2
    (2, 3, 3, 16, 3, 0.25),      # shift >= H and >= W: empty groups
    (1, 1, 9, 24, 1, 0.25),      # H = 1
    (1, 9, 1, 24, 1, 0.25),      # W = 1
    (1, 8, 8, 20, 1, 0.2),       # g = 4
    (1, 8, 8, 24, 1, 0.25),      # g = 6: vectors straddle group boundaries
    (2, 6, 6, 32, 0, 0.25),      # shift 0
    (1, 6, 6, 32, 1, 0.0),       # gamma 0: every channel copied
    (2, 64, 64, 1024, 1, 0.25),  # the 1024^2 grid at C = 1024
    # the listing's bounds int(C*gamma*j) where C*gamma is not an integer
    (2, 3, 4, 10, 2, 0.25),      # bounds 2, 5, 7, 10
    (1, 5, 6, 50, 1, 0.145),     # double rounding: last bound 28, channels 28.. copied
    (2, 8, 8, 48, 1, 0.125),     # bounds 6, 12, 18, 24: vectors straddle, 24.. copied
    (1, 8, 8, 64, 1, 0.125),     # bounds 8, 16, 24, 32: half the channels copied
    (2, 4, 5, 26, 1, 0.25),      # bounds 6, 13, 19, 26
]


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("use_mu", [True, False])
@pytest.mark.parametrize("B,H,W,C,s,gamma", QS_CASES)
def test_qshift_bit_exact(vk, oracle_mod, dt, use_mu, B, H, W, C, s, gamma):
    seed = 1000 + B * 7 + H * 13 + W * 17 + C + s
    x = synth.draw(seed, "x", (B, H * W, C), ("normal", 1.0))
    mu = synth.draw(seed, "mu_k", (C,), ("uniform", 0.0, 1.0))
    xt, xd = to_device(x, dt)
    mut, mud = vec_f32(mu)
    out = vk.qshift(xt, H, W, s, gamma, mu=mut if use_mu else None)
    want = oracle_mod.qshift_f32(xd.astype(np.float32), H, W, s, gamma,
                                 mu=mud.astype(np.float32) if use_mu else None,
                                 round_bf16=(dt == "bf16"))
    np.testing.assert_array_equal(to_numpy(out), want.astype(np.float64))


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_qshift_unaligned_pointers(vk, oracle_mod, dt):
    import torch
    B, H, W, C = 2, 5, 6, 32
    x = synth.draw(5, "x", (B, H * W, C), ("normal", 1.0))
    mu = synth.draw(5, "mu_k", (C,), ("uniform", 0.0, 1.0))
    xt, xd = to_device(x, dt)
    buf = torch.empty(B * H * W * C + 1, dtype=torch_dtype(dt), device="cuda")
    xs = buf[1:].view(B, H * W, C)
    xs.copy_(xt)
    obuf = torch.empty_like(buf)
    os_ = obuf[1:].view(B, H * W, C)
    mut, mud = vec_f32(mu)
    vk.qshift(xs, H, W, 1, 0.25, mu=mut, out=os_)
    want = oracle_mod.qshift_f32(xd.astype(np.float32), H, W, 1, 0.25, mu=mud.astype(np.float32),
                                 round_bf16=(dt == "bf16"))
    np.testing.assert_array_equal(to_numpy(os_), want.astype(np.float64))


# ---------------------------------------------------------------------------
# Fused Bi-WKV / spatial gate
# ---------------------------------------------------------------------------
def _custom(call, B, H, W, C, dt, seed, s=1, gamma=0.25, **d):
    dists = {"x": ("normal", 1.0), "r": ("normal", 1.0), "k": ("normal", 1.0),
             "v": ("normal", 1.0), "w": ("uniform", -5.0, 5.0), "u": ("normal", 1.0)}
    dists.update(d)
    return synth.Workload(f"{call}_{B}x{H}x{W}x{C}_{dt}", B, H, W, C, dt, call, dists,
                          shift_pixel=s, gamma=gamma, seed=seed)


# The last run_fused call's error figures (for tests that report them).
_LAST = {}


# Workspace of the global-exchange kernels, shared by every "gx" test on the
# one stream (the kernels leave it ready for the next call).
_GX = {"on": False, "ws": None}


def _workspace(vk, B, T, C):
    need = vk.fwd_workspace_bytes(B, T, C)
    if _GX["ws"] is None or _GX["ws"].numel() < need:
        import torch
        _GX["ws"] = torch.zeros(max(need, 64 << 20), dtype=torch.uint8, device="cuda")
    return _GX["ws"]


def run_fused(vk, oracle, wl, mu_none=False, kshift=0.0, return_out=False):
    """Run the workload's call on the GPU and compare with the oracle."""
    inp = wl.generate()
    dt = wl.dtype
    dev, ref = {}, {}
    for name in wl.tensor_names():
        a = inp[name] + (kshift if name in ("k", "x") and wl.call == "biwkv" else 0.0)
        dev[name], ref[name] = to_device(a, dt)
    for name in ("w", "u", "mu_r", "mu_k", "mu_v"):
        if name in inp:
            dev[name], ref[name] = vec_f32(inp[name])
    if mu_none:
        for name in ("mu_r", "mu_k", "mu_v"):
            dev[name] = None
            ref[name] = None
    H, W, s, g = wl.H, wl.W, wl.shift_pixel, wl.gamma
    w, u = ref["w"], ref["u"]

    ws = _workspace(vk, wl.B, wl.T, wl.C) if _GX["on"] else None
    if wl.call == "biwkv":
        out = vk.biwkv_fwd(dev["k"], dev["v"], dev["w"], dev["u"], workspace=ws)
        ks, vs, rs = ref["k"], ref["v"], None
    elif wl.call == "gate":
        out = vk.spatial_gate(dev["r"], dev["k"], dev["v"], dev["w"], dev["u"], workspace=ws)
        ks, vs, rs = ref["k"], ref["v"], ref["r"]
    elif wl.call == "gate_x":
        x = dev["x"]
        out = vk.spatial_gate(x, x, x, dev["w"], dev["u"], workspace=ws)
        ks = vs = rs = ref["x"]
    else:
        qs = vk.QShift(H, W, s, g, dev.get("mu_r"), dev.get("mu_k"), dev.get("mu_v"))
        if wl.call == "qshift_biwkv":
            out = vk.biwkv_fwd(dev["k"], dev["v"], dev["w"], dev["u"], qs=qs, workspace=ws)
            kin, vin, rin = ref["k"], ref["v"], None
        elif wl.call == "gate_qs":
            out = vk.spatial_gate(dev["r"], dev["k"], dev["v"], dev["w"], dev["u"], qs=qs,
                                  workspace=ws)
            kin, vin, rin = ref["k"], ref["v"], ref["r"]
        else:  # gate_qs_x: one x feeds r, k and v
            x = dev["x"]
            out = vk.spatial_gate(x, x, x, dev["w"], dev["u"], qs=qs, workspace=ws)
            kin = vin = rin = ref["x"]
        ks = oracle.qshift(kin, H, W, s, g, ref["mu_k"])
        vs = oracle.qshift(vin, H, W, s, g, ref["mu_v"])
        rs = None if rin is None else oracle.qshift(rin, H, W, s, g, ref["mu_r"])
    vk.device_status()  # no kernel's bounded wait ran out
    got = to_numpy(out)
    assert np.isfinite(got).all()

    B, T, C = ks.shape
    small = B * C * T * T <= 4e8
    want = oracle.biwkv_direct(ks, vs, w, u) if small else oracle.biwkv_rnn(ks, vs, w, u)
    scale = biwkv_scale(oracle, ks, vs, w, u)
    if rs is not None:
        want = oracle.gate(rs, want)
        scale = oracle.gate(rs, scale)
    tol = TOL[dt]
    err = scaled_error(got, want, scale)
    assert err <= tol, f"{wl.name}: scaled error {err:.3e} > {tol}"
    # the plain relative error where the weighted mean does not cancel
    # (|wkv| at least half the weighted mean of |v|): bounded by 2 tol
    well = np.abs(want) >= 0.5 * scale
    if well.any():
        plain = plain_relative_error(got[well], want[well])
        assert plain <= 2 * tol, f"{wl.name}: plain relative error {plain:.3e} > {2 * tol}"
    _LAST["plain_all"] = plain_relative_error(got, want)
    _LAST["plain_well"] = plain_relative_error(got[well], want[well]) if well.any() else 0.0
    _LAST["scaled"] = err
    if not small:
        rng = np.random.default_rng(wl.seed)
        idx = rng.choice(got.size, size=min(got.size, 3000), replace=False)
        pts = oracle.biwkv_points(ks, vs, w, u, idx)
        if rs is not None:
            pts = oracle.gate(rs.reshape(-1)[idx], pts)
        perr = scaled_error(got.reshape(-1)[idx], pts, scale.reshape(-1)[idx])
        assert perr <= tol, f"{wl.name}: sampled eq. 5 error {perr:.3e} > {tol}"
    return (got, err) if return_out else err


@pytest.fixture(params=["default", "narrow", "flat", "tm", "wide", "tma8", "gx", "generic"])
def kernel_path(request, monkeypatch):
    """Run a test on the default path (the 32-token tensor-memory kernel for
    columns of more than 512 tokens, else the 8-channel TMA kernel with
    16-token thread chunks, on 256-token CTAs for columns of at most 256
    tokens, where the shape and cluster geometry allow), on the latter alone
    ("narrow"), on it with Q-Shift through the flat token view everywhere and
    512-token CTAs at any length ("flat"), on the tensor-memory kernel
    wherever it qualifies ("tm"), on the 16-channel slab kernel where the
    shape qualifies ("wide"), on the 8-channel kernel held to 8-token chunks,
    on its workspace variant (global-memory exchange instead of clusters) and
    with the generic kernel forced."""
    if request.param == "generic":
        monkeypatch.setenv("VRWKV_DISABLE_TMA", "1")
    else:
        monkeypatch.delenv("VRWKV_DISABLE_TMA", raising=False)
    if request.param == "tma8":
        monkeypatch.setenv("VRWKV_TMA_CHUNK", "8")
    else:
        monkeypatch.delenv("VRWKV_TMA_CHUNK", raising=False)
    if request.param == "flat":
        monkeypatch.setenv("VRWKV_QS_VIEW", "flat")
        monkeypatch.setenv("VRWKV_SHORT_CTA", "0")
    else:
        monkeypatch.delenv("VRWKV_QS_VIEW", raising=False)
        monkeypatch.delenv("VRWKV_SHORT_CTA", raising=False)
    forward = {"wide": "wide", "tm": "tm", "narrow": "narrow", "tma8": "narrow",
               "flat": "narrow"}.get(request.param)
    if forward:
        monkeypatch.setenv("VRWKV_FORWARD", forward)
    else:
        monkeypatch.delenv("VRWKV_FORWARD", raising=False)
    _GX["on"] = request.param == "gx"
    yield request.param
    _GX["on"] = False


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
def test_workload_full_size(vk, oracle_mod, cfg, kernel_path):
    wl = synth.WORKLOADS[cfg]
    run_fused(vk, oracle_mod, wl)


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
def test_plain_relative_error_reported(vk, oracle_mod, cfg, record_property, monkeypatch, capsys):
    # The parity bar is the scaled error (|delta| / S_t, S_t the eq. 5-weighted
    # mean of |v|); the plain max |delta| / max(|wkv|, 1e-6) is reported beside
    # it, over all outputs and over those where |wkv| >= S_t / 2.
    for name in ("VRWKV_FORWARD", "VRWKV_QS_VIEW", "VRWKV_SHORT_CTA", "VRWKV_DISABLE_TMA"):
        monkeypatch.delenv(name, raising=False)
    wl = synth.WORKLOADS[cfg]
    run_fused(vk, oracle_mod, wl)
    for k in ("scaled", "plain_all", "plain_well"):
        record_property(k, _LAST[k])
    with capsys.disabled():
        print(f"\n{wl.name}: scaled {_LAST['scaled']:.3e}, plain (all) {_LAST['plain_all']:.3e}, "
              f"plain (|wkv| >= S/2) {_LAST['plain_well']:.3e}")


@pytest.mark.parametrize("cfg", [4, 5])
def test_default_forward_is_the_tensor_memory_kernel(vk, oracle_mod, cfg, monkeypatch):
    monkeypatch.delenv("VRWKV_FORWARD", raising=False)
    wl = synth.WORKLOADS[cfg]
    run_fused(vk, oracle_mod, wl)
    assert vk.load_library().vrwkv_last_kernel().decode() == "biwkv_tm_kernel"


@pytest.mark.parametrize("cfg", [1, 2, 3])
def test_14x14_grids_take_the_8_channel_kernel(vk, oracle_mod, cfg, monkeypatch):
    # W = 14 is not a multiple of 8: Q-Shift goes through the flat token view
    for name in ("VRWKV_FORWARD", "VRWKV_QS_VIEW", "VRWKV_SHORT_CTA", "VRWKV_DISABLE_TMA"):
        monkeypatch.delenv(name, raising=False)
    wl = synth.WORKLOADS[cfg]
    run_fused(vk, oracle_mod, wl)
    assert vk.load_library().vrwkv_last_kernel().decode() == "biwkv_tma_kernel"


@pytest.mark.parametrize("cfg", [4, 5])
def test_forward_selection_takes_the_16_channel_kernel(vk, oracle_mod, cfg, monkeypatch):
    monkeypatch.setenv("VRWKV_FORWARD", "wide")
    wl = synth.WORKLOADS[cfg]
    run_fused(vk, oracle_mod, wl)
    assert vk.load_library().vrwkv_last_kernel().decode() == "biwkv_wide_kernel"


# Shapes aimed at the 16-channel slab kernel's geometry: rows of 16 to 64
# tokens (vertical halo of 1 to 4 chunks), a last CTA holding one chunk, 1 to
# 8 CTAs per column, copied channels (gamma = 1/8) and the three source
# layouts; `wide` says whether the shape qualifies for it.
WIDE_CASES = [
    # call, B, H, W, C, dtype, gamma, shift, wide
    ("gate_qs_x", 1, 32, 16, 64, "bf16", 0.25, 1, True),     # W = 16: one chunk per image row
    ("gate_qs", 2, 33, 16, 64, "f32", 0.25, 1, True),        # T = 528: the second CTA holds one chunk
    ("qshift_biwkv", 1, 64, 48, 64, "bf16", 0.25, 1, True),  # W = 48: halo of 3 chunks, 6 CTAs
    ("gate_qs_x", 2, 16, 32, 128, "f32", 0.125, 1, True),    # copied channels 64..127
    ("gate_qs_x", 1, 64, 64, 64, "bf16", 0.25, 2, False),    # shift 2 on the horizontal groups
    ("gate_qs", 1, 8, 64, 128, "bf16", 0.25, 1, True),       # one CTA
    ("biwkv", 3, 1, 2048, 32, "bf16", 0.25, 1, True),        # 4 CTAs, no Q-Shift
    ("biwkv", 1, 1, 1000, 32, "bf16", 0.25, 1, False),       # T not a multiple of 16
]


@pytest.mark.parametrize("case", WIDE_CASES, ids=lambda c: "_".join(map(str, c)))
def test_wide_kernel_shapes(vk, oracle_mod, case, monkeypatch):
    monkeypatch.setenv("VRWKV_FORWARD", "wide")
    call, B, H, W, C, dt, gamma, shift, wide = case
    wl = _custom(call, B, H, W, C, dt, seed=zlib.crc32(repr(case).encode()) % 100000, gamma=gamma, s=shift)
    run_fused(vk, oracle_mod, wl)
    got = vk.load_library().vrwkv_last_kernel().decode()
    assert (got == "biwkv_wide_kernel") == wide, got


# Shapes aimed at the 32-token tensor-memory kernel's geometry: 1024-token
# CTAs (16 image rows of 64), CTAs of 768 tokens (W = 48, 96), a last CTA
# holding one token, 8-CTA clusters at T = 8192, float32 tiles (three or one
# CTA per SM), separate r, k, v with Q-Shift (six tiles) and copied channels.
TM_CASES = [
    # call, B, H, W, C, dtype, gamma
    ("gate_qs_x", 1, 128, 64, 64, "bf16", 0.25),   # T = 8192: 8 CTAs
    ("biwkv", 2, 1, 8192, 16, "f32", 0.25),        # 8 CTAs, no Q-Shift, float32
    ("biwkv", 1, 1, 2049, 16, "bf16", 0.25),       # the third CTA holds one token
    ("gate_qs", 1, 32, 96, 32, "f32", 0.25),       # W = 96: CTAs of 8 rows (768 tokens)
    ("gate_qs_x", 2, 48, 48, 32, "bf16", 0.25),    # W = 48: CTAs of 16 rows (768 tokens)
    ("qshift_biwkv", 1, 32, 64, 64, "bf16", 0.25),  # no gate, Q-Shift
    ("gate_qs_x", 1, 64, 64, 128, "bf16", 0.125),  # copied channels 64..127
    ("gate_qs", 2, 64, 64, 32, "bf16", 0.25),      # r, k, v with Q-Shift: six tiles
    ("gate_qs_x", 1, 12, 16, 64, "bf16", 0.25),    # T = 192: one CTA, 6 of 32 chunks used
    ("gate", 2, 1, 4096, 64, "bf16", 0.25),        # r, k, v without Q-Shift: gate in k's slots
    ("gate", 1, 1, 3000, 32, "f32", 0.25),         # the same in float32, ragged last CTA
    ("gate_x", 2, 1, 4096, 32, "bf16", 0.25),      # one x without Q-Shift: gate in an extra tile
    ("gate_qs_x", 1, 36, 36, 64, "bf16", 0.25),    # W = 36: flat token view, 2 CTAs
    ("gate_qs", 1, 45, 50, 32, "f32", 0.25),       # W = 50: flat view in float32, 3 CTAs
    ("qshift_biwkv", 2, 14, 14, 64, "bf16", 0.25),  # 14 x 14: flat view, one CTA
]


@pytest.mark.parametrize("rot", ["rot", "natural"])
@pytest.mark.parametrize("case", TM_CASES, ids=lambda c: "_".join(map(str, c)))
def test_tm_kernel_shapes(vk, oracle_mod, case, rot, monkeypatch):
    # "rot": the rotated sub-chunk order wherever it is planned (bfloat16
    # rows, room for the stash); "natural": sub-chunks in order everywhere
    monkeypatch.setenv("VRWKV_FORWARD", "tm")
    monkeypatch.setenv("VRWKV_TM_ROT", "1" if rot == "rot" else "0")
    call, B, H, W, C, dt, gamma = case
    wl = _custom(call, B, H, W, C, dt, seed=zlib.crc32(repr(case).encode()) % 100000, gamma=gamma)
    run_fused(vk, oracle_mod, wl)
    assert vk.load_library().vrwkv_last_kernel().decode() == "biwkv_tm_kernel"


# The default selection on both sides of its switch: the 8-channel kernel up
# to 512 tokens, the tensor-memory kernel (one CTA per column) above.
SWITCH_CASES = [
    # call, B, H, W, C, dtype, kernel
    ("gate_qs_x", 2, 16, 32, 64, "bf16", "biwkv_tma_kernel"),   # T = 512
    ("biwkv", 2, 1, 512, 16, "f32", "biwkv_tma_kernel"),         # T = 512, no Q-Shift
    ("biwkv", 2, 1, 513, 16, "bf16", "biwkv_tm_kernel"),         # T = 513: 17 chunks, one holding a token
    ("gate_qs_x", 2, 24, 32, 64, "bf16", "biwkv_tm_kernel"),    # T = 768, image view
    ("gate_qs", 1, 25, 40, 32, "f32", "biwkv_tm_kernel"),       # T = 1000, W = 40: flat view
]


@pytest.mark.parametrize("case", SWITCH_CASES, ids=lambda c: "_".join(map(str, c[:6])))
def test_default_forward_switch(vk, oracle_mod, case, monkeypatch):
    for name in ("VRWKV_FORWARD", "VRWKV_QS_VIEW", "VRWKV_SHORT_CTA", "VRWKV_DISABLE_TMA", "VRWKV_TM_ROT"):
        monkeypatch.delenv(name, raising=False)
    call, B, H, W, C, dt, kernel = case
    wl = _custom(call, B, H, W, C, dt, seed=zlib.crc32(repr(case).encode()) % 100000)
    run_fused(vk, oracle_mod, wl)
    assert vk.load_library().vrwkv_last_kernel().decode() == kernel


# The tensor-memory kernel's copy shapes: each tile in one residue-major box
# (image view with Q-Shift, flat tokens without or at any W) or in
# lane-strided boxes, and results stored in one residue-major box or in
# lane-strided 256-token boxes.
COPY_CASES = [
    # call, B, H, W, C, dtype
    ("gate_qs_x", 2, 64, 64, 64, "bf16"),     # image view, 16 rows per CTA
    ("gate_qs", 1, 32, 32, 32, "f32"),        # image view, 32 rows per CTA, float32
    ("qshift_biwkv", 1, 48, 96, 32, "bf16"),  # W = 96: 768-token CTAs (lane-strided loads only)
    ("biwkv", 2, 1, 3072, 32, "bf16"),        # flat tokens, 3 CTAs
    ("gate_x", 1, 1, 1288, 16, "f32"),        # flat tokens, a second CTA of 264 tokens
    ("gate_qs_x", 1, 40, 40, 32, "bf16"),     # W = 40: flat view, shifted tiles lane-strided
    ("gate", 1, 1, 1000, 16, "bf16"),         # one CTA of 1000 tokens
]


@pytest.mark.parametrize("ostore", ["1", "0"])
@pytest.mark.parametrize("imaj", ["1", "0"])
@pytest.mark.parametrize("case", COPY_CASES, ids=lambda c: "_".join(map(str, c)))
def test_tm_copy_shapes(vk, oracle_mod, case, imaj, ostore, monkeypatch):
    monkeypatch.setenv("VRWKV_FORWARD", "tm")
    monkeypatch.setenv("VRWKV_TM_IMAJ", imaj)
    monkeypatch.setenv("VRWKV_TM_OSTORE", ostore)
    call, B, H, W, C, dt = case
    wl = _custom(call, B, H, W, C, dt, seed=zlib.crc32(repr(case).encode()) % 100000)
    run_fused(vk, oracle_mod, wl)
    assert vk.load_library().vrwkv_last_kernel().decode() == "biwkv_tm_kernel"


# Sequences past 4096 tokens: the pages' efficiency comparison runs 2048^2
# images at patch 16, T = 16384 ("Vision-RWKV Backbone", Ablation /
# efficiency analysis, Fig. 3(b)).  With a workspace the 16-channel kernel
# splits a column into segments of one 8-CTA cluster (4096 tokens) that meet
# through it; checked against the RNN form over every output and eq. 5 at
# sampled positions.
LONG_CASES = [
    # call, B, H, W, C, dtype
    ("gate_qs_x", 1, 128, 128, 64, "bf16"),   # T = 16384: four segments
    ("gate_qs", 1, 128, 64, 64, "f32"),       # T = 8192: two segments
    ("biwkv", 2, 1, 12288, 16, "bf16"),       # T = 12288: three segments, no Q-Shift
    ("gate_qs_x", 1, 72, 64, 64, "bf16"),     # T = 4608: the last segment holds one CTA's tokens
    ("qshift_biwkv", 1, 256, 128, 64, "bf16"),  # T = 32768: eight segments
]


@pytest.mark.parametrize("case", LONG_CASES, ids=lambda c: "_".join(map(str, c)))
def test_long_sequences_with_workspace(vk, oracle_mod, case):
    call, B, H, W, C, dt = case
    wl = _custom(call, B, H, W, C, dt, seed=zlib.crc32(repr(case).encode()) % 100000)
    _GX["on"] = True
    try:
        run_fused(vk, oracle_mod, wl)
    finally:
        _GX["on"] = False
    assert vk.load_library().vrwkv_last_kernel().decode() == "biwkv_wide_kernel"


def test_long_sequence_without_workspace_is_refused(vk):
    import torch
    x = torch.zeros(1, 16384, 64, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(64, device="cuda")
    with pytest.raises(vk.VrwkvError) as ei:
        vk.spatial_gate(x, x, x, w, w)
    assert ei.value.status == 2  # VRWKV_ERR_UNSUPPORTED


def test_workload2_qshift_of_x_full_size(vk, oracle_mod):
    wl = synth.WORKLOADS[2]
    inp = wl.generate()
    xt, xd = to_device(inp["x"], "f32")
    mut, mud = vec_f32(inp["mu_r"])
    out = vk.qshift(xt, wl.H, wl.W, 1, 0.25, mu=mut)
    want = oracle_mod.qshift_f32(xd.astype(np.float32), wl.H, wl.W, 1, 0.25,
                                 mu=mud.astype(np.float32))
    np.testing.assert_array_equal(to_numpy(out), want.astype(np.float64))


EDGE = [
    # call, B, H, W, C, dtype
    ("biwkv", 2, 1, 1, 16, "f32"),          # T = 1
    ("biwkv", 2, 1, 2, 16, "f32"),          # T = 2
    ("biwkv", 1, 1, 7, 5, "f32"),           # one ragged chunk, C odd
    ("biwkv", 3, 3, 11, 17, "f32"),         # T = 33, C = 17
    ("biwkv", 1, 1, 1, 1, "bf16"),          # smallest problem
    ("biwkv", 2, 27, 19, 40, "bf16"),       # T = 513: two CTAs, ragged tail
    ("biwkv", 2, 25, 40, 32, "f32"),        # T = 1000
    ("biwkv", 1, 64, 64, 32, "f32"),        # T = 4096 in float32
    ("biwkv", 1, 50, 60, 24, "bf16"),       # T = 3000
    ("qshift_biwkv", 2, 1, 9, 24, "f32"),   # H = 1
    ("qshift_biwkv", 2, 9, 1, 24, "f32"),   # W = 1
    ("qshift_biwkv", 2, 20, 31, 40, "f32"), # T = 620: halo across CTAs
    ("qshift_biwkv", 1, 64, 64, 48, "f32"), # 8 CTAs, halo 64
    ("gate_qs", 2, 7, 9, 20, "bf16"),
    ("gate_qs", 1, 33, 33, 24, "bf16"),     # T = 1089: 3 CTAs
    ("gate_qs_x", 2, 14, 14, 96, "bf16"),
    ("gate_qs_x", 1, 40, 40, 64, "f32"),    # T = 1600 in float32
    ("gate_qs_x", 1, 3, 11, 6, "bf16"),
    ("gate_qs_x", 2, 16, 16, 64, "bf16"),   # T = 256: half a CTA
    ("gate_qs_x", 1, 40, 40, 64, "bf16"),   # W = 40: 8-token chunks, 5-CTA cluster
    ("gate_qs", 2, 64, 64, 64, "bf16"),     # 8-CTA cluster, separate r, k, v
    ("qshift_biwkv", 1, 48, 64, 64, "bf16"),
    ("qshift_biwkv", 2, 24, 24, 64, "f32"),  # W = 24: 8 rows of 24 per CTA
    ("biwkv", 2, 1, 4096, 16, "bf16"),      # 8 CTAs without Q-Shift
    ("biwkv", 3, 1, 257, 32, "f32"),        # one token into a second CTA
    ("gate", 2, 1, 2048, 16, "bf16"),       # r, k, v without Q-Shift
    ("gate_x", 1, 1, 700, 24, "f32"),       # one x without Q-Shift, ragged
]


@pytest.mark.parametrize("case", EDGE, ids=lambda c: "_".join(map(str, c)))
def test_edge_shapes(vk, oracle_mod, case, kernel_path):
    call, B, H, W, C, dt = case
    wl = _custom(call, B, H, W, C, dt, seed=zlib.crc32(repr(case).encode()) % 100000)
    run_fused(vk, oracle_mod, wl)


@pytest.mark.parametrize("s,H,W", [(2, 6, 7), (3, 2, 300), (5, 4, 4), (2, 32, 64), (70, 8, 64), (3, 10, 13)])
def test_large_shifts(vk, oracle_mod, s, H, W, kernel_path):
    # C = 64: group bounds 16, 32, 48, 64, so the TMA kernels qualify (through
    # the flat token view where W is not a multiple of 8 or exceeds 256)
    C = 64
    wl = _custom("gate_qs", 1, H, W, C, "bf16", seed=77 + s, s=s)
    run_fused(vk, oracle_mod, wl)
    wl = _custom("gate_qs_x", 1, H, W, C, "f32", seed=78 + s, s=s)
    run_fused(vk, oracle_mod, wl)


# Channel groups at the listing's bounds int(C*gamma*j): unequal groups when
# C*gamma is not an integer, copied channels when gamma < 1/4, on the generic
# kernel and (bounds all multiples of 8) on the TMA path.
LISTING_BOUNDS = [
    # call, B, H, W, C, dtype, gamma
    ("gate_qs_x", 1, 8, 16, 10, "bf16", 0.25),       # bounds 2, 5, 7, 10
    ("gate_qs", 2, 12, 16, 26, "f32", 0.25),         # bounds 6, 13, 19, 26
    ("qshift_biwkv", 1, 16, 16, 50, "f32", 0.145),   # bounds 7, 14, 21, 28
    ("gate_qs_x", 2, 32, 32, 96, "bf16", 0.125),     # bounds 12, 24, 36, 48
    ("gate_qs_x", 1, 64, 64, 64, "bf16", 0.125),     # TMA path: 8, 16, 24, 32
    ("gate_qs", 2, 16, 64, 192, "bf16", 0.125),      # TMA path: 24, 48, 72, 96
]


@pytest.mark.parametrize("case", LISTING_BOUNDS, ids=lambda c: "_".join(map(str, c)))
def test_listing_group_bounds(vk, oracle_mod, case, kernel_path):
    call, B, H, W, C, dt, gamma = case
    wl = _custom(call, B, H, W, C, dt, seed=zlib.crc32(repr(case).encode()) % 100000, gamma=gamma)
    run_fused(vk, oracle_mod, wl)


def test_mu_none_is_pure_shift(vk, oracle_mod):
    wl = _custom("gate_qs", 2, 10, 10, 32, "f32", seed=91)
    run_fused(vk, oracle_mod, wl, mu_none=True)
    wl = _custom("qshift_biwkv", 1, 30, 30, 16, "f32", seed=92)
    run_fused(vk, oracle_mod, wl, mu_none=True)


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_shift_invariance_in_k(vk, oracle_mod, dt, kernel_path):
    # adding 80 to every k would overflow exp(k) in float32 without the
    # running-maximum renormalisation; the result must not change
    wl = _custom("biwkv", 2, 40, 40, 32, dt, seed=93)
    a, _ = run_fused(vk, oracle_mod, wl, return_out=True)
    b, _ = run_fused(vk, oracle_mod, wl, kshift=80.0, return_out=True)
    # each run matched the oracle on its own inputs above; in bfloat16, k + 80
    # is re-rounded (ulp 0.5 at 80), so only float32 inputs stay comparable
    if dt == "f32":
        assert np.max(np.abs(a - b)) <= 1e-5


@pytest.mark.parametrize("w_kind", ["zero", "huge_positive", "strong_negative"])
def test_decay_extremes(vk, oracle_mod, w_kind, kernel_path):
    T = 24 * 30
    d = {"zero": ("uniform", 0.0, 0.0), "huge_positive": ("uniform", 60.0 * T, 60.0 * T),
         "strong_negative": ("uniform", -20.0, -10.0)}[w_kind]
    wl = _custom("biwkv", 1, 24, 30, 32, "f32", seed=94, w=d)
    run_fused(vk, oracle_mod, wl)


def test_large_bonus(vk, oracle_mod):
    wl = _custom("biwkv", 1, 16, 16, 16, "f32", seed=95, u=("uniform", 30.0, 40.0))
    run_fused(vk, oracle_mod, wl)


def test_deterministic(vk):
    import torch
    wl = synth.workload(5, B=2, H=64, W=64, C=64)
    inp = wl.generate()
    x, _ = to_device(inp["x"], "bf16")
    f = {k: vec_f32(inp[k])[0] for k in ("w", "u", "mu_r", "mu_k", "mu_v")}
    qs = vk.QShift(64, 64, 1, 0.25, f["mu_r"], f["mu_k"], f["mu_v"])
    a = vk.spatial_gate(x, x, x, f["w"], f["u"], qs=qs)
    b = vk.spatial_gate(x, x, x, f["w"], f["u"], qs=qs)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_unaligned_fused(vk, oracle_mod):
    import torch
    wl = _custom("gate_qs_x", 1, 12, 12, 32, "bf16", seed=96)
    inp = wl.generate()
    xt, xd = to_device(inp["x"], "bf16")
    buf = torch.empty(xt.numel() + 1, dtype=torch.bfloat16, device="cuda")
    xs = buf[1:].view(xt.shape)
    xs.copy_(xt)
    obuf = torch.empty_like(buf)
    os_ = obuf[1:].view(xt.shape)
    f = {k: vec_f32(inp[k]) for k in ("w", "u", "mu_r", "mu_k", "mu_v")}
    qs = vk.QShift(12, 12, 1, 0.25, f["mu_r"][0], f["mu_k"][0], f["mu_v"][0])
    vk.spatial_gate(xs, xs, xs, f["w"][0], f["u"][0], qs=qs, out=os_)
    ref = {k: v[1] for k, v in f.items()}
    want = oracle_mod.spatial_core(xd, xd, xd, ref["w"], ref["u"], 12, 12, 1, 0.25,
                                   ref["mu_r"], ref["mu_k"], ref["mu_v"])
    ks = oracle_mod.qshift(xd, 12, 12, 1, 0.25, ref["mu_k"])
    vs = oracle_mod.qshift(xd, 12, 12, 1, 0.25, ref["mu_v"])
    rs = oracle_mod.qshift(xd, 12, 12, 1, 0.25, ref["mu_r"])
    scale = oracle_mod.gate(rs, biwkv_scale(oracle_mod, ks, vs, ref["w"], ref["u"]))
    assert scaled_error(to_numpy(os_), want, scale) <= TOL["bf16"]


def test_invalid_arguments_raise(vk):
    import torch
    x = torch.zeros(1, 12, 8, device="cuda")
    w = torch.zeros(8, device="cuda")
    with pytest.raises(vk.VrwkvError, match="H\\*W"):
        vk.biwkv_fwd(x, x, w, w, qs=vk.QShift(3, 5))
    with pytest.raises(vk.VrwkvError, match="overlaps"):
        vk.biwkv_fwd(x, x, w, w, out=x)


def test_workspace_reuse_across_launches(vk, oracle_mod, monkeypatch):
    # the global-exchange kernels (the 32-token one at T = 4096, the 8-channel
    # one at T = 1600) reset their counters and advance a generation at the
    # end of every launch: back-to-back launches on one workspace (different
    # shapes, then the same one again) stay exact, and equal the same
    # kernel's cluster exchange bit for bit
    import torch
    ws = torch.zeros(vk.fwd_workspace_bytes(8, 4096, 1024), dtype=torch.uint8, device="cuda")
    outs = []
    for B, H, W, C in [(2, 64, 64, 64), (1, 40, 40, 64), (2, 64, 64, 64), (2, 64, 64, 64)]:
        wl = _custom("gate_qs_x", B, H, W, C, "bf16", seed=4242)
        inp = wl.generate()
        x, _ = to_device(inp["x"], "bf16")
        w, _ = vec_f32(inp["w"])
        u, _ = vec_f32(inp["u"])
        mus = [vec_f32(inp[n])[0] for n in ("mu_r", "mu_k", "mu_v")]
        qs = vk.QShift(H, W, 1, 0.25, *mus)
        a = vk.spatial_gate(x, x, x, w, u, qs=qs, workspace=ws)
        b = vk.spatial_gate(x, x, x, w, u, qs=qs)  # the same kernel's cluster exchange
        vk.device_status()
        assert torch.equal(a, b)
        outs.append(a)
    assert torch.equal(outs[0], outs[2]) and torch.equal(outs[2], outs[3])
    ctl = ws[:12].view(torch.int32).cpu().tolist()
    assert ctl[0] == 0 and ctl[1] == 0 and ctl[2] >= 4  # counters reset, 4+ generations


def test_workspace_rejects_bad_arguments(vk):
    import torch
    x = torch.zeros(1, 512, 64, device="cuda", dtype=torch.bfloat16)
    w = torch.zeros(64, device="cuda")
    small = torch.zeros(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(vk.VrwkvError):
        vk.spatial_gate(x, x, x, w, w, workspace=small)
    big = torch.zeros(vk.fwd_workspace_bytes(1, 512, 64) + 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(vk.VrwkvError):
        vk.spatial_gate(x, x, x, w, w, workspace=big[1:])  # misaligned
