"""vrwkv_spatial_gate_static: the fused forward on the library's fixed
workspace (for callers that cannot allocate device memory).  Collected last
on purpose: on two calls in a row, whether it runs alone or after every
other test has used the library (and the workspace kernels) on this device,
it must give the same bits as vrwkv_spatial_gate_ws with a caller's
workspace (the same kernels, the exchange state in another array) and agree
within the parity tolerance with vrwkv_spatial_gate."""
import numpy as np
import pytest

from linear_complexity_vision_b200 import synth
from helpers import TOL, scaled_error, to_device, vec_f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def vk():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import linear_complexity_vision_b200 as vk
    vk.load_library()
    return vk


def _inputs(B, H, W, C, dt, seed):
    x = synth.draw(seed, "x", (B, H * W, C), ("normal", 1.0))
    w = synth.draw(seed, "w", (C,), ("uniform", -5.0, 5.0))
    u = synth.draw(seed, "u", (C,), ("normal", 1.0))
    mus = [synth.draw(seed, n, (C,), ("uniform", 0.0, 1.0)) for n in ("mu_r", "mu_k", "mu_v")]
    xt, xd = to_device(x, dt)
    dev = [vec_f32(a) for a in (w, u, *mus)]
    return xt, xd, [d[0] for d in dev], [d[1] for d in dev]


@pytest.mark.parametrize("dt,B,H,W,C", [
    ("bf16", 2, 64, 64, 64),    # tensor-memory kernel, 4 CTAs of 1024 tokens per column exchanging in the static workspace
    ("f32", 1, 40, 40, 64),     # W = 40: flat-view Q-Shift, CTAs of 1024 and 576 tokens
    ("bf16", 1, 128, 64, 64),   # T = 8192: 16-channel kernel, two 4096-token segments meeting in the static workspace
    ("bf16", 8, 64, 64, 1024),  # 1024 columns: the full-size workload
    ("bf16", 2, 14, 14, 96),    # one 256-token CTA per column: no exchange
    ("bf16", 2, 25, 40, 64),    # T = 1000: one tensor-memory CTA per column (flat view: W = 40)
])
def test_static_matches_spatial_gate_twice(vk, oracle_mod, dt, B, H, W, C):
    import torch
    x, xd, (w, u, *mus), (wd, ud, *musd) = _inputs(B, H, W, C, dt, seed=777 + C)
    qs = vk.QShift(H, W, 1, 0.25, *mus)
    want_default = vk.spatial_gate(x, x, x, w, u, qs=qs)
    want = vk.spatial_gate(x, x, x, w, u, qs=qs, workspace=vk.fwd_workspace(B, H * W, C))
    r, k, v = (oracle_mod.qshift(xd, H, W, 1, 0.25, m) for m in musd)
    scale = oracle_mod.gate(r, oracle_mod.biwkv_rnn(k, np.abs(v), wd, ud))
    for _ in range(2):  # two calls in a row on the same workspace
        got = vk.spatial_gate_static(x, x, x, w, u, qs=qs, out=torch.empty_like(x))
        vk.device_status()
        assert torch.equal(got, want)
        err = scaled_error(got.double().cpu().numpy(), want_default.double().cpu().numpy(), scale)
        assert err <= TOL[dt], err


def test_static_8_channel_exchange(vk, oracle_mod, monkeypatch):
    # the 8-channel kernel held to (the default at T = 1000 is the 32-token
    # kernel): 8-token chunks, 4 CTAs of 8 image rows per column exchanging in
    # the static workspace, twice in a row, bit-equal to the workspace call
    import torch
    monkeypatch.setenv("VRWKV_FORWARD", "narrow")
    B, H, W, C = 2, 25, 40, 64
    x, _, (w, u, *mus), _ = _inputs(B, H, W, C, "bf16", seed=1000)
    qs = vk.QShift(H, W, 1, 0.25, *mus)
    want = vk.spatial_gate(x, x, x, w, u, qs=qs, workspace=vk.fwd_workspace(B, H * W, C))
    assert vk.load_library().vrwkv_last_kernel().decode() == "biwkv_tma_kernel"
    for _ in range(2):
        got = vk.spatial_gate_static(x, x, x, w, u, qs=qs, out=torch.empty_like(x))
        vk.device_status()
        assert torch.equal(got, want)


def test_static_long_sequence_matches_workspace_call(vk):
    # T = 16384 (a 2048^2 image at patch 16): the 16-channel kernel's
    # segments meet through the static array as they do through a caller's
    # workspace
    import torch
    B, H, W, C = 1, 128, 128, 64
    x, _, (w, u, *mus), _ = _inputs(B, H, W, C, "bf16", seed=4242)
    qs = vk.QShift(H, W, 1, 0.25, *mus)
    want = vk.spatial_gate(x, x, x, w, u, qs=qs, workspace=vk.fwd_workspace(B, H * W, C))
    for _ in range(2):
        got = vk.spatial_gate_static(x, x, x, w, u, qs=qs, out=torch.empty_like(x))
        vk.device_status()
        assert torch.equal(got, want)


def test_static_rejects_oversize(vk):
    import torch
    # 8 x ceil(16384/8) = 16384 columns exceed the fixed workspace
    x = torch.zeros(8, 512, 16384, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(16384, device="cuda")
    with pytest.raises(vk.VrwkvError) as ei:
        vk.spatial_gate_static(x, x, x, w, w)
    assert ei.value.status == 2  # VRWKV_ERR_UNSUPPORTED
