"""vrwkv_spatial_gate_host: the spatial-mix core (eq. 2, eq. 5, eq. 9) on
page-locked host buffers, with batch slices streamed through two device
slots so the copies overlap the kernels.  Each slice is an exact
sub-problem, so the result equals vrwkv_spatial_gate on device copies of the
same inputs bit for bit (and that call is checked against the oracle
elsewhere)."""
import numpy as np
import pytest

from linear_complexity_vision_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def vk():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import linear_complexity_vision_b200 as m
    m.load_library()
    return m


def _setup(B, H, W, C, dt, distinct, seed):
    import torch
    tdt = torch.float32 if dt == "f32" else torch.bfloat16
    names = ("r", "k", "v") if distinct else ("x",)
    hosts = {n: torch.from_numpy(synth.draw(seed, n, (B, H * W, C), ("normal", 1.0))).to(tdt).pin_memory()
             for n in names}
    w = torch.from_numpy(synth.draw(seed, "w", (C,), ("uniform", -5.0, 5.0))).float().cuda()
    u = torch.from_numpy(synth.draw(seed, "u", (C,), ("normal", 1.0))).float().cuda()
    mus = [torch.from_numpy(synth.draw(seed, n, (C,), ("uniform", 0.0, 1.0))).float().cuda()
           for n in ("mu_r", "mu_k", "mu_v")]
    if distinct:
        r, k, v = hosts["r"], hosts["k"], hosts["v"]
    else:
        r = k = v = hosts["x"]
    return r, k, v, w, u, mus


@pytest.mark.parametrize("dt,B,H,W,C,distinct,slice_b", [
    ("bf16", 8, 64, 64, 1024, False, 1),   # the full-size workload, one row per slice
    ("bf16", 8, 64, 64, 256, False, 3),    # ragged slices 3, 3, 2
    ("f32", 5, 14, 14, 96, True, 2),       # separate r, k, v
    ("bf16", 2, 7, 9, 20, True, 2),        # one slice, generic kernel
])
def test_host_pipeline_equals_device_call(vk, dt, B, H, W, C, distinct, slice_b):
    import torch
    r, k, v, w, u, mus = _setup(B, H, W, C, dt, distinct, seed=5150 + C + B)
    qs = vk.QShift(H, W, 1, 0.25, *mus)
    want = vk.spatial_gate(r.cuda(), k.cuda(), v.cuda(), w, u, qs=qs).cpu()
    buf = vk.spatial_gate_host_buffer(r, k, v, slice_b)
    for _ in range(2):  # the staging buffer and streams are reused
        out = torch.full_like(k, float("nan")).pin_memory()
        vk.spatial_gate_host(r, k, v, w, u, qs=qs, out=out, slice_b=slice_b, dev_buf=buf)
        torch.cuda.current_stream().synchronize()
        vk.device_status()
        assert torch.equal(out, want)


def test_host_pipeline_with_two_slots(vk):
    # a staging buffer of two slots (the minimum) gives the same results
    import torch
    B, H, W, C = 5, 32, 32, 256
    r, k, v, w, u, mus = _setup(B, H, W, C, "bf16", False, seed=4321)
    qs = vk.QShift(H, W, 1, 0.25, *mus)
    want = vk.spatial_gate(r.cuda(), k.cuda(), v.cuda(), w, u, qs=qs).cpu()
    full = vk.spatial_gate_host_buffer(r, k, v, 1)
    two = full[: full.numel() * 2 // 3]
    out = torch.full_like(k, float("nan")).pin_memory()
    vk.spatial_gate_host(r, k, v, w, u, qs=qs, out=out, slice_b=1, dev_buf=two)
    torch.cuda.current_stream().synchronize()
    vk.device_status()
    assert torch.equal(out, want)


def test_host_pipeline_rejects_pageable_memory(vk):
    import torch
    x = torch.zeros(2, 16, 32, dtype=torch.bfloat16)  # not page-locked
    w = torch.zeros(32, device="cuda")
    with pytest.raises(ValueError):
        vk.spatial_gate_host(x, x, x, w, w)
    # the C entry point checks it too
    import ctypes
    lib = vk.load_library()
    out = torch.empty_like(x).pin_memory()
    buf = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    st = lib.vrwkv_spatial_gate_host(x.data_ptr(), x.data_ptr(), x.data_ptr(), w.data_ptr(), w.data_ptr(),
                                     out.data_ptr(), 2, 16, 32, 1, None, 1, buf.data_ptr(),
                                     buf.numel(), None)
    assert st == 1 and b"page-locked" in lib.vrwkv_last_error()
