"""vrwkv_spatial_gate_static: the fused forward on the library's fixed
workspace (for callers that cannot allocate device memory).  Collected last
on purpose: it must give the same bits as vrwkv_spatial_gate on two calls in
a row whether it runs alone or after every other test has used the library
(and the workspace kernels) on this device."""
import numpy as np
import pytest

from linear_complexity_vision_b200 import synth
from helpers import to_device, vec_f32

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
    return (to_device(x, dt)[0], vec_f32(w)[0], vec_f32(u)[0], [vec_f32(m)[0] for m in mus])


@pytest.mark.parametrize("dt,B,H,W,C", [
    ("bf16", 2, 64, 64, 64),    # 16 CTAs per column: the exchange runs in the static workspace
    ("f32", 1, 40, 40, 64),     # 10 CTAs per column
    ("bf16", 8, 64, 64, 1024),  # 1024 columns: the full-size workload
    ("bf16", 2, 14, 14, 96),    # one CTA per column: no exchange
])
def test_static_matches_spatial_gate_twice(vk, dt, B, H, W, C):
    import torch
    x, w, u, mus = _inputs(B, H, W, C, dt, seed=777 + C)
    qs = vk.QShift(H, W, 1, 0.25, *mus)
    want = vk.spatial_gate(x, x, x, w, u, qs=qs)
    for _ in range(2):  # two calls in a row on the same workspace
        got = vk.spatial_gate_static(x, x, x, w, u, qs=qs)
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
