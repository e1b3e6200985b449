"""The bounded-wait error path, exercised without a fault.

In the workspace variants the CTAs of one (batch row, channel slab) column
take consecutive tickets from a counter in the workspace, publish their
aggregates and wait, with a bounded spin, for their column peers' flags.
Presetting the counter makes one CTA take the last rank of the column while
its peer takes a ticket past the grid and stops at once (error flag 4): the
first CTA's wait for the missing peer's record runs out after the wait limit
(flag 2), the kernel finishes, and vrwkv_device_status reports
VRWKV_ERR_TIMEOUT.  The context stays usable: the next call is correct.
"""
import time

import numpy as np
import pytest

from helpers import TOL, biwkv_scale, scaled_error, to_device, to_numpy, vec_f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def vk():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import linear_complexity_vision_b200 as m
    m.load_library()
    return m


def _inputs(B, T, C):
    rng = np.random.default_rng(4242)
    k = rng.standard_normal((B, T, C))
    v = rng.standard_normal((B, T, C))
    w = rng.uniform(-3, 3, C)
    u = rng.normal(0, 0.5, C)
    return k, v, w, u


@pytest.mark.parametrize("T,kernel,forward", [(1000, "biwkv_tma_kernel", "narrow"),
                                              (2048, "biwkv_tm_kernel", None)])
def test_workspace_peer_wait_runs_out_and_is_reported(vk, oracle_mod, T, kernel, forward, monkeypatch):
    import torch
    # fast paths without Q-Shift, one 8-channel slab: 512-token CTAs of the
    # 8-channel kernel at T = 1000 (held to it: the default there is the
    # 32-token kernel), 1024-token CTAs of the 32-token kernel at T = 2048, so
    # the grid holds exactly two CTAs, ranks 0 and 1 of one column (the CTA
    # that finds its ticket past the grid leaves before it takes any tensor
    # memory)
    if forward:
        monkeypatch.setenv("VRWKV_FORWARD", forward)
    else:
        monkeypatch.delenv("VRWKV_FORWARD", raising=False)
    B, C = 1, 8
    k, v, w, u = _inputs(B, T, C)
    kt, kd = to_device(k, "bf16")
    vt, vd = to_device(v, "bf16")
    wt, wd = vec_f32(w)
    ut, ud = vec_f32(u)
    vk.device_status()  # start from a clear error word
    ws = vk.fwd_workspace(B, T, C)
    ws.view(torch.int32)[0] = 1  # next ticket: 1 (rank 1), then 2 (past the grid)
    vk.set_wait_limit(1e-3)
    try:
        t0 = time.perf_counter()
        vk.biwkv_fwd(kt, vt, wt, ut, workspace=ws)
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
        with pytest.raises(vk.VrwkvError) as err:
            vk.device_status()
        msg = str(err.value)
        assert err.value.status == 4, msg  # VRWKV_ERR_TIMEOUT
        assert "flags 0x6" in msg, msg  # 2: a peer's record never came; 4: a ticket past the grid
        assert elapsed < 1.0, elapsed  # the 1 ms limit, not the 2 s default
    finally:
        vk.set_wait_limit(2.0)
    vk.device_status()  # the word was cleared by the report
    # the context is intact: a fresh workspace gives the oracle's result
    out = vk.biwkv_fwd(kt, vt, wt, ut, workspace=vk.fwd_workspace(B, T, C))
    vk.device_status()
    assert vk.load_library().vrwkv_last_kernel().decode() == kernel
    got = to_numpy(out)
    want = oracle_mod.biwkv_direct(kd, vd, wd, ud)
    err = scaled_error(got, want, biwkv_scale(oracle_mod, kd, vd, wd, ud))
    assert err <= TOL["bf16"], err
