"""The C ABI library loads, exports every function include/vrwkv.h declares,
and rejects invalid arguments on the host (no GPU is touched: validation
precedes every CUDA call)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "vrwkv.h")


@pytest.fixture(scope="module")
def lib():
    from linear_complexity_vision_b200 import build
    build.build()
    import linear_complexity_vision_b200 as vk
    return vk.load_library()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(vrwkv_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_three_operations():
    names = _declared_functions()
    for n in ("vrwkv_qshift", "vrwkv_biwkv_fwd", "vrwkv_spatial_gate",
              "vrwkv_status_string", "vrwkv_last_error"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    assert lib.vrwkv_status_string(0) == b"VRWKV_OK"
    assert lib.vrwkv_status_string(1) == b"VRWKV_ERR_INVALID_ARG"
    assert lib.vrwkv_status_string(99) == b"VRWKV_ERR_UNKNOWN"


FAKE = 1 << 20  # non-null, never dereferenced: validation fails first


def _qs(H, W, s=1, gamma=0.25):
    import linear_complexity_vision_b200 as vk
    return ctypes.byref(vk._QsParams(H, W, s, gamma, None, None, None))


@pytest.mark.parametrize("args,frag", [
    (dict(B=0), "positive"),
    (dict(C=-1), "positive"),
    (dict(k=None), "NULL"),
    (dict(dtype=7), "dtype"),
    (dict(k=FAKE + 1, dtype=1), "misaligned"),
    (dict(out=FAKE), "overlaps"),
    (dict(qs=(14, 15)), "H*W"),
    (dict(qs=(14, 14, -1)), "shift_pixel"),
    (dict(qs=(14, 14, 1, 0.3)), "gamma"),
    (dict(T=8192, qs=None), "T = 8192"),
])
def test_biwkv_rejects_invalid_arguments(lib, args, frag):
    a = dict(k=FAKE, v=FAKE + (1 << 24), w=FAKE + (2 << 24), u=FAKE + (3 << 24),
             out=FAKE + (4 << 24), B=2, T=196, C=32, dtype=0, qs=None)
    a.update(args)
    qs = _qs(*a["qs"]) if a["qs"] else None
    st = lib.vrwkv_biwkv_fwd(a["k"], a["v"], a["w"], a["u"], a["out"], a["B"], a["T"],
                             a["C"], a["dtype"], qs, None)
    assert st in (1, 2)
    assert frag in lib.vrwkv_last_error().decode()


def test_spatial_gate_requires_r(lib):
    st = lib.vrwkv_spatial_gate(None, FAKE, FAKE, FAKE, FAKE, FAKE + (1 << 24), 1, 4, 4, 0,
                                None, None)
    assert st == 1


def test_qshift_rejects_invalid_arguments(lib):
    assert lib.vrwkv_qshift(FAKE, FAKE + (1 << 24), None, 1, 0, 4, 8, 1, 0.25, 0, None) == 1
    assert lib.vrwkv_qshift(FAKE, FAKE + (1 << 24), None, 1, 4, 4, 8, 1, 0.26, 0, None) == 1
    assert lib.vrwkv_qshift(FAKE, FAKE + 4, None, 1, 4, 4, 8, 1, 0.25, 0, None) == 1
    assert b"overlaps" in lib.vrwkv_last_error()


@pytest.mark.parametrize("args,frag", [
    (dict(B=0), "positive"),
    (dict(T=-3), "positive"),
    (dict(x=None), "NULL"),
    (dict(dtype=5), "dtype"),
    (dict(x=FAKE + 1, dtype=1), "misaligned"),
    (dict(out=FAKE + 64), "overlaps"),
    (dict(qs=(14, 15)), "H*W"),
    (dict(qs=(14, 14, 1, -0.1)), "gamma"),
    (dict(B=1 << 16, T=1 << 15), "2^31"),
])
def test_channel_mix_rejects_invalid_arguments(lib, args, frag):
    a = dict(x=FAKE, out=FAKE + (1 << 24), B=2, T=196, C=32, dtype=0, qs=None)
    a.update(args)
    qs = _qs(*a["qs"]) if a["qs"] else None
    st = lib.vrwkv_channel_mix(a["x"], a["out"], a["B"], a["T"], a["C"], a["dtype"], qs, None)
    assert st in (1, 2)
    assert frag in lib.vrwkv_last_error().decode()


@pytest.mark.parametrize("args,frag", [
    (dict(B=0), "positive"),
    (dict(gy=None), "NULL"),
    (dict(gw=None), "NULL"),
    (dict(dtype=9), "dtype"),
    (dict(T=4097), "exceeds"),
    (dict(k=FAKE + 1, dtype=1), "misaligned"),
    (dict(gk=FAKE + 64), "overlaps"),
    (dict(gw_total=FAKE + (6 << 24) + 4, gu_total=FAKE + (6 << 24)), "overlap"),
])
def test_biwkv_bwd_rejects_invalid_arguments(lib, args, frag):
    a = dict(k=FAKE, v=FAKE + (1 << 24), w=FAKE + (2 << 24), u=FAKE + (3 << 24), gy=FAKE + (4 << 24),
             gk=FAKE + (5 << 24), gv=FAKE + (5 << 24) + (1 << 22), gw=FAKE + (6 << 24) + (1 << 20),
             gu=FAKE + (6 << 24) + (2 << 20), gw_total=None, gu_total=None,
             B=2, T=196, C=32, dtype=0)
    a.update(args)
    st = lib.vrwkv_biwkv_bwd(a["k"], a["v"], a["w"], a["u"], a["gy"], a["gk"], a["gv"], a["gw"],
                             a["gu"], a["gw_total"], a["gu_total"], a["B"], a["T"], a["C"],
                             a["dtype"], None)
    assert st in (1, 2)
    assert frag in lib.vrwkv_last_error().decode()


def test_static_entry_rejects_on_the_host(lib):
    # validation and the size limit come before any device work
    assert lib.vrwkv_spatial_gate_static(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + (1 << 24), 0, 4, 16, 1,
                                         None, None) == 1
    assert lib.vrwkv_spatial_gate_static(None, FAKE, FAKE, FAKE, FAKE, FAKE + (1 << 24), 1, 4, 16, 1,
                                         None, None) == 1
    st = lib.vrwkv_spatial_gate_static(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + (1 << 24), 64, 4, 16384,
                                       1, None, None)
    assert st == 2 and b"static workspace" in lib.vrwkv_last_error()


@pytest.mark.parametrize("args,frag", [
    (dict(B=0), "positive"),
    (dict(x=None), "NULL"),
    (dict(dtype=4), "dtype"),
    (dict(s=-1), "shift_pixel"),
    (dict(gamma=0.3), "gamma"),
    (dict(x=FAKE + 1, dtype=1), "misaligned"),
    (dict(out=FAKE + 64), "overlaps"),
])
def test_bishift_rejects_invalid_arguments(lib, args, frag):
    a = dict(x=FAKE, out=FAKE + (1 << 24), mu=None, B=2, H=14, W=14, C=32, s=1, gamma=0.25, dtype=0)
    a.update(args)
    st = lib.vrwkv_bishift(a["x"], a["out"], a["mu"], a["B"], a["H"], a["W"], a["C"], a["s"],
                           a["gamma"], a["dtype"], None)
    assert st in (1, 2)
    assert frag in lib.vrwkv_last_error().decode()


def test_qshift_params_mode_is_checked(lib):
    import linear_complexity_vision_b200 as vk
    qs = vk._QsParams(14, 14, 1, 0.25, None, None, None, 7)
    st = lib.vrwkv_biwkv_fwd(FAKE, FAKE + (1 << 24), FAKE + (2 << 24), FAKE + (3 << 24),
                             FAKE + (4 << 24), 2, 196, 32, 0, ctypes.byref(qs), None)
    assert st == 1 and b"mode" in lib.vrwkv_last_error()


def test_workspace_variants_reject_bad_workspaces(lib):
    B, T, C = 2, 1024, 32
    need = lib.vrwkv_fwd_workspace_bytes(B, T, C)
    assert need > 0
    base = dict(k=FAKE, v=FAKE + (1 << 24), w=FAKE + (2 << 24), u=FAKE + (3 << 24), out=FAKE + (4 << 24))
    ws_ok = FAKE + (8 << 24)

    def call(ws, nbytes):
        return lib.vrwkv_biwkv_fwd_ws(base["k"], base["v"], base["w"], base["u"], base["out"], B, T, C,
                                      0, None, ws, nbytes, None)
    assert call(None, need) == 1 and b"NULL" in lib.vrwkv_last_error()
    assert call(ws_ok + 128, need) == 1 and b"256-byte" in lib.vrwkv_last_error()
    assert call(ws_ok, need - 1) == 1 and b"smaller" in lib.vrwkv_last_error()
    assert call(base["k"], need) == 1 and b"overlaps" in lib.vrwkv_last_error()
    st = lib.vrwkv_spatial_gate_ws(FAKE, FAKE, FAKE, base["w"], base["u"], base["out"], B, T, C, 0,
                                   None, None, need, None)
    assert st == 1 and b"NULL" in lib.vrwkv_last_error()


@pytest.mark.parametrize("args,frag", [
    (dict(B=0), "positive"),
    (dict(x=None), "NULL"),
    (dict(w_o=None), "NULL"),
    (dict(ws=None), "NULL"),
    (dict(dtype=3), "dtype"),
    (dict(eps=-1.0), "ln_eps"),
    (dict(x=FAKE + 8), "16-byte"),
    (dict(ws=FAKE + (9 << 24) + 64), "256-byte"),
    (dict(ws_bytes=16), "smaller"),
    (dict(out=FAKE), "overlaps"),
])
def test_block_rejects_invalid_arguments(lib, args, frag):
    B, T, C = 2, 196, 64
    a = dict(x=FAKE, w_r=FAKE + (1 << 24), w_k=FAKE + (2 << 24), w_v=FAKE + (3 << 24),
             w_o=FAKE + (4 << 24), w=FAKE + (5 << 24), u=FAKE + (5 << 24) + 4096,
             g=FAKE + (5 << 24) + 8192, be=FAKE + (5 << 24) + 12288, eps=1e-5, out=FAKE + (6 << 24),
             B=B, T=T, C=C, dtype=1, ws=FAKE + (9 << 24), ws_bytes=None)
    a.update(args)
    need = lib.vrwkv_block_workspace_bytes(B, T, C, 1)
    assert need > 0
    nb = need if a["ws_bytes"] is None else a["ws_bytes"]
    st = lib.vrwkv_spatial_mix_block(a["x"], a["w_r"], a["w_k"], a["w_v"], a["w_o"], a["w"], a["u"],
                                     a["g"], a["be"], a["eps"], a["out"], a["B"], a["T"], a["C"],
                                     a["dtype"], _qs(14, 14), a["ws"], nb, None)
    assert st in (1, 2)
    assert frag in lib.vrwkv_last_error().decode()


@pytest.mark.parametrize("seconds", [0.0, -1.0, 61.0, float("nan")])
def test_wait_limit_outside_range_is_rejected_on_the_host(lib, seconds):
    lib.vrwkv_set_wait_limit.argtypes = [ctypes.c_double]
    assert lib.vrwkv_set_wait_limit(seconds) == 1  # VRWKV_ERR_INVALID_ARG
    assert b"wait limit" in lib.vrwkv_last_error()


def test_host_buffer_bytes(lib):
    f = lib.vrwkv_spatial_gate_host_buffer_bytes
    f.argtypes = [ctypes.c_int] * 5
    f.restype = ctypes.c_size_t
    # three slots of (inputs + 1) tensors of slice_b * T * C elements, 256-byte rounded
    assert f(1, 4096, 1024, 1, 1) == 3 * 2 * 4096 * 1024 * 2
    assert f(2, 196, 768, 0, 3) == 3 * 4 * ((2 * 196 * 768 * 4 + 255) // 256 * 256)
    assert f(1, 3, 5, 1, 1) == 3 * 2 * 256
    for bad in ((0, 16, 16, 1, 1), (1, 16, 16, 1, 0), (1, 16, 16, 1, 4), (1, 16, 16, 7, 1)):
        assert f(*bad) == 0


@pytest.mark.parametrize("args,frag", [
    (dict(B=0), "positive"),
    (dict(slice_b=0), "slice_b"),
    (dict(slice_b=9), "slice_b"),
    (dict(dev_buf=None), "NULL"),
    (dict(dtype=7), "dtype"),
    (dict(dev_bytes=100), "device buffer"),
    (dict(dev_buf=FAKE + 16), "aligned"),
])
def test_host_pipeline_rejects_bad_arguments_on_the_host(lib, args, frag):
    a = dict(r=FAKE, k=FAKE, v=FAKE, w=FAKE, u=FAKE, out=2 * FAKE, B=8, T=64, C=32, dtype=1,
             slice_b=1, dev_buf=4 * FAKE, dev_bytes=1 << 30)
    a.update(args)
    vp, ci = ctypes.c_void_p, ctypes.c_int
    fn = lib.vrwkv_spatial_gate_host
    fn.argtypes = [vp] * 6 + [ci] * 4 + [vp, ci, vp, ctypes.c_size_t, vp]
    st = fn(a["r"], a["k"], a["v"], a["w"], a["u"], a["out"], a["B"], a["T"], a["C"], a["dtype"],
            None, a["slice_b"], a["dev_buf"], a["dev_bytes"], None)
    assert st == 1, lib.vrwkv_last_error()
    assert frag in lib.vrwkv_last_error().decode()
