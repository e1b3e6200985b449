"""Python binding of the B200 (sm_100a) Vision-RWKV spatial-mix core.

Thin ctypes marshalling over ``libvrwkv.so`` (the C ABI in include/vrwkv.h):
every step of Q-Shift, Bi-WKV and the sigma(R) gate runs in the library's
CUDA kernels.  PyTorch provides device memory and the current stream only.
There is no fallback: if the library is missing, the calls raise.

    qshift(x, H, W, shift_pixel=1, gamma=0.25, mu=None)
    bishift(x, H, W, shift_pixel=1, gamma=0.25, mu=None)  # sparse (MAE) inputs
    biwkv_fwd(k, v, w, u, qs=None, workspace=None)
    spatial_gate(r, k, v, w, u, qs=None, workspace=None)
    fwd_workspace(B, T, C, device)  # a zeroed workspace for the two calls above
    spatial_gate_host(r, k, v, w, u, qs=None, out=None, slice_b=1)  # host tensors, copies overlapped
    channel_mix(x, qs=None)
    biwkv_bwd(k, v, w, u, gy)  # -> gk, gv, gw (B, C), gu (B, C), gw_total, gu_total
    spatial_mix_block(x, weights, w, u, ln_gamma, ln_beta, qs, workspace=None)
    device_status()     # synchronise; raise if a kernel's bounded wait ran out

Token tensors are contiguous (B, T, C) CUDA tensors of dtype float32 or
bfloat16; w, u and mu vectors are contiguous float32 CUDA tensors of
length C.  ``qs`` is a ``QShift`` (grid, shift, gamma and the three mu
vectors).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libvrwkv.so")

VRWKV_OK = 0
VRWKV_F32 = 0
VRWKV_BF16 = 1

_lib = None


class VrwkvError(RuntimeError):
    """A non-OK status returned by the C ABI."""

    def __init__(self, status: int, message: str):
        super().__init__(message)
        self.status = status


class _QsParams(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int), ("W", ctypes.c_int), ("shift_pixel", ctypes.c_int),
                ("gamma", ctypes.c_double), ("mu_r", ctypes.c_void_p),
                ("mu_k", ctypes.c_void_p), ("mu_v", ctypes.c_void_p), ("mode", ctypes.c_int)]


def load_library():
    """Load libvrwkv.so; raise if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m linear_complexity_vision_b200.build` (nvcc, sm_100a)")
        lib = ctypes.CDLL(LIB_PATH)
        vp, ci, cd = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
        lib.vrwkv_qshift.argtypes = [vp, vp, vp, ci, ci, ci, ci, ci, cd, ci, vp]
        lib.vrwkv_qshift.restype = ci
        lib.vrwkv_bishift.argtypes = [vp, vp, vp, ci, ci, ci, ci, ci, cd, ci, vp]
        lib.vrwkv_bishift.restype = ci
        for name in ("vrwkv_biwkv_fwd",):
            getattr(lib, name).argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci,
                                           ctypes.POINTER(_QsParams), vp]
            getattr(lib, name).restype = ci
        lib.vrwkv_spatial_gate.argtypes = [vp, vp, vp, vp, vp, vp, ci, ci, ci, ci,
                                           ctypes.POINTER(_QsParams), vp]
        lib.vrwkv_spatial_gate.restype = ci
        lib.vrwkv_fwd_workspace_bytes.argtypes = [ci, ci, ci]
        lib.vrwkv_fwd_workspace_bytes.restype = ctypes.c_size_t
        lib.vrwkv_biwkv_fwd_ws.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci,
                                           ctypes.POINTER(_QsParams), vp, ctypes.c_size_t, vp]
        lib.vrwkv_biwkv_fwd_ws.restype = ci
        lib.vrwkv_spatial_gate_ws.argtypes = [vp, vp, vp, vp, vp, vp, ci, ci, ci, ci,
                                              ctypes.POINTER(_QsParams), vp, ctypes.c_size_t, vp]
        lib.vrwkv_spatial_gate_ws.restype = ci
        lib.vrwkv_block_workspace_bytes.argtypes = [ci, ci, ci, ci]
        lib.vrwkv_block_workspace_bytes.restype = ctypes.c_size_t
        lib.vrwkv_spatial_mix_block.argtypes = [vp] * 9 + [ctypes.c_float, vp, ci, ci, ci, ci,
                                                ctypes.POINTER(_QsParams), vp, ctypes.c_size_t, vp]
        lib.vrwkv_spatial_mix_block.restype = ci
        lib.vrwkv_spatial_gate_static.argtypes = [vp, vp, vp, vp, vp, vp, ci, ci, ci, ci,
                                                  ctypes.POINTER(_QsParams), vp]
        lib.vrwkv_spatial_gate_static.restype = ci
        lib.vrwkv_spatial_gate_host.argtypes = [vp, vp, vp, vp, vp, vp, ci, ci, ci, ci,
                                                ctypes.POINTER(_QsParams), ci, vp, ctypes.c_size_t, vp]
        lib.vrwkv_spatial_gate_host.restype = ci
        lib.vrwkv_spatial_gate_host_buffer_bytes.argtypes = [ci, ci, ci, ci, ci]
        lib.vrwkv_spatial_gate_host_buffer_bytes.restype = ctypes.c_size_t
        lib.vrwkv_biwkv_bwd.argtypes = [vp] * 11 + [ci] * 4 + [vp]
        lib.vrwkv_biwkv_bwd.restype = ci
        lib.vrwkv_channel_mix.argtypes = [vp, vp, ci, ci, ci, ci, ctypes.POINTER(_QsParams), vp]
        lib.vrwkv_channel_mix.restype = ci
        lib.vrwkv_device_status.argtypes = []
        lib.vrwkv_device_status.restype = ci
        lib.vrwkv_set_wait_limit.argtypes = [ctypes.c_double]
        lib.vrwkv_set_wait_limit.restype = ci
        lib.vrwkv_status_string.argtypes = [ci]
        lib.vrwkv_status_string.restype = ctypes.c_char_p
        lib.vrwkv_last_kernel.argtypes = []
        lib.vrwkv_last_kernel.restype = ctypes.c_char_p
        lib.vrwkv_last_error.argtypes = []
        lib.vrwkv_last_error.restype = ctypes.c_char_p
        _lib = lib
    return _lib


def _check(status: int) -> None:
    if status != VRWKV_OK:
        lib = load_library()
        name = lib.vrwkv_status_string(status).decode()
        msg = lib.vrwkv_last_error().decode()
        raise VrwkvError(status, f"{name}: {msg}")


@dataclass
class QShift:
    """Q-Shift parameters: patch grid H x W, shift_pixel, gamma and the
    interpolation weights mu_r, mu_k, mu_v (float32 (C,) CUDA tensors or
    None for the pure shifted tensor)."""
    H: int
    W: int
    shift_pixel: int = 1
    gamma: float = 0.25
    mu_r: Optional[object] = None
    mu_k: Optional[object] = None
    mu_v: Optional[object] = None
    mode: int = 0  # 0: Q-Shift (eq. 9); 1: bidirectional shift for sparse (MAE) inputs

    def _struct(self) -> _QsParams:
        def ptr(t):
            return None if t is None else t.data_ptr()
        return _QsParams(int(self.H), int(self.W), int(self.shift_pixel), float(self.gamma),
                         ptr(self.mu_r), ptr(self.mu_k), ptr(self.mu_v), int(self.mode))


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float32:
        return VRWKV_F32
    if t.dtype == torch.bfloat16:
        return VRWKV_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _stream_ptr(t) -> int:
    import torch
    return torch.cuda.current_stream(t.device).cuda_stream


def _require(t, name: str) -> None:
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")


def _require_tokens(*named) -> None:
    """(name, tensor) pairs of token tensors: contiguous CUDA (B, T, C)
    tensors of one shape, dtype and device (the C ABI cannot see sizes, so a
    mismatched output would be written past its end)."""
    ref_name, ref = named[0]
    for name, t in named:
        _require(t, name)
        if t.dim() != 3:
            raise ValueError(f"{name} must be a (B, T, C) tensor")
        if t.shape != ref.shape or t.dtype != ref.dtype or t.device != ref.device:
            raise ValueError(f"{name} must match {ref_name} in shape, dtype and device")


def _require_vec(t, C: int, device, name: str) -> None:
    """A per-channel parameter: a contiguous float32 CUDA tensor of C
    elements on `device` (read as float32[C] by the kernels)."""
    import torch
    _require(t, name)
    if t.dtype != torch.float32 or t.numel() != C or t.device != device:
        raise ValueError(f"{name} must be a float32 tensor of {C} elements on {device}")


def _qs_ptr(qs, C: int, device):
    """ctypes pointer to the Q-Shift parameters (None without Q-Shift), after
    checking the mu vectors."""
    if qs is None:
        return None
    for name in ("mu_r", "mu_k", "mu_v"):
        t = getattr(qs, name)
        if t is not None:
            _require_vec(t, C, device, f"qs.{name}")
    return ctypes.byref(qs._struct())


def qshift(x, H: int, W: int, shift_pixel: int = 1, gamma: float = 0.25, mu=None, out=None):
    """Q-Shift of x (B, H*W, C): the shifted tensor, or mu*x + (1-mu)*shifted."""
    import torch
    _require_tokens(("x", x))
    B, T, C = x.shape
    if mu is not None:
        _require_vec(mu, C, x.device, "mu")
    if out is None:
        out = torch.empty_like(x)
    _require_tokens(("x", x), ("out", out))
    _check(load_library().vrwkv_qshift(
        x.data_ptr(), out.data_ptr(), None if mu is None else mu.data_ptr(), B, H, W, C,
        shift_pixel, float(gamma), _dtype_code(x), _stream_ptr(x)))
    return out


def bishift(x, H: int, W: int, shift_pixel: int = 1, gamma: float = 0.25, mu=None, out=None):
    """The bidirectional shift of sparse (MAE) inputs (QShift mode 1) of x
    (B, H*W, C): the shifted tensor, or mu*x + (1-mu)*shifted."""
    import torch
    _require_tokens(("x", x))
    B, T, C = x.shape
    if mu is not None:
        _require_vec(mu, C, x.device, "mu")
    if out is None:
        out = torch.empty_like(x)
    _require_tokens(("x", x), ("out", out))
    _check(load_library().vrwkv_bishift(
        x.data_ptr(), out.data_ptr(), None if mu is None else mu.data_ptr(), B, H, W, C,
        shift_pixel, float(gamma), _dtype_code(x), _stream_ptr(x)))
    return out


def fwd_workspace_bytes(B: int, T: int, C: int) -> int:
    """Bytes of workspace the *_ws forward entry points need."""
    return int(load_library().vrwkv_fwd_workspace_bytes(B, T, C))


def fwd_workspace(B: int, T: int, C: int, device="cuda"):
    """A zero-filled uint8 CUDA tensor usable as the forward workspace of
    (B, T, C) problems (and smaller ones) on one stream at a time."""
    import torch
    return torch.zeros(fwd_workspace_bytes(B, T, C), dtype=torch.uint8, device=device)


def biwkv_fwd(k, v, w, u, qs: Optional[QShift] = None, out=None, workspace=None):
    """Bi-WKV forward of eq. 5 on (B, T, C) tensors; Q-Shift on load if qs.
    With a workspace (see fwd_workspace) the CTAs of long sequences exchange
    their sums through it instead of a thread-block cluster."""
    import torch
    _require_tokens(("k", k), ("v", v))
    B, T, C = k.shape
    for t, name in ((w, "w"), (u, "u")):
        _require_vec(t, C, k.device, name)
    if out is None:
        out = torch.empty_like(k)
    _require_tokens(("k", k), ("out", out))
    qsp = _qs_ptr(qs, C, k.device)
    lib = load_library()
    if workspace is None:
        _check(lib.vrwkv_biwkv_fwd(
            k.data_ptr(), v.data_ptr(), w.data_ptr(), u.data_ptr(), out.data_ptr(), B, T, C,
            _dtype_code(k), qsp, _stream_ptr(k)))
    else:
        _require(workspace, "workspace")
        _check(lib.vrwkv_biwkv_fwd_ws(
            k.data_ptr(), v.data_ptr(), w.data_ptr(), u.data_ptr(), out.data_ptr(), B, T, C,
            _dtype_code(k), qsp, workspace.data_ptr(), workspace.numel() * workspace.element_size(),
            _stream_ptr(k)))
    return out


def spatial_gate(r, k, v, w, u, qs: Optional[QShift] = None, out=None, workspace=None):
    """sigma(QS_R(r)) * Bi-WKV(QS_K(k), QS_V(v)); r, k, v may be one tensor.
    workspace: as for biwkv_fwd."""
    import torch
    _require_tokens(("k", k), ("r", r), ("v", v))
    B, T, C = k.shape
    for t, name in ((w, "w"), (u, "u")):
        _require_vec(t, C, k.device, name)
    if out is None:
        out = torch.empty_like(k)
    _require_tokens(("k", k), ("out", out))
    qsp = _qs_ptr(qs, C, k.device)
    lib = load_library()
    if workspace is None:
        _check(lib.vrwkv_spatial_gate(
            r.data_ptr(), k.data_ptr(), v.data_ptr(), w.data_ptr(), u.data_ptr(), out.data_ptr(),
            B, T, C, _dtype_code(k), qsp, _stream_ptr(k)))
    else:
        _require(workspace, "workspace")
        _check(lib.vrwkv_spatial_gate_ws(
            r.data_ptr(), k.data_ptr(), v.data_ptr(), w.data_ptr(), u.data_ptr(), out.data_ptr(),
            B, T, C, _dtype_code(k), qsp, workspace.data_ptr(),
            workspace.numel() * workspace.element_size(), _stream_ptr(k)))
    return out


def channel_mix(x, qs: Optional[QShift] = None, out=None):
    """sigma(QS_R(x)) * max(QS_K(x), 0)^2 on a (B, T, C) tensor (eq. 3-4 with
    identity projections); QS is the identity if qs is None."""
    import torch
    _require_tokens(("x", x))
    B, T, C = x.shape
    if out is None:
        out = torch.empty_like(x)
    _require_tokens(("x", x), ("out", out))
    qsp = _qs_ptr(qs, C, x.device)
    _check(load_library().vrwkv_channel_mix(
        x.data_ptr(), out.data_ptr(), B, T, C, _dtype_code(x), qsp, _stream_ptr(x)))
    return out


def spatial_gate_static(r, k, v, w, u, qs: Optional[QShift] = None, out=None):
    """spatial_gate for callers that cannot allocate device memory: the
    column exchange runs in a fixed workspace the library reserved at load
    time (up to ~1600 (batch row, 8-channel) columns).  Calls overlapping in
    time on other streams share that workspace and race.

    The C entry point allocates nothing.  Pass ``out`` (a preallocated
    tensor like ``k``) to allocate nothing here either; without it this
    wrapper allocates the output with torch."""
    import torch
    _require_tokens(("k", k), ("r", r), ("v", v))
    B, T, C = k.shape
    for t, name in ((w, "w"), (u, "u")):
        _require_vec(t, C, k.device, name)
    if out is None:
        out = torch.empty_like(k)
    _require_tokens(("k", k), ("out", out))
    qsp = _qs_ptr(qs, C, k.device)
    _check(load_library().vrwkv_spatial_gate_static(
        r.data_ptr(), k.data_ptr(), v.data_ptr(), w.data_ptr(), u.data_ptr(), out.data_ptr(),
        B, T, C, _dtype_code(k), qsp, _stream_ptr(k)))
    return out


def spatial_gate_host_buffer(r, k, v, slice_b: int = 1, device="cuda"):
    """A device staging buffer for spatial_gate_host on host tensors r, k, v
    (the number of distinct buffers among them decides its size)."""
    import torch
    B, T, C = k.shape
    inputs = len({t.data_ptr() for t in (r, k, v)})
    n = int(load_library().vrwkv_spatial_gate_host_buffer_bytes(
        int(slice_b), T, C, _dtype_code(k), inputs))
    if n == 0:
        raise ValueError("invalid arguments for the host staging buffer")
    return torch.empty(n, dtype=torch.uint8, device=device)


def spatial_gate_host(r, k, v, w, u, qs: Optional[QShift] = None, out=None, slice_b: int = 1,
                      dev_buf=None, stream=None):
    """spatial_gate on page-locked HOST tensors r, k, v (may be one tensor)
    with the result written to the page-locked host tensor ``out``: batch
    slices of ``slice_b`` rows stream through ``dev_buf`` (see
    spatial_gate_host_buffer) with both copy directions overlapping the
    kernels.  w, u and the QShift mu vectors are CUDA tensors.  Asynchronous
    on ``stream`` (default: the current stream of w's device)."""
    import torch
    for t, name in ((k, "k"), (r, "r"), (v, "v")):
        if t.device.type != "cpu" or not t.is_pinned() or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous page-locked CPU tensor")
        if t.shape != k.shape or t.dtype != k.dtype:
            raise ValueError(f"{name} must match k in shape and dtype")
    if k.dim() != 3:
        raise ValueError("k must be (B, T, C)")
    B, T, C = k.shape
    for t, name in ((w, "w"), (u, "u")):
        _require_vec(t, C, w.device, name)
    if out is None:
        out = torch.empty_like(k).pin_memory()
    if out.shape != k.shape or out.dtype != k.dtype or not out.is_pinned() or not out.is_contiguous():
        raise ValueError("out must be a contiguous page-locked CPU tensor like k")
    if dev_buf is None:
        dev_buf = spatial_gate_host_buffer(r, k, v, slice_b, device=w.device)
    qsp = _qs_ptr(qs, C, w.device)
    s = stream if stream is not None else torch.cuda.current_stream(w.device)
    _check(load_library().vrwkv_spatial_gate_host(
        r.data_ptr(), k.data_ptr(), v.data_ptr(), w.data_ptr(), u.data_ptr(), out.data_ptr(),
        B, T, C, _dtype_code(k), qsp, int(slice_b), dev_buf.data_ptr(),
        dev_buf.numel() * dev_buf.element_size(), s.cuda_stream))
    return out


def block_workspace(B: int, T: int, C: int, dtype, device="cuda"):
    """A uint8 CUDA tensor large enough for spatial_mix_block on (B, T, C)."""
    import torch
    code = VRWKV_F32 if dtype == torch.float32 else VRWKV_BF16
    n = int(load_library().vrwkv_block_workspace_bytes(B, T, C, code))
    return torch.empty(n, dtype=torch.uint8, device=device)


def spatial_mix_block(x, weights, w, u, ln_gamma, ln_beta, qs: QShift, ln_eps: float = 1e-5,
                      workspace=None, out=None):
    """LayerNorm((sigma(R) * Bi-WKV(K, V)) W_O) with R, K, V = QS_*(x) W_*
    (eq. 1-2).  weights = (W_R, W_K, W_V, W_O), each (C, C) in x's dtype,
    row-major (C_in, C_out).  workspace: see block_workspace."""
    import torch
    _require_tokens(("x", x))
    B, T, C = x.shape
    if len(weights) != 4:
        raise ValueError("weights must be (W_R, W_K, W_V, W_O)")
    for i, t in enumerate(weights):
        _require(t, f"weights[{i}]")
        if tuple(t.shape) != (C, C) or t.dtype != x.dtype or t.device != x.device:
            raise ValueError(f"weights[{i}] must be a ({C}, {C}) tensor in x's dtype on x's device")
    for t, name in ((w, "w"), (u, "u"), (ln_gamma, "ln_gamma"), (ln_beta, "ln_beta")):
        _require_vec(t, C, x.device, name)
    if qs is None:
        raise ValueError("spatial_mix_block needs the Q-Shift parameters")
    for name in ("mu_r", "mu_k", "mu_v"):
        t = getattr(qs, name)
        if t is not None:
            _require_vec(t, C, x.device, f"qs.{name}")
    if out is None:
        out = torch.empty_like(x)
    _require_tokens(("x", x), ("out", out))
    if workspace is None:
        workspace = block_workspace(B, T, C, x.dtype, device=x.device)
    wr, wk, wv, wo = weights
    _check(load_library().vrwkv_spatial_mix_block(
        x.data_ptr(), wr.data_ptr(), wk.data_ptr(), wv.data_ptr(), wo.data_ptr(), w.data_ptr(),
        u.data_ptr(), ln_gamma.data_ptr(), ln_beta.data_ptr(), float(ln_eps), out.data_ptr(),
        B, T, C, _dtype_code(x), ctypes.byref(qs._struct()), workspace.data_ptr(),
        workspace.numel() * workspace.element_size(), _stream_ptr(x)))
    return out


def biwkv_bwd(k, v, w, u, gy, totals: bool = True, out=None):
    """Gradients of eq. 5 for the upstream gradient gy: gk, gv (B, T, C) in
    the input dtype, gw, gu float32 (B, C) per batch row and, if totals, their
    sums over the batch (float32 (C,)); otherwise those two are None.
    out: optional (gk, gv, gw, gu) to write instead of allocating them."""
    import torch
    _require_tokens(("k", k), ("v", v), ("gy", gy))
    B, T, C = k.shape
    for t, name in ((w, "w"), (u, "u")):
        _require_vec(t, C, k.device, name)
    if out is None:
        gk, gv = torch.empty_like(k), torch.empty_like(k)
        gw = torch.empty((B, C), dtype=torch.float32, device=k.device)
        gu = torch.empty((B, C), dtype=torch.float32, device=k.device)
    else:
        gk, gv, gw, gu = out
        _require_tokens(("k", k), ("gk", gk), ("gv", gv))
        for t, name in ((gw, "gw"), (gu, "gu")):
            if (t.dtype != torch.float32 or t.device != k.device or not t.is_contiguous()
                    or t.numel() != B * C):
                raise ValueError(f"{name} must be a contiguous float32 tensor of B*C elements on {k.device}")
    gwt = torch.empty(C, dtype=torch.float32, device=k.device) if totals else None
    gut = torch.empty(C, dtype=torch.float32, device=k.device) if totals else None
    _check(load_library().vrwkv_biwkv_bwd(
        k.data_ptr(), v.data_ptr(), w.data_ptr(), u.data_ptr(), gy.data_ptr(), gk.data_ptr(),
        gv.data_ptr(), gw.data_ptr(), gu.data_ptr(), None if gwt is None else gwt.data_ptr(),
        None if gut is None else gut.data_ptr(), B, T, C, _dtype_code(k), _stream_ptr(k)))
    return gk, gv, gw, gu, gwt, gut


def set_wait_limit(seconds: float) -> None:
    """Limit of every bounded wait in the kernels on the current device
    (vrwkv_set_wait_limit; default 2 s).  Call outside stream capture."""
    _check(load_library().vrwkv_set_wait_limit(float(seconds)))


def device_status() -> None:
    """Synchronise with the current device and raise VrwkvError if a kernel
    recorded a timed-out wait since the last check (vrwkv_device_status)."""
    _check(load_library().vrwkv_device_status())
