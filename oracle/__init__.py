"""Float64 CPU oracle for the Vision-RWKV spatial-mix core.

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may use this package; the product path (the
CUDA library and its Python binding) never imports, links or loads it, and
this package imports nothing from the product.

It wraps ``vrwkv_oracle.c`` (plain C, float64, OpenMP over channel columns):

* ``qshift``        -- Q-Shift of "Vision-RWKV Backbone" (Quad-Directional
                       Token Shift, eq. 9) with the group layout of the
                       q_shift listing on "LinXin's Blog".
* ``qshift_f32``    -- the same interpolation in binary32 with a fixed
                       operation order, optionally rounded to bfloat16; used
                       for bit-exact comparisons.
* ``biwkv_direct``  -- Bi-WKV by direct summation of eq. 5 (O(T^2)).
* ``biwkv_points``  -- eq. 5 at selected (b, t, c) positions.
* ``biwkv_rnn``     -- Bi-WKV by the RNN form, eq. 6-7 (O(T)).
* ``biwkv_rnn_literal`` -- eq. 6-7 with the subtract-and-divide update the
                       page describes (short sequences only).
* ``gate``          -- sigma(R) (.) wkv of eq. 2.
* ``spatial_core``  -- gate(QS_R(r), Bi-WKV(QS_K(k), QS_V(v))).
* ``biwkv_bwd``     -- gradients of eq. 5 (dk, dv and per-batch dw, du) for
                       an upstream gradient gy, by the chain rule, O(T^2).
* ``biwkv_bwd_columns`` -- the same for selected (b, c) columns only.
* ``layer_norm``    -- LayerNorm over channels (biased variance).
* ``spatial_mix_block`` -- the spatial-mix block with projections: Q-Shift,
                       R/K/V projections (eq. 1), Bi-WKV and the sigma gate
                       (eq. 5, eq. 2), output projection W_O and LayerNorm.
* ``bishift``, ``bishift_f32`` -- the bidirectional shift for sparse (MAE)
                       inputs: Q-Shift's two row groups only, other channels
                       unchanged (a reading; see the C source).
* ``channel_mix``   -- sigma(QS_R(x)) * max(QS_K(x), 0)^2, the channel-mix
                       module of eq. 3-4 without projections.
* ``spatial_core_points`` -- the same at selected output positions only, by
                       direct summation of eq. 5 over each needed column.

Every array is row-major (B, T, C) with token index t = h*W + w.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "vrwkv_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile vrwkv_oracle.c into liboracle.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or (
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        dp = ctypes.POINTER(ctypes.c_double)
        fp = ctypes.POINTER(ctypes.c_float)
        i64p = ctypes.POINTER(ctypes.c_int64)
        ci, cd, cl = ctypes.c_int, ctypes.c_double, ctypes.c_long
        lib.oracle_qshift_f64.argtypes = [dp, dp, dp, ci, ci, ci, ci, ci, cd, ci]
        lib.oracle_qshift_f32.argtypes = [fp, fp, fp, ci, ci, ci, ci, ci, cd, ci]
        lib.oracle_round_bf16.argtypes = [fp, fp, cl]
        for name in ("oracle_biwkv_direct", "oracle_biwkv_rnn",
                     "oracle_biwkv_rnn_literal"):
            getattr(lib, name).argtypes = [dp, dp, dp, dp, dp, ci, ci, ci]
        lib.oracle_biwkv_direct_points.argtypes = [dp, dp, dp, dp, ci, ci, ci,
                                                   i64p, cl, dp]
        lib.oracle_gate.argtypes = [dp, dp, dp, cl]
        lib.oracle_biwkv_bwd_direct.argtypes = [dp, dp, dp, dp, dp, ci, ci, ci, dp, dp, dp, dp]
        lib.oracle_biwkv_bwd_columns.argtypes = [dp, dp, dp, dp, dp, ci, ci, ci, ctypes.c_void_p,
                                                 ctypes.c_long, dp, dp, dp, dp, dp]
        lib.oracle_bishift_f64.argtypes = [dp, dp, dp, ci, ci, ci, ci, ci, cd]
        lib.oracle_bishift_f32.argtypes = [ctypes.POINTER(ctypes.c_float)] * 3 + [ci, ci, ci, ci, ci, cd, ci]
        lib.oracle_channel_mix.argtypes = [dp, dp, dp, dp, ci, ci, ci, ci, ci, cd]
        lib.oracle_spatial_core_points.argtypes = [dp, dp, dp, dp, dp, dp, dp, dp, ci, ci, ci,
                                                   ci, ci, cd, ci, ci, i64p, cl, dp]
        lib.oracle_num_threads.restype = ci
        _lib = lib
    return _lib


def _d(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a: np.ndarray, ctype=ctypes.c_double):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def qshift(x, H: int, W: int, shift_pixel: int = 1, gamma: float = 0.25,
           mu=None, eq9_order: bool = False) -> np.ndarray:
    """Q-Shift of x (B, H*W, C): X^dagger, or mu*X + (1-mu)*X^dagger."""
    x = _d(x)
    B, T, C = x.shape
    assert T == H * W
    out = np.empty_like(x)
    mu_p = None
    if mu is not None:
        mu = _d(mu)
        assert mu.shape == (C,)
        mu_p = _ptr(mu)
    _load().oracle_qshift_f64(_ptr(x), _ptr(out), mu_p, B, H, W, C,
                              int(shift_pixel), float(gamma), int(eq9_order))
    return out


def qshift_f32(x, H: int, W: int, shift_pixel: int = 1, gamma: float = 0.25,
               mu=None, round_bf16: bool = False) -> np.ndarray:
    """Q-Shift in binary32 with the fixed operation order
    t1 = mu*x, t2 = (1-mu)*x_dagger, out = t1 + t2 (each rounded), then an
    optional round-to-nearest-even to bfloat16.  Returns float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    B, T, C = x.shape
    assert T == H * W
    out = np.empty_like(x)
    mu_p = None
    if mu is not None:
        mu = np.ascontiguousarray(mu, dtype=np.float32)
        mu_p = _ptr(mu, ctypes.c_float)
    _load().oracle_qshift_f32(_ptr(x, ctypes.c_float), _ptr(out, ctypes.c_float),
                              mu_p, B, H, W, C, int(shift_pixel), float(gamma),
                              int(round_bf16))
    return out


def round_bf16(a) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even)."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    out = np.empty_like(a)
    _load().oracle_round_bf16(_ptr(a, ctypes.c_float), _ptr(out, ctypes.c_float),
                              a.size)
    return out


def _biwkv(fn_name: str, k, v, w, u) -> np.ndarray:
    k, v, w, u = _d(k), _d(v), _d(w), _d(u)
    B, T, C = k.shape
    assert v.shape == k.shape and w.shape == (C,) and u.shape == (C,)
    out = np.empty_like(k)
    getattr(_load(), fn_name)(_ptr(k), _ptr(v), _ptr(w), _ptr(u), _ptr(out),
                              B, T, C)
    return out


def biwkv_direct(k, v, w, u) -> np.ndarray:
    """Bi-WKV by direct evaluation of eq. 5, O(B*C*T^2)."""
    return _biwkv("oracle_biwkv_direct", k, v, w, u)


def biwkv_rnn(k, v, w, u) -> np.ndarray:
    """Bi-WKV by the RNN form of eq. 6-7, O(B*C*T)."""
    return _biwkv("oracle_biwkv_rnn", k, v, w, u)


def biwkv_rnn_literal(k, v, w, u) -> np.ndarray:
    """Bi-WKV by eq. 6-7 with subtract-and-divide updates for b and d."""
    return _biwkv("oracle_biwkv_rnn_literal", k, v, w, u)


def biwkv_points(k, v, w, u, flat_idx) -> np.ndarray:
    """eq. 5 evaluated only at flat indices (b*T + t)*C + c."""
    k, v, w, u = _d(k), _d(v), _d(w), _d(u)
    B, T, C = k.shape
    idx = np.ascontiguousarray(flat_idx, dtype=np.int64)
    out = np.empty(idx.shape[0], dtype=np.float64)
    _load().oracle_biwkv_direct_points(
        _ptr(k), _ptr(v), _ptr(w), _ptr(u), B, T, C,
        idx.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), idx.shape[0],
        _ptr(out))
    return out


def gate(r, wkv) -> np.ndarray:
    """sigma(r) * wkv (eq. 2)."""
    r, wkv = _d(r), _d(wkv)
    out = np.empty_like(wkv)
    _load().oracle_gate(_ptr(r), _ptr(wkv), _ptr(out), wkv.size)
    return out


def spatial_core(r, k, v, w, u, H=None, W=None, shift_pixel=1, gamma=0.25,
                 mu_r=None, mu_k=None, mu_v=None, qshift_on=True,
                 method: str = "direct") -> np.ndarray:
    """sigma(QS_R(r)) * Bi-WKV(QS_K(k), QS_V(v)); without Q-Shift when
    qshift_on is False.  method selects eq. 5 ("direct") or eq. 6-7 ("rnn")."""
    if qshift_on:
        r = qshift(r, H, W, shift_pixel, gamma, mu_r)
        k = qshift(k, H, W, shift_pixel, gamma, mu_k)
        v = qshift(v, H, W, shift_pixel, gamma, mu_v)
    f = biwkv_direct if method == "direct" else biwkv_rnn
    return gate(r, f(k, v, w, u))


def spatial_core_points(r, k, v, w, u, H, W, flat_idx, shift_pixel=1, gamma=0.25,
                        mu_r=None, mu_k=None, mu_v=None, qshift_on=True,
                        gate_on=True) -> np.ndarray:
    """spatial_core (or Bi-WKV alone when gate_on is False) at flat indices
    (b*T + t)*C + c, building each needed Q-Shifted column on the fly."""
    k, v, w, u = _d(k), _d(v), _d(w), _d(u)
    r = _d(r) if r is not None else k
    B, T, C = k.shape
    assert T == H * W
    idx = np.ascontiguousarray(flat_idx, dtype=np.int64)
    out = np.empty(idx.shape[0], dtype=np.float64)
    mus = [None if m is None else _d(m) for m in (mu_r, mu_k, mu_v)]
    mps = [None if m is None else _ptr(m) for m in mus]
    _load().oracle_spatial_core_points(
        _ptr(r), _ptr(k), _ptr(v), _ptr(w), _ptr(u), mps[0], mps[1], mps[2], B, H, W, C,
        int(shift_pixel), float(gamma), int(qshift_on), int(gate_on),
        idx.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), idx.shape[0], _ptr(out))
    return out


def channel_mix(x, H, W, shift_pixel=1, gamma=0.25, mu_r=None, mu_k=None) -> np.ndarray:
    """sigma(QS_R(x)) * SquaredReLU(QS_K(x)) (eq. 3-4, identity projections)."""
    x = _d(x)
    B, T, C = x.shape
    assert T == H * W
    out = np.empty_like(x)
    mus = [None if m is None else _d(m) for m in (mu_r, mu_k)]
    _load().oracle_channel_mix(_ptr(x), None if mus[0] is None else _ptr(mus[0]),
                               None if mus[1] is None else _ptr(mus[1]), _ptr(out), B, H, W, C,
                               int(shift_pixel), float(gamma))
    return out


def biwkv_bwd(k, v, w, u, gy):
    """Gradients of eq. 5: (gk, gv) of shape (B, T, C) and (gw, gu) of shape
    (B, C), the per-batch contributions to dL/dw and dL/du."""
    k, v, gy = _d(k), _d(v), _d(gy)
    w, u = _d(w), _d(u)
    B, T, C = k.shape
    gk, gv = np.empty_like(k), np.empty_like(k)
    gw, gu = np.empty((B, C)), np.empty((B, C))
    _load().oracle_biwkv_bwd_direct(_ptr(k), _ptr(v), _ptr(w), _ptr(u), _ptr(gy), B, T, C,
                                    _ptr(gk), _ptr(gv), _ptr(gw), _ptr(gu))
    return gk, gv, gw, gu


def biwkv_bwd_columns(k, v, w, u, gy, cols, with_scale: bool = False):
    """biwkv_bwd restricted to the flat columns cols[j] = b*C + c: gk, gv of
    shape (n, T); gw, gu of shape (n,).  With with_scale, also the sums of
    the absolute values of each gradient's terms: (sk, sv) of shape (n, T)
    and (sw, su) of shape (n,)."""
    k, v, gy = _d(k), _d(v), _d(gy)
    w, u = _d(w), _d(u)
    B, T, C = k.shape
    cols = np.ascontiguousarray(cols, dtype=np.int64)
    n = cols.size
    gk, gv = np.empty((n, T)), np.empty((n, T))
    gw, gu = np.empty(n), np.empty(n)
    sc = np.empty((n, 2 * T + 2)) if with_scale else None
    _load().oracle_biwkv_bwd_columns(_ptr(k), _ptr(v), _ptr(w), _ptr(u), _ptr(gy), B, T, C,
                                     cols.ctypes.data, n, _ptr(gk), _ptr(gv), _ptr(gw), _ptr(gu),
                                     None if sc is None else _ptr(sc))
    if with_scale:
        return gk, gv, gw, gu, (sc[:, :T], sc[:, T:2 * T], sc[:, 2 * T], sc[:, 2 * T + 1])
    return gk, gv, gw, gu


def layer_norm(y, g, b, eps: float = 1e-5) -> np.ndarray:
    """LayerNorm over the last (channel) axis: g * (y - mean) / sqrt(var + eps)
    + b, with the biased variance, in float64."""
    y = _d(y)
    mean = y.mean(axis=-1, keepdims=True)
    var = ((y - mean) ** 2).mean(axis=-1, keepdims=True)
    return _d(g) * (y - mean) / np.sqrt(var + eps) + _d(b)


def _bf16(a):
    """Round float64 values to bfloat16 (nearest even), back to float64."""
    a32 = np.ascontiguousarray(a, dtype=np.float32)
    return round_bf16(a32).astype(np.float64)


def spatial_mix_block(x, w_r, w_k, w_v, w_o, w, u, mu_r, mu_k, mu_v, ln_g, ln_b, H, W,
                      shift_pixel=1, gamma=0.25, eps=1e-5, method="rnn",
                      round_like_bf16: bool = False) -> np.ndarray:
    """The spatial-mix block of "Vision-RWKV Backbone", Overall Architecture:
    R = QS_R(x) W_R, K = QS_K(x) W_K, V = QS_V(x) W_V (eq. 1, Q-Shift of eq. 9),
    O = (sigma(R) (.) Bi-WKV(K, V)) W_O (eq. 2, eq. 5), then LayerNorm of O over
    channels (the pages normalise after the output projection).  Weights are
    (C_in, C_out): row vectors times W.  With round_like_bf16 the stored
    intermediates (the three shifted inputs, R, K, V, the gated core and O)
    are rounded to bfloat16, as a bfloat16 implementation stores them."""
    x = _d(x)
    B, T, C = x.shape
    rnd = _bf16 if round_like_bf16 else (lambda a: a)
    xr = rnd(qshift(x, H, W, shift_pixel, gamma, mu_r))
    xk = rnd(qshift(x, H, W, shift_pixel, gamma, mu_k))
    xv = rnd(qshift(x, H, W, shift_pixel, gamma, mu_v))
    R = rnd(xr @ _d(w_r))
    K = rnd(xk @ _d(w_k))
    V = rnd(xv @ _d(w_v))
    f = biwkv_direct if method == "direct" else biwkv_rnn
    core = rnd(gate(R, f(K, V, w, u)))
    O = rnd(core @ _d(w_o))
    return layer_norm(O, ln_g, ln_b, eps)


def bishift(x, H, W, shift_pixel=1, gamma=0.25, mu=None) -> np.ndarray:
    """Bidirectional shift (sparse-input Q-Shift): [0, g) from w - s,
    [g, 2g) from w + s (zero past the row), other channels unchanged; or the
    mu interpolation with x, in float64."""
    x = _d(x)
    B, T, C = x.shape
    assert T == H * W
    out = np.empty_like(x)
    _load().oracle_bishift_f64(_ptr(x), _ptr(out), None if mu is None else _ptr(_d(mu)), B, H, W, C,
                               int(shift_pixel), float(gamma))
    return out


def bishift_f32(x, H, W, shift_pixel=1, gamma=0.25, mu=None, round_bf16=False) -> np.ndarray:
    """bishift in binary32 with the fixed operation order of qshift_f32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    B, T, C = x.shape
    out = np.empty_like(x)
    fp = ctypes.POINTER(ctypes.c_float)
    m = None if mu is None else np.ascontiguousarray(mu, dtype=np.float32)
    _load().oracle_bishift_f32(_ptr(x, ctypes.c_float), _ptr(out, ctypes.c_float),
                               None if m is None else _ptr(m, ctypes.c_float), B, H, W, C,
                               int(shift_pixel), float(gamma), int(round_bf16))
    return out
