"""Seeded synthetic inputs shaped like the Vision-RWKV spatial-mix workloads.

This module only draws numbers; it holds none of the method's arithmetic, so
both the CUDA path and the float64 oracle can consume its output.

Generator: SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom
number generators", OOPSLA 2014) used as a counter-based stream.  Value i of
stream (seed, sid) is mix(key + (i + 1) * 0x9E3779B97F4A7C15) with
key = mix(seed * 256 + sid); a uniform in [0, 1) is the top 53 bits times
2^-53, and a normal pairs uniforms 2i and 2i+1 through the Box-Muller
transform.  Everything is drawn in float64 and then rounded once to the
input/output dtype (float32 or bfloat16, round-to-nearest-even); the rounded
values, widened back to float64, are what the oracle sees.

Workload recipes (token grids of 14x14 = 224^2 images and 64x64 = 1024^2
images at patch 16; distribution "N(0, s)" means standard deviation s):
  1  Bi-WKV only,              B=1,  14x14, C=192,  fp32
  2  Q-Shift + Bi-WKV,         B=32, 14x14, C=384,  fp32
  3  Q-Shift + Bi-WKV + gate,  B=64, 14x14, C=768,  bf16 (separate r, k, v)
  4  Bi-WKV only,              B=4,  64x64, C=768,  bf16
  5  Q-Shift + Bi-WKV + gate,  B=8,  64x64, C=1024, bf16 (one x feeds r,k,v)
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# stream ids of each named tensor
STREAMS = {"x": 0, "r": 1, "k": 2, "v": 3, "w": 4, "u": 5,
           "mu_r": 6, "mu_k": 7, "mu_v": 8}


def _mix(z: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def _key(seed: int, sid: int) -> np.uint64:
    base = np.array([(seed * 256 + sid) & 0xFFFFFFFFFFFFFFFF], dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix(base + _GOLDEN)[0]


def uniform(seed: int, sid: int, n: int, offset: int = 0) -> np.ndarray:
    """n uniforms in [0, 1) from stream (seed, sid), starting at counter offset."""
    i = np.arange(offset + 1, offset + n + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = _mix(_key(seed, sid) + i * _GOLDEN)
    return (z >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)


def normal(seed: int, sid: int, n: int) -> np.ndarray:
    """n standard normals (Box-Muller on consecutive uniform pairs)."""
    u = uniform(seed, sid, 2 * n)
    u1, u2 = u[0::2], u[1::2]
    return np.sqrt(-2.0 * np.log1p(-u1)) * np.cos(2.0 * np.pi * u2)


def draw(seed: int, name: str, shape, dist: tuple) -> np.ndarray:
    """Draw a float64 array: dist = ("normal", std) or ("uniform", lo, hi)."""
    n = int(np.prod(shape))
    sid = STREAMS[name]
    if dist[0] == "normal":
        a = dist[1] * normal(seed, sid, n)
    elif dist[0] == "uniform":
        a = dist[1] + (dist[2] - dist[1]) * uniform(seed, sid, n)
    else:
        raise ValueError(dist)
    return a.reshape(shape)


@dataclass
class Workload:
    """One synthetic workload: shapes, I/O dtype, call and distributions."""
    name: str
    B: int
    H: int
    W: int
    C: int
    dtype: str                  # "f32" or "bf16"
    call: str                   # "biwkv", "qshift_biwkv", "gate_qs", "gate_qs_x"
    dists: dict = field(default_factory=dict)
    shift_pixel: int = 1
    gamma: float = 0.25
    seed: int = 0

    @property
    def T(self) -> int:
        return self.H * self.W

    @property
    def N(self) -> int:
        return self.B * self.T * self.C

    def tensor_names(self):
        if self.call == "biwkv":
            return ["k", "v"]
        if self.call == "qshift_biwkv":
            return ["x", "k", "v"]
        if self.call == "gate_qs":
            return ["r", "k", "v"]
        if self.call == "gate_qs_x":
            return ["x"]
        if self.call == "gate":      # sigma(r) * Bi-WKV(k, v), no Q-Shift
            return ["r", "k", "v"]
        if self.call == "gate_x":    # one x feeds r, k and v, no Q-Shift
            return ["x"]
        raise ValueError(self.call)

    def generate(self) -> dict:
        """All float64 inputs of the workload, keyed by name."""
        out = {}
        for name in self.tensor_names():
            out[name] = draw(self.seed, name, (self.B, self.T, self.C),
                             self.dists[name])
        for name in ("w", "u"):
            out[name] = draw(self.seed, name, (self.C,), self.dists[name])
        if self.call not in ("biwkv", "gate", "gate_x"):
            for name in ("mu_r", "mu_k", "mu_v"):
                out[name] = draw(self.seed, name, (self.C,), ("uniform", 0.0, 1.0))
        return out


def _n(s):
    return ("normal", s)


def _u(lo, hi):
    return ("uniform", lo, hi)


WORKLOADS = {
    1: Workload("biwkv_B1_T196_C192_f32", 1, 14, 14, 192, "f32", "biwkv",
                {"k": _n(1.0), "v": _n(1.0), "w": _n(1.0), "u": _n(0.5)}),
    2: Workload("qshift_biwkv_B32_T196_C384_f32", 32, 14, 14, 384, "f32",
                "qshift_biwkv",
                {"x": _n(1.0), "k": _n(1.0), "v": _n(1.0), "w": _u(-3, 3),
                 "u": _n(0.5)}),
    3: Workload("spatial_gate_B64_T196_C768_bf16", 64, 14, 14, 768, "bf16",
                "gate_qs",
                {"r": _n(1.0), "k": _n(1.0), "v": _n(1.0), "w": _u(-3, 3),
                 "u": _n(0.5)}),
    4: Workload("biwkv_B4_T4096_C768_bf16", 4, 64, 64, 768, "bf16", "biwkv",
                {"k": _n(2.0), "v": _n(1.0), "w": _u(-8, 8), "u": _n(1.0)}),
    5: Workload("spatial_gate_x_B8_T4096_C1024_bf16", 8, 64, 64, 1024, "bf16",
                "gate_qs_x",
                {"x": _n(1.0), "w": _u(-5, 5), "u": _n(1.0)}),
}
for _i, _wl in WORKLOADS.items():
    _wl.seed = 20260000 + _i


def workload(i: int, **overrides) -> Workload:
    """A copy of recipe i with fields overridden (e.g. a smaller B)."""
    import dataclasses
    return dataclasses.replace(WORKLOADS[i], **overrides)
