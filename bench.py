#!/usr/bin/env python
"""Benchmark of the B200 Vision-RWKV spatial-mix core.

One step = one pass of the whole hot path over one batch: Q-Shift of x into
r, k and v, Bi-WKV (eq. 5) and the sigma(R) gate, fused in one kernel launch
(default workload: B=8, 64x64 token grid (T=4096, a 1024^2 image at patch
16), C=1024, bfloat16 I/O, one x shared by r, k and v).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 1..5]
                    [--impl ours|reference]

Timing: the K timed launches are replayed from CUDA graphs (one graph of
min(K, 64-ish) launches replayed, one more for any remainder, so every timed
launch is graph-replayed at any K) between a barrier + synchronize on each
side, timed with CUDA events on the launching stream; the max over ranks is
taken.  SM clocks are sampled from a short pre-roll of the same launches
(about 0.3 s, just before the timed region) through the end of the timed
region, so a short region still gets many samples.  Inputs and outputs rotate over enough
buffer sets that every launch reads and writes memory not touched for more
than an L2's worth of traffic.  Multi-GPU runs are replicas (every (b, c)
column is independent): each rank processes its own batch, no collective
touches the data path, and the value is the whole-job throughput.

The JSON line also carries the roofline of the fused kernel (algorithmic
bytes / average launch time against the measured HBM copy bandwidth), its
instruction-issue roofline (``issue_roofline``: ncu's warp-instruction count
per launch over the launch time, against 4 per SM per clock; the kernel is
bound by issue, not by HBM), an
end-to-end figure through the C ABI with host buffers, the float64 CPU
oracle timed on a bounded sample, and SM clocks sampled during the timed
region.  ``--impl reference`` times the CPU oracle alone on the same metric.
``rows.channel_mix`` adds the roofline of the channel-mix elementwise path
(eq. 3-4 with identity projections) on the same x buffers and
``rows.biwkv_bwd`` that of the Bi-WKV backward at the workload's shape;
``rows.fused_workspace`` times the main step through the workspace entry
points (global-memory exchange instead of clusters), and
``rows.spatial_mix_block`` the block with projections and LayerNorm.  Each is timed in its
own region after the main one (``--no-rows`` skips them).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from linear_complexity_vision_b200 import synth  # noqa: E402

METRIC = ("Bi-WKV fused fwd tokens·ch/s and HBM GB/s (% of B200 peak) "
          "at T=196–4096")
UNIT = "tokens*ch/s"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, nominal (~8 TB/s)
CSRC = os.path.join(ROOT, "linear_complexity_vision_b200", "csrc")


# CUDA sources each kernel is compiled from; a traffic record holds only while
# they are unchanged (a change of launch shape comes with a new capture).
KERNEL_SOURCES = {
    "biwkv_tma_kernel": ("common.cuh", "biwkv_tma.cuh"),
    "biwkv_tm_kernel": ("common.cuh", "biwkv_tma.cuh", "biwkv_tm.cuh"),
    "biwkv_wide_kernel": ("common.cuh", "biwkv_tma.cuh", "biwkv_wide.cuh"),
    "biwkv_fused_kernel": ("common.cuh", "qshift.cuh", "biwkv.cuh"),
    "channel_mix_vec_kernel": ("common.cuh", "qshift.cuh", "channel_mix.cuh"),
    "biwkv_bwd_kernel": ("common.cuh", "biwkv_tma.cuh", "biwkv_bwd.cuh"),
    "biwkv_bwd_tm_kernel": ("common.cuh", "biwkv_tma.cuh", "biwkv_tm.cuh", "biwkv_bwd.cuh", "biwkv_bwd_tm.cuh"),
}


def code_only(text: str) -> str:
    """CUDA/C++ source without comments, trailing blanks or empty lines: the
    part that decides what the kernel does (the sources hold no string that
    contains a comment marker)."""
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = (re.sub(r"//.*$", "", ln).rstrip() for ln in text.splitlines())
    return "\n".join(ln for ln in lines if ln)


def kernel_source_hash(kernel: str) -> str:
    """Hash of the code (comments and blank lines left out) of the CUDA
    sources `kernel` is built from: a traffic record stays valid across
    comment edits and is dropped by any change to the code."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(CSRC, f), encoding="utf-8") as fh:
            h.update(f.encode())
            h.update(code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def algorithmic_bytes(wl) -> dict:
    """Bytes a launch must move at minimum: inputs read once, output written
    once, parameter vectors read once.  Returns per-call bytes."""
    es = 4 if wl.dtype == "f32" else 2
    N, C = wl.N, wl.C
    if wl.call == "biwkv":
        return {"fused": 3 * N * es + 2 * C * 4}
    if wl.call == "qshift_biwkv":
        return {"qshift": 2 * N * es + C * 4, "fused": 3 * N * es + 4 * C * 4}
    if wl.call == "gate_qs":
        return {"fused": 4 * N * es + 5 * C * 4}
    return {"fused": 2 * N * es + 5 * C * 4}  # gate_qs_x: x once, out once


# ---------------------------------------------------------------------------
# distributed plumbing (replicas; used for the barrier and max-over-ranks)
# ---------------------------------------------------------------------------
class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None

    def init(self, backend: str):
        if self.world > 1:
            import torch.distributed as dist
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
            self.pg = dist

    def barrier(self):
        if self.pg is not None:
            self.pg.barrier()

    def max(self, x: float, device) -> float:
        if self.pg is None:
            return x
        import torch
        t = torch.tensor([x], dtype=torch.float64, device=device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg is not None:
            self.pg.destroy_process_group()


# ---------------------------------------------------------------------------
# clocks sampled during the timed region (NVML, read-only queries)
# ---------------------------------------------------------------------------
class ClockSampler:
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x2: "applications_clocks_setting", 0x10: "sync_boost", 0x1: "gpu_idle"}

    def __init__(self, local_rank: int, period_s: float = 0.01,
                 window: str = "pre-roll of the same launches (~0.3 s) + the timed region"):
        self.samples, self.reasons = [], 0
        self.window = window
        self.max_mhz = None
        self.ok = False
        self.period = period_s
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = local_rank
            if vis:
                ids = [v.strip() for v in vis.split(",") if v.strip()]
                if local_rank < len(ids) and ids[local_rank].isdigit():
                    idx = int(ids[local_rank])
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self._reason_fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                getattr(pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons")
            self.ok = True
        except Exception:  # no NVML: report no clocks rather than fail
            self.ok = False

    def _sample(self):
        try:
            mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
            rs = int(self._reason_fn(self.h))
            self.samples.append(mhz)
            self.reasons |= rs & ~0x1
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if self.ok:
            self._sample()
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return None
        return {"sm_mhz": float(np.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "samples": len(self.samples),
                "window": self.window,
                "reasons": sorted(n for b, n in self.REASONS.items() if self.reasons & b)}


def row_clocks(dev) -> ClockSampler:
    """SM clocks sampled every 2 ms over one row's timed region (a row times
    tens of milliseconds, after other rows that may have heated the GPU)."""
    c = ClockSampler(dev.index or 0, period_s=0.002, window="the row's timed region")
    c.start()
    return c


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def measured_hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def committed_record(key: str, kernel: str):
    """The committed ncu record of `kernel` on this workload, if it was taken
    on the kernel as currently written (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            rec = json.load(f)
        # the workload's record, or one kept for another kernel of the same
        # workload (e.g. "wide/<workload>")
        for k, ent in rec.items():
            if not isinstance(ent, dict) or not (k == key or k.endswith("/" + key)):
                continue
            if ent.get("kernel") == kernel and ent.get("kernel_sha") == kernel_source_hash(kernel):
                return ent
    except Exception:
        pass
    return None


def committed_traffic(key: str, kernel: str):
    """dram bytes per launch from the committed ncu summary, if it was taken
    on `kernel` as currently written and on this workload."""
    ent = committed_record(key, kernel)
    return float(ent["dram_bytes_per_launch"]) if ent else None


WARP_SCHEDULERS_PER_SM = 4  # one warp-instruction issued per scheduler per clock


def issue_roofline(warp_inst_per_launch, launch_s, sms, sm_mhz):
    """Instruction-issue roofline of a kernel bound by its arithmetic rather
    than by HBM: warp-instructions per launch (ncu smsp__inst_executed.sum)
    over the launch time, against SMs x 4 schedulers x 1 per clock at the SM
    clock sampled during the run."""
    if not warp_inst_per_launch or not launch_s or not sms or not sm_mhz:
        return None
    achieved = warp_inst_per_launch / launch_s / 1e9
    peak = sms * WARP_SCHEDULERS_PER_SM * sm_mhz / 1e3
    return {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "G warp-instructions/s",
            "frac": achieved / peak, "warp_inst_per_launch": warp_inst_per_launch,
            "peak_basis": f"{sms} SMs x {WARP_SCHEDULERS_PER_SM} schedulers x 1/clock x {sm_mhz:.0f} MHz"}


def make_inputs(wl, torch, dev, rank):
    """Device tensors of one input set plus float64 copies for checks."""
    import dataclasses
    wlr = dataclasses.replace(wl, seed=wl.seed + 1000003 * rank)
    inp = wlr.generate()
    tdt = torch.float32 if wl.dtype == "f32" else torch.bfloat16
    host = {n: torch.from_numpy(inp[n]).to(tdt) for n in wl.tensor_names()}
    par = {n: torch.from_numpy(inp[n]).to(torch.float32) for n in inp if n not in host}
    return inp, host, par, tdt


def rotation_sets(wl) -> int:
    """Input/output buffer sets the timed launches rotate over: enough that
    every launch reads and writes memory untouched for over 3x the L2."""
    es = 4 if wl.dtype == "f32" else 2
    per_set = (len(wl.tensor_names()) + 1) * wl.N * es
    return max(2, int(np.ceil(3 * L2_BYTES / per_set)) + 1)


def bench_config(wl, world: int) -> dict:
    """The workload as both arms report it."""
    n = rotation_sets(wl)
    es = 4 if wl.dtype == "f32" else 2
    mb = n * (len(wl.tensor_names()) + 1) * wl.N * es / 1e6
    return {"workload": wl.name, "B": wl.B, "T": wl.T, "H": wl.H, "W": wl.W, "C": wl.C,
            "call": wl.call, "shift_pixel": wl.shift_pixel, "gamma": wl.gamma,
            "io_dtype": wl.dtype, "accumulate": "f32",
            "l2": f"inputs larger than L2: rotating {n} input/output buffer sets "
                  f"({mb:.0f} MB > 126 MB L2)",
            "parallelism": f"replicas x{world} (independent batches, no collective)"}


class Runner:
    """Holds the rotating buffer sets and launches one step on set i."""

    def __init__(self, vk, wl, torch, dev, rank):
        self.vk, self.wl, self.torch = vk, wl, torch
        self.inp, host, par, tdt = make_inputs(wl, torch, dev, rank)
        self.host = host
        self.par = {n: t.to(dev) for n, t in par.items()}
        self.nsets = rotation_sets(wl)
        self.sets = []
        shape = (wl.B, wl.T, wl.C)
        for _ in range(self.nsets):
            d = {n: t.to(dev) for n, t in host.items()}
            d["out"] = torch.empty(shape, dtype=tdt, device=dev)
            if wl.call == "qshift_biwkv":
                d["xs"] = torch.empty(shape, dtype=tdt, device=dev)
            self.sets.append(d)
        if wl.call != "biwkv":
            self.qs = vk.QShift(wl.H, wl.W, wl.shift_pixel, wl.gamma, self.par.get("mu_r"),
                                self.par.get("mu_k"), self.par.get("mu_v"))
        self.launches_per_step = 2 if wl.call == "qshift_biwkv" else 1

    @property
    def kernel_name(self) -> str:
        """Name of the fused kernel the library launched last on this thread."""
        return self.vk.load_library().vrwkv_last_kernel().decode()

    def step(self, i: int):
        d = self.sets[i % self.nsets]
        vk, p, wl = self.vk, self.par, self.wl
        if wl.call == "biwkv":
            vk.biwkv_fwd(d["k"], d["v"], p["w"], p["u"], out=d["out"])
        elif wl.call == "qshift_biwkv":
            vk.qshift(d["x"], wl.H, wl.W, wl.shift_pixel, wl.gamma, mu=p["mu_r"], out=d["xs"])
            vk.biwkv_fwd(d["k"], d["v"], p["w"], p["u"], qs=self.qs, out=d["out"])
        elif wl.call == "gate_qs":
            vk.spatial_gate(d["r"], d["k"], d["v"], p["w"], p["u"], qs=self.qs, out=d["out"])
        else:
            x = d["x"]
            vk.spatial_gate(x, x, x, p["w"], p["u"], qs=self.qs, out=d["out"])
        return d["out"]

    def step_host(self, hin: dict, hout, dbuf: dict):
        """One end-to-end step: pinned host inputs -> device -> C ABI -> host."""
        for n, t in hin.items():
            dbuf[n].copy_(t, non_blocking=True)
        out = self.step_on(dbuf)
        hout.copy_(out, non_blocking=True)

    def step_on(self, d):
        saved = self.sets
        self.sets = [d]
        try:
            return self.step(0)
        finally:
            self.sets = saved


def time_channel_mix(runner, stream, torch, dev, launches: int, peak: float):
    """Roofline of the channel-mix elementwise path (eq. 3-4 with identity
    projections) on the workload's x buffers, outside the main timed region:
    CUDA graphs over the same rotating buffer sets, events on the stream."""
    wl, vk = runner.wl, runner.vk
    if "x" not in runner.sets[0]:
        return None
    n = runner.nsets
    outs = [torch.empty_like(d["x"]) for d in runner.sets]

    def launch(i):
        vk.channel_mix(runner.sets[i % n]["x"], runner.qs, out=outs[i % n])

    with torch.cuda.stream(stream):
        for i in range(3):
            launch(i)
    torch.cuda.synchronize(dev)
    G = n * max(1, 64 // n)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(G):
            launch(i)
    reps = max(1, launches // G)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    row_clk = row_clocks(dev)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(reps):
            graph.replay()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    row_clk.stop()
    del graph
    us = e0.elapsed_time(e1) * 1e3 / (reps * G)
    es = 4 if wl.dtype == "f32" else 2
    nbytes = 2 * wl.N * es + 2 * wl.C * 4  # x once, out once, mu_r and mu_k
    achieved = nbytes / (us * 1e-6) / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak,
            "traffic": committed_traffic("channel_mix/" + wl.name, runner.kernel_name),
            "kernel": runner.kernel_name,
            "algorithmic_bytes_per_launch": nbytes, "avg_launch_us": us,
            "launches": reps * G, "clocks": row_clk.summary()}


def time_fused_ws(runner, stream, torch, dev, launches: int, peak: float):
    """The main step through the workspace entry points (the CTAs of a column
    exchange their sums through global memory instead of a cluster), graph-
    replayed over the same rotating buffer sets."""
    wl, vk = runner.wl, runner.vk
    if wl.T <= 256:
        return None
    ws = vk.fwd_workspace(wl.B, wl.T, wl.C, device=dev)
    n = runner.nsets

    def launch(i):
        d, p = runner.sets[i % n], runner.par
        if wl.call == "biwkv":
            vk.biwkv_fwd(d["k"], d["v"], p["w"], p["u"], out=d["out"], workspace=ws)
        elif wl.call == "qshift_biwkv":
            vk.biwkv_fwd(d["k"], d["v"], p["w"], p["u"], qs=runner.qs, out=d["out"], workspace=ws)
        elif wl.call == "gate_qs":
            vk.spatial_gate(d["r"], d["k"], d["v"], p["w"], p["u"], qs=runner.qs, out=d["out"],
                            workspace=ws)
        else:
            x = d["x"]
            vk.spatial_gate(x, x, x, p["w"], p["u"], qs=runner.qs, out=d["out"], workspace=ws)

    with torch.cuda.stream(stream):
        for i in range(3):
            launch(i)
    torch.cuda.synchronize(dev)
    G = n * max(1, 64 // n)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(G):
            launch(i)
    reps = max(1, launches // G)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    row_clk = row_clocks(dev)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(reps):
            graph.replay()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    row_clk.stop()
    del graph
    vk.device_status()
    us = e0.elapsed_time(e1) * 1e3 / (reps * G)
    nbytes = algorithmic_bytes(wl)["fused"]
    achieved = nbytes / (us * 1e-6) / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "kernel": runner.kernel_name,
            "algorithmic_bytes_per_launch": nbytes, "avg_launch_us": us, "launches": reps * G,
            "exchange": "global-memory workspace (no clusters)", "clocks": row_clk.summary()}


def measured_tensor_peak():
    """Measured dense bf16 GEMM throughput (burst), TFLOP/s."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


def time_block(runner, stream, torch, dev, launches: int):
    """The spatial-mix block with projections (vrwkv_spatial_mix_block) at the
    workload's (B, T, C): Q-Shift, four tcgen05 GEMMs, the fused core and a
    LayerNorm per launch.  Roofline against the dense bf16 peak with the four
    GEMMs' 8*B*T*C^2 FLOPs; random weights of scale 1/sqrt(C)."""
    wl, vk = runner.wl, runner.vk
    if wl.call == "biwkv" or wl.dtype != "bf16":
        return None
    g = torch.Generator(device=dev).manual_seed(20260202)
    C = wl.C
    mats = tuple((torch.randn(C, C, generator=g, device=dev) / C ** 0.5).to(torch.bfloat16)
                 for _ in range(4))
    lg = 1 + 0.1 * torch.randn(C, generator=g, device=dev)
    lb = 0.1 * torch.randn(C, generator=g, device=dev)
    p = runner.par
    ws = vk.block_workspace(wl.B, wl.T, C, torch.bfloat16, device=dev)
    n = runner.nsets
    key = "x" if "x" in runner.sets[0] else "k"
    outs = [torch.empty_like(d[key]) for d in runner.sets]  # the main step's outputs stay intact

    def launch(i):
        d = runner.sets[i % n]
        vk.spatial_mix_block(d[key], mats, p["w"], p["u"], lg, lb, runner.qs, workspace=ws,
                             out=outs[i % n])

    with torch.cuda.stream(stream):
        for i in range(3):
            launch(i)
    torch.cuda.synchronize(dev)
    # replayed from a CUDA graph (the block issues about 13 launches per step:
    # weight transposes, GEMMs, mixes, the core, LayerNorm; the graph keeps
    # host time out of the measurement)
    G = n * max(1, 8 // n)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(G):
            launch(i)
    reps = max(1, launches // G)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    row_clk = row_clocks(dev)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(reps):
            graph.replay()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    row_clk.stop()
    del graph
    vk.device_status()
    us = e0.elapsed_time(e1) * 1e3 / (reps * G)
    launches = reps * G
    flops = 8.0 * wl.B * wl.T * C * C
    peak, kind = measured_tensor_peak()
    achieved = flops / (us * 1e-6) / 1e12
    return {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak, "peak_source": kind, "kernel": "spatial_mix_block",
            "flops_per_launch": flops, "avg_launch_us": us, "launches": launches,
            "gemm": ("hand-written tcgen05 kernel, bf16 operands, float32 accumulation in tensor memory: "
                     + ("gemm_tc_kernel (one CTA per 128x256 tile)" if os.environ.get("VRWKV_GEMM_1CTA") == "1"
                        else "gemm_tc2_kernel (CTA pairs, cta_group::2, 256x256 tiles)")),
            "timing": "CUDA graphs over the rotating buffer sets", "clocks": row_clk.summary()}


def time_biwkv_bwd(runner, stream, torch, dev, launches: int, peak: float, sm_mhz=None):
    """Roofline of the Bi-WKV backward (vrwkv_biwkv_bwd) at the workload's
    (B, T, C) and dtype, timed in its own region: k, v and gy read once, gk
    and gv written once, w, u read and the per-row dw, du written."""
    wl, vk = runner.wl, runner.vk
    if wl.T > 4096:
        return None
    tdt = torch.float32 if wl.dtype == "f32" else torch.bfloat16
    shape = (wl.B, wl.T, wl.C)
    per_set = 5 * wl.N * (4 if wl.dtype == "f32" else 2)
    nsets = max(2, int(np.ceil(2 * L2_BYTES / per_set)))
    g = torch.Generator(device=dev).manual_seed(20260101)
    sets = []
    for _ in range(nsets):
        d = {n: torch.randn(shape, generator=g, device=dev).to(tdt) for n in ("k", "v", "gy")}
        sets.append(d)
    w = torch.rand(wl.C, generator=g, device=dev) * 10 - 5
    u = torch.randn(wl.C, generator=g, device=dev)
    outs = [(torch.empty(shape, dtype=tdt, device=dev), torch.empty(shape, dtype=tdt, device=dev),
             torch.empty((wl.B, wl.C), dtype=torch.float32, device=dev),
             torch.empty((wl.B, wl.C), dtype=torch.float32, device=dev)) for _ in range(2)]

    def launch(i):
        d = sets[i % nsets]
        vk.biwkv_bwd(d["k"], d["v"], w, u, d["gy"], totals=False, out=outs[i % 2])

    with torch.cuda.stream(stream):
        for i in range(3):
            launch(i)
    torch.cuda.synchronize(dev)
    kname = runner.kernel_name
    # the launches as one CUDA graph (preallocated outputs), replayed once
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(graph, stream=stream):
            for i in range(launches):
                launch(i)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    row_clk = row_clocks(dev)
    with torch.cuda.stream(stream):
        e0.record(stream)
        graph.replay()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    row_clk.stop()
    del graph
    us = e0.elapsed_time(e1) * 1e3 / launches
    es = 4 if wl.dtype == "f32" else 2
    nbytes = 5 * wl.N * es + 2 * wl.C * 4 + 2 * wl.B * wl.C * 4
    achieved = nbytes / (us * 1e-6) / 1e9
    rec = committed_record("biwkv_bwd/" + wl.name, kname)
    issue = issue_roofline(rec.get("warp_inst_per_launch") if rec else None, us * 1e-6,
                           torch.cuda.get_device_properties(dev).multi_processor_count, sm_mhz)
    return {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "traffic": committed_traffic("biwkv_bwd/" + wl.name, kname),
            "kernel": kname, "algorithmic_bytes_per_launch": nbytes, "avg_launch_us": us,
            "issue_roofline": issue,
            "launches": launches, "timing": "one CUDA graph of the launches (preallocated outputs)",
            "clocks": row_clk.summary()}


def parity_sample(runner, out_dev, oracle, npts=128):
    """GPU against the float64 oracle on a seeded sample of output positions:
    (max |GPU - oracle|, max |GPU - oracle| / max(|oracle|, 1e-6)); the second,
    a plain relative error, is for information (outputs near zero inflate it)."""
    wl, inp = runner.wl, runner.inp
    got = out_dev.to(runner.torch.float64).cpu().numpy().reshape(-1)
    rng = np.random.default_rng(7)
    idx = np.sort(rng.choice(got.size, size=npts, replace=False))
    tdt = runner.torch.float32 if wl.dtype == "f32" else runner.torch.bfloat16
    r64 = {n: runner.torch.from_numpy(inp[n]).to(tdt).to(runner.torch.float64).numpy()
           for n in wl.tensor_names()}
    p64 = {n: runner.torch.from_numpy(inp[n]).to(runner.torch.float32).double().numpy()
           for n in inp if n not in r64}
    if wl.call == "gate_qs_x":
        r = k = v = r64["x"]
    else:
        r, k, v = r64.get("r"), r64["k"], r64["v"]
    want = oracle.spatial_core_points(
        r, k, v, p64["w"], p64["u"], wl.H, wl.W, idx, wl.shift_pixel, wl.gamma,
        p64.get("mu_r"), p64.get("mu_k"), p64.get("mu_v"),
        qshift_on=wl.call != "biwkv", gate_on=wl.call in ("gate_qs", "gate_qs_x"))
    d = np.abs(got[idx] - want)
    return float(np.max(d)), float(np.max(d / np.maximum(np.abs(want), 1e-6)))


def oracle_throughput(wl, oracle, target_s: float, max_points: int = 1 << 20):
    """The float64 oracle (eq. 5 directly, per output position, with Q-Shift
    and gate) on a seeded sample of output positions of the workload, sized
    to take about target_s seconds.  Returns (tokens*ch/s, points, seconds)."""
    inp = wl.generate()
    if wl.call == "gate_qs_x":
        r = k = v = inp["x"]
    else:
        r, k, v = inp.get("r"), inp["k"], inp["v"]
    qs_on = wl.call != "biwkv"
    gate_on = wl.call in ("gate_qs", "gate_qs_x")
    rng = np.random.default_rng(11)

    def run(n):
        idx = rng.integers(0, wl.N, size=n)
        t0 = time.perf_counter()
        oracle.spatial_core_points(r, k, v, inp["w"], inp["u"], wl.H, wl.W, idx, wl.shift_pixel,
                                   wl.gamma, inp.get("mu_r"), inp.get("mu_k"), inp.get("mu_v"),
                                   qshift_on=qs_on, gate_on=gate_on)
        return time.perf_counter() - t0

    n = 4 * oracle.num_threads()
    dt = run(n)
    while dt < 0.5 and n < max_points:
        n *= 4
        dt = run(n)
    n = int(min(max_points, max(n, n * target_s / max(dt, 1e-9))))
    dt = run(n)
    return n / dt, n, dt


def run_ours(args, dist):
    import torch
    import linear_complexity_vision_b200 as vk
    vk.load_library()  # fail loudly if the CUDA library is missing
    dev = torch.device("cuda", dist.local_rank)
    torch.cuda.set_device(dev)
    dist.init("nccl")
    wl = synth.WORKLOADS[args.workload]
    runner = Runner(vk, wl, torch, dev, dist.rank)
    stream = torch.cuda.Stream(device=dev)

    # warm-up (also raises the kernel's shared-memory limit before capture)
    with torch.cuda.stream(stream):
        for i in range(max(3, args.warmup)):
            out = runner.step(i)
    torch.cuda.synchronize(dev)

    # The timed launches as CUDA graphs: G = min(K, one rotation period of
    # about 64 launches) replayed reps times, then a graph of the remaining
    # launches, so every timed launch is graph-replayed whatever K is.
    # Launch i uses buffer set i mod nsets; G is a multiple of nsets whenever
    # it repeats, so no set is used twice in a row.
    Gmax = runner.nsets * max(1, 64 // runner.nsets)
    G = min(args.steps, Gmax)
    reps, rem = divmod(args.steps, G)

    def capture(n, first):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=stream):
            for i in range(first, first + n):
                runner.step(i)
        return gr

    graph = capture(G, 0)
    graph_rem = capture(rem, reps * G) if rem else None
    torch.cuda.synchronize(dev)

    # clocks: sampled from a pre-roll of the same launches (untimed, about
    # 0.3 s) right before the timed region through its end
    clocks = ClockSampler(dist.local_rank, period_s=0.005)
    clocks.start()
    t_pre = time.perf_counter()
    with torch.cuda.stream(stream):
        while time.perf_counter() - t_pre < 0.3:
            graph.replay()
            torch.cuda.synchronize(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):
        ev0.record(stream)
        for _ in range(reps):
            graph.replay()
        if graph_rem is not None:
            graph_rem.replay()
        ev1.record(stream)
    torch.cuda.synchronize(dev)
    clocks.stop()
    dist.barrier()
    ms_local = ev0.elapsed_time(ev1)
    ms = dist.max(ms_local, dev)
    del graph, graph_rem

    steps = args.steps
    units = wl.N
    value = dist.world * steps * units / (ms / 1e3)
    ms_per_step = ms / steps

    # roofline of the fused kernel: the timed region holds only our launches
    # back to back, so the average launch time is (region / launches)
    ab = algorithmic_bytes(wl)
    launch_s = (ms_local / 1e3) / (steps * runner.launches_per_step)
    fused_bytes = ab["fused"]
    if wl.call == "qshift_biwkv":  # two kernels: attribute by bytes
        fused_share = ab["fused"] / (ab["fused"] + ab["qshift"])
        launch_s = (ms_local / 1e3) * fused_share / steps
    peak, peak_kind = measured_hbm_peak()
    achieved = fused_bytes / launch_s / 1e9
    traffic = committed_traffic(wl.name, runner.kernel_name)
    rec = committed_record(wl.name, runner.kernel_name)
    clk = clocks.summary()
    issue = issue_roofline(rec.get("warp_inst_per_launch") if rec else None, launch_s,
                           torch.cuda.get_device_properties(dev).multi_processor_count,
                           (clk or {}).get("sm_mhz") or (clk or {}).get("sm_max_mhz"))

    # end to end through the C ABI with pinned host buffers.  The gated
    # workloads call vrwkv_spatial_gate_host, which streams batch slices of
    # one row through two device slots so the host-to-device copies, the
    # kernels and the copies back overlap; the others copy in, run and copy
    # out in order on one stream.
    e2e_steps = max(3, min(args.steps, 50))
    hin = {n: t.pin_memory() for n, t in runner.host.items()}
    hout = torch.empty((wl.B, wl.T, wl.C), dtype=next(iter(hin.values())).dtype).pin_memory()
    dbuf = dict(runner.sets[0])
    if wl.call in ("gate_qs", "gate_qs_x"):
        if wl.call == "gate_qs_x":
            hr = hk = hv = hin["x"]
        else:
            hr, hk, hv = hin["r"], hin["k"], hin["v"]
        stage = vk.spatial_gate_host_buffer(hr, hk, hv, 1, device=dev)

        def e2e_step():
            vk.spatial_gate_host(hr, hk, hv, runner.par["w"], runner.par["u"], qs=runner.qs, out=hout,
                                 slice_b=1, dev_buf=stage, stream=stream)
        e2e_path = ("vrwkv_spatial_gate_host: batch slices of 1 row, copy-in / kernel / copy-out "
                    "on three streams, overlapped")
    else:
        def e2e_step():
            runner.step_host(hin, hout, dbuf)
        e2e_path = "copy in, C ABI call, copy out, in order on one stream"
    with torch.cuda.stream(stream):
        e2e_step()
    torch.cuda.synchronize(dev)
    dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = dist.max(e0.elapsed_time(e1), dev)
    h2d = sum(t.numel() * t.element_size() for t in hin.values())
    d2h = hout.numel() * hout.element_size()
    e2e = {"value": dist.world * e2e_steps * units / (e2e_ms / 1e3), "unit": UNIT,
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
           "path": e2e_path}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": dist.world,
        "steps": steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": wl.dtype, "data": "synthetic",
        "config": bench_config(wl, dist.world),
        "timing": (f"{reps} replay(s) of a CUDA graph of {G} launches"
                   + (f" + a graph of {rem}" if rem else "")
                   + ", events on the launching stream"),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic, "peak_source": peak_kind,
                     "frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS,
                     "kernel": runner.kernel_name,
                     "algorithmic_bytes_per_launch": fused_bytes,
                     "avg_launch_us": launch_s * 1e6},
        "issue_roofline": issue,
        "e2e": e2e,
        "gpu_launches": steps * runner.launches_per_step,
        "clocks": clk,
    }
    # correctness guard on the main step's last output (first set of the
    # rotation), taken before the rows below reuse the device
    parity_err = (None, None)
    if dist.rank == 0:
        import oracle
        parity_err = parity_sample(runner, runner.sets[0]["out"], oracle)
    # the next hot-path rows on the same shape (each its own timed region)
    if args.rows:
        cm = time_channel_mix(runner, stream, torch, dev, args.row_launches, peak)
        rows = {}
        if cm is not None:
            rows["channel_mix"] = cm
        gx = time_fused_ws(runner, stream, torch, dev, args.row_launches, peak)
        if gx is not None:
            rows["fused_workspace"] = gx
        blk = time_block(runner, stream, torch, dev, max(20, args.row_launches // 20))
        if blk is not None:
            rows["spatial_mix_block"] = blk
        bw = time_biwkv_bwd(runner, stream, torch, dev, max(20, args.row_launches // 20), peak,
                            sm_mhz=(clk or {}).get("sm_mhz"))
        if bw is not None:
            rows["biwkv_bwd"] = bw
        if rows:
            line["rows"] = rows
    # the guard's result and, on one GPU, the CPU oracle baseline (rank 0)
    if dist.rank == 0:
        import oracle
        line["parity_sample_max_abs_err"] = parity_err[0]
        line["parity_sample_max_rel_err_plain"] = parity_err[1]
        if dist.world == 1 and not args.no_cpu_baseline:
            v, n, dt = oracle_throughput(wl, oracle, target_s=args.cpu_seconds)
            line["cpu_baseline"] = {
                "value": v, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                "sample": f"{n} seeded output positions of the workload; each by direct "
                          f"eq. 5 summation over its T={wl.T} column with Q-Shift and gate, "
                          f"float64 ({dt:.1f} s)"}
        print(json.dumps(line), flush=True)
    dist.close()


# ---------------------------------------------------------------------------
# reference arm: the float64 CPU oracle as it stands
# ---------------------------------------------------------------------------
def run_reference(args, dist):
    if dist.rank != 0:
        return
    import oracle
    wl = synth.WORKLOADS[args.workload]
    inp = wl.generate()
    if wl.call == "gate_qs_x":
        r = k = v = inp["x"]
    else:
        r, k, v = inp.get("r"), inp["k"], inp["v"]
    qs_on, gate_on = wl.call != "biwkv", wl.call in ("gate_qs", "gate_qs_x")
    rng = np.random.default_rng(13)

    def step(n):
        idx = rng.integers(0, wl.N, size=n)
        oracle.spatial_core_points(r, k, v, inp["w"], inp["u"], wl.H, wl.W, idx, wl.shift_pixel,
                                   wl.gamma, inp.get("mu_r"), inp.get("mu_k"), inp.get("mu_v"),
                                   qshift_on=qs_on, gate_on=gate_on)

    # size each step so that warm-up + timed steps take about budget seconds
    t0 = time.perf_counter()
    step(oracle.num_threads())
    per_point = (time.perf_counter() - t0) / oracle.num_threads()
    total = max(1, args.steps + args.warmup)
    n = max(1, int(args.reference_seconds / total / per_point))
    for _ in range(args.warmup):
        step(n)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step(n)
    dt = time.perf_counter() - t0
    value = args.steps * n / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": dist.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": bench_config(wl, dist.world),
        "cpu_baseline": {"value": value, "unit": UNIT, "kind": "oracle",
                         "cores": oracle.num_threads(),
                         "sample": f"{n} seeded output positions per step, each by direct eq. 5 "
                                   f"summation over its T={wl.T} column with Q-Shift and gate"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--workload", type=int, default=5, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--reference-seconds", type=float, default=60.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-rows", dest="rows", action="store_false",
                    help="skip the channel-mix and backward row measurements")
    ap.add_argument("--row-launches", type=int, default=4000)
    args = ap.parse_args(argv)
    dist = Dist()
    if args.impl == "reference":
        run_reference(args, dist)
    else:
        run_ours(args, dist)


if __name__ == "__main__":
    main()
