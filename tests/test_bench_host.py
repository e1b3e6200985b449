"""Host-side logic of bench.py on CPU: the max-over-ranks timing reduction and
barrier with world_size 2 over gloo, the reference arm's rank gating, and the
algorithmic byte accounting."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    d = bench.Dist()
    d.init("gloo")
    d.barrier()
    got = d.max(10.0 * (rank + 1), "cpu")
    d.close()
    q.put((rank, got))


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(2))
    assert res == {0: 20.0, 1: 20.0}


def test_single_process_dist_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    d = bench.Dist()
    assert d.world == int(os.environ.get("WORLD_SIZE", "1"))
    if d.world == 1:
        d.init("gloo")
        assert d.max(3.5, "cpu") == 3.5
        d.barrier()
        d.close()


def test_reference_arm_only_runs_on_rank0(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    d = bench.Dist()
    bench.run_reference(type("A", (), {"workload": 1, "steps": 1, "warmup": 0,
                                       "reference_seconds": 1.0})(), d)
    assert capsys.readouterr().out == ""


def test_algorithmic_bytes():
    sys.path.insert(0, ROOT)
    import bench
    from linear_complexity_vision_b200 import synth
    wl = synth.WORKLOADS[5]
    assert bench.algorithmic_bytes(wl)["fused"] == 2 * wl.N * 2 + 5 * wl.C * 4
    wl4 = synth.WORKLOADS[4]
    assert bench.algorithmic_bytes(wl4)["fused"] == 3 * wl4.N * 2 + 2 * wl4.C * 4
    wl2 = synth.WORKLOADS[2]
    ab = bench.algorithmic_bytes(wl2)
    assert ab["qshift"] == 2 * wl2.N * 4 + wl2.C * 4 and ab["fused"] == 3 * wl2.N * 4 + 4 * wl2.C * 4


def test_kernel_source_hash_is_stable():
    sys.path.insert(0, ROOT)
    import bench
    for kern in bench.KERNEL_SOURCES:
        assert bench.kernel_source_hash(kern) == bench.kernel_source_hash(kern)
        assert len(bench.kernel_source_hash(kern)) == 16
    assert bench.kernel_source_hash("biwkv_tma_kernel") != bench.kernel_source_hash("biwkv_bwd_kernel")


def test_issue_roofline_arithmetic():
    import bench
    # 45.7 M warp-instructions in 100 us on 148 SMs at 2000 MHz:
    # 457 G/s of 148 * 4 * 2 = 1184 G/s
    r = bench.issue_roofline(45.7e6, 100e-6, 148, 2000.0)
    assert r["bound"] == "alu"
    assert abs(r["achieved"] - 457.0) < 1e-9
    assert abs(r["peak"] - 1184.0) < 1e-9
    assert abs(r["frac"] - 457.0 / 1184.0) < 1e-12
    assert bench.issue_roofline(None, 100e-6, 148, 2000.0) is None
    assert bench.issue_roofline(45.7e6, 100e-6, 148, None) is None


def test_kernel_hash_ignores_comments_not_code(tmp_path, monkeypatch):
    import shutil
    import bench
    for f in bench.KERNEL_SOURCES["biwkv_tma_kernel"]:
        shutil.copy(os.path.join(bench.CSRC, f), tmp_path / f)
    monkeypatch.setattr(bench, "CSRC", str(tmp_path))
    h0 = bench.kernel_source_hash("biwkv_tma_kernel")
    src = tmp_path / "biwkv_tma.cuh"
    text = src.read_text()
    src.write_text("// a new comment line\n" + text.replace("#pragma once", "#pragma once  // trailing", 1)
                   + "\n/* block\n comment */\n\n")
    assert bench.kernel_source_hash("biwkv_tma_kernel") == h0
    src.write_text(text.replace("constexpr int kL = 8;", "constexpr int kL = 9;", 1))
    assert bench.kernel_source_hash("biwkv_tma_kernel") != h0
