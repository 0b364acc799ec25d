"""Multi-process (gloo, world size 2, CPU) checks of the N > 1 host logic of
bench.py: per-rank batches, the max-over-ranks timing reduction, the whole-job
throughput, and the reference arm running on rank 0 only.
"""
from __future__ import annotations

import datetime
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

from tests.conftest import ROOT


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, q):
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        sys.path.insert(0, ROOT)
        import bench
        from mxfp4_block_fake_b200 import workloads as W

        ms = bench.reduce_max([10.0 + rank, 3.0 * (rank + 1)], world, "cpu")
        x, counts, _ = W.moe_grouped(64, 32, 8, seed=bench.rank_seed(4, rank))
        q.put((rank, ms, float(x.float().sum()), counts.tolist()))
    finally:
        dist.destroy_process_group()


def test_two_rank_reduction_and_distinct_batches():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    ps = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in ps:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort()
    # every rank sees the max over ranks
    assert out[0][1] == out[1][1] == [11.0, 6.0]
    # ranks quantise different batches (weak scaling) with the same group recipe
    assert out[0][2] != out[1][2]
    assert sum(out[0][3]) == sum(out[1][3]) == 64


def test_weak_value():
    sys.path.insert(0, ROOT)
    import bench

    # 2 ranks x 10 steps x 1e9 bytes over 4 ms -> 5000 GB/s
    assert bench.weak_value(10 ** 9, 10, 2, 4.0) == pytest.approx(5000.0)
    b = bench.step_bytes(65536, 7168, 2172)
    assert b["step"] == b["fwd"] + b["bwd"]
    n = 65536 * 7168
    assert b["fwd"] == n * 2 + 2 * n * 2 + 2 * (n // 2) + 65536 * 224 + 2172 * 7168 + 2 * 65536 * 896


def test_reference_arm_under_torchrun_prints_once():
    """The oracle arm runs on rank 0 alone; the other rank exits 0 without work."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "0", "--rows", "2048", "--cols", "512", "--groups", "16"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["unit"] == "GB/s" and j["value"] > 0
    assert j["e2e"]["h2d_bytes_per_step"] == 0 and j["cpu_baseline"]["kind"] == "oracle"


def test_all_cores_cpu_baseline_matches_single_process_work():
    """The all-cores oracle baseline (spawned processes over whole groups)
    covers every row and group exactly once: the chunk boundaries fall on
    group ends and the bytes are those of one full step."""
    sys.path.insert(0, ROOT)
    import bench
    from mxfp4_block_fake_b200 import workloads as W

    class A:
        rows, cols, groups, scale_mode = 1024, 256, 12, "page"

    x_h, _, offsets = W.moe_grouped(A.rows, A.cols, A.groups, seed=4)
    g_h = W.train_step_grad(A.rows, A.cols, seed=5)
    r = bench.cpu_baseline_all_cores(A, x_h, g_h, offsets, max_procs=3)
    assert 1 <= r["cores"] <= 3
    assert r["value"] > 0 and r["seconds"] > 0
