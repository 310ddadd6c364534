"""The multi-process plumbing of bench.py on CPU ranks (gloo, world size 2): every rank gets the
max of the ranks' times, the whole-job value counts every replica, and under torchrun only rank
0 of the reference arm prints its line.  The data path itself has no collective: each rank's
GPU runs an independent replica of the workload."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, ws, port, q):
    import datetime

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(ws)
        ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        got = bench.max_over_ranks(ws, ms)
        q.put((rank, got, bench.weak_value(ws, 1e9, got)))
        bench.barrier(ws)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_value_gloo():
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(120)
    assert all(p.exitcode == 0 for p in ps)
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, got, value in res:
        assert got == 15.0  # every rank sees the slowest rank's time
        assert value == pytest.approx(2 * 1e9 / 15e-3 / 1e9)  # both replicas' bytes over that time


def test_weak_value_single_rank():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(1, 3.5) == 3.5
    assert bench.weak_value(1, 2e9, 1000.0) == pytest.approx(2.0)


def test_reference_arm_under_torchrun_prints_once():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2", "--master-addr",
           "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"), "--impl", "reference",
           "--gpus", "2", "--steps", "2", "--warmup", "0"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["steps"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
