"""The benchmark's multi-rank host logic on CPU, with gloo ranks (world size 2).

The library itself has nothing to exchange between GPUs (every head is
independent), so `bench.py --gpus N` runs N replicas; what needs covering is
the host side: the maximum of the per-rank step times, the whole-job rate
computed from it, and the reference arm printing on rank 0 only.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench as b
    dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%d" % port, rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ms = b.max_over_ranks(dist, times[rank], "cpu")
        dist.barrier()
        out.put((rank, ms, b.job_tflops(world, 1e12, ms)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_rate_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    times = [3.0, 5.0]  # ms per step on rank 0 and rank 1
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, times, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # both ranks see the slowest rank's time, and the job rate counts both ranks' work
    assert [g[1] for g in got] == [5.0, 5.0]
    assert all(abs(g[2] - 2 * 1e12 / 5e-3 / 1e12) < 1e-9 for g in got)


def test_single_process_helpers():
    assert bench.max_over_ranks(None, 4.25, "cpu") == 4.25
    assert abs(bench.job_tflops(1, 2e12, 2.0) - 1000.0) < 1e-9


def test_reference_arm_under_torchrun_prints_once_on_rank_zero():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0", "--ref-seconds", "1"]
    env = dict(os.environ, OMP_NUM_THREADS=os.environ.get("OMP_NUM_THREADS", "4"))
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
