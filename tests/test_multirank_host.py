"""Host logic of the N > 1 benchmark run, on CPU: ranks as processes over gloo (world size 2).

The GEMM has no exchange step, so N GPUs run N independent replicas of the workload; the job's time per step
is the slowest rank's, and its throughput counts every rank's work.
"""
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


def _worker(rank, world, port, local_ms, q):
    import datetime

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        ms, value = bench.whole_job_throughput(1e12, local_ms[rank], world)
        bench.barrier(world)
        q.put((rank, ms, value))
    finally:
        dist.destroy_process_group()


def test_whole_job_throughput_takes_the_slowest_rank():
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    world, port = 2, _free_port()
    local_ms = [1.0, 2.5]
    procs = [ctx.Process(target=_worker, args=(r, world, port, local_ms, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms, value in got:
        assert ms == 2.5
        # 2 replicas x 1e12 flop in 2.5 ms = 800 TFLOP/s
        assert value == pytest.approx(2 * 1e12 / 2.5e-3 / 1e12)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    ms, value = bench.whole_job_throughput(3e12, 1.5, 1)
    assert ms == 1.5 and value == pytest.approx(2000.0)


def test_reference_arm_under_torchrun_prints_one_line():
    """`bench.py --impl reference` launched with two ranks: rank 0 alone runs the oracle and prints the line,
    the other rank exits 0 without work."""
    import json

    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2", "--master-addr",
           "127.0.0.1", "--master-port", str(_free_port()), os.path.join(ROOT, "bench.py"), "--impl", "reference",
           "--gpus", "2", "--workload", "1", "--steps", "1", "--warmup", "1"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(l) for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = lines[0]
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
