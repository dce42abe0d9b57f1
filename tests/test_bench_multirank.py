"""The multi-rank side of bench.py on CPU: two gloo ranks.

Under torchrun every rank runs its own replica of the workload (the path
shards by rows with no exchange); the job's time is the slowest rank's and
its throughput is all ranks' work over that time.  The reference arm runs on
rank 0 only and the other ranks exit without work."""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 * (rank + 1)  # rank 1 is the slow one
        worst = bench.max_over_ranks(local_ms, world, "cpu")
        value = bench.job_throughput_tflops(2e12, world, 5, worst)
        q.put((rank, worst, value))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, worst, value in got:
        assert worst == 20.0
        # 2 ranks x 5 steps x 2 TFLOP in 20 ms = 1000 TFLOP/s
        assert abs(value - 1000.0) < 1e-9


def test_single_rank_is_a_no_op_reduction():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5
    assert abs(bench.job_throughput_tflops(1e12, 1, 10, 10.0) - 1000.0) < 1e-9


def test_reference_arm_nonzero_rank_exits_quietly():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_quantile_interpolates_between_order_statistics():
    sys.path.insert(0, ROOT)
    import bench
    v = [5.0, 1.0, 4.0, 2.0, 3.0]
    assert bench.quantile(v, 0.0) == 1.0
    assert bench.quantile(v, 1.0) == 5.0
    assert bench.quantile(v, 0.5) == 3.0
    assert abs(bench.quantile(v, 0.1) - 1.4) < 1e-12
    assert abs(bench.quantile(v, 0.9) - 4.6) < 1e-12
    assert bench.quantile([7.0], 0.9) == 7.0
