"""The benchmark's multi-process path on the CPU: two gloo ranks, each a
replica of the layer, report the whole-job throughput over the slowest
rank's time; the reference arm runs on rank 0 only."""
import os
import socket
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        elapsed_local = 2.0 if rank == 1 else 1.0          # rank 1 is the slowest
        value, elapsed = bench.job_throughput(1_000_000_000, 10, elapsed_local, world, device="cpu")
        q.put((rank, value, elapsed))
    finally:
        dist.destroy_process_group()


def test_two_replicas_use_the_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, value, elapsed in got:
        assert elapsed == 2.0
        # 2 ranks x 10 steps x 1 GB in 2 s
        assert abs(value - 10.0) < 1e-9


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0
    assert out.stdout.strip() == ""


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.all_max(3.5, 1) == 3.5
    value, elapsed = bench.job_throughput(500_000_000, 4, 0.5, 1, device="cpu")
    assert elapsed == 0.5 and abs(value - 4.0) < 1e-12
