"""Multi-rank host logic of bench.py on CPU: two gloo ranks.

With N GPUs the benchmark runs one independent replica per rank (the path has
no exchange step); the only collectives are control-plane: the elapsed time is
the max over ranks and the throughput counts every rank's units.
"""
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
        ms = [12.5, 30.25][rank]
        ms_max = bench.max_over_ranks(ms, world, torch.device("cpu"))
        value = bench.aggregate_throughput(65536, world, 4, ms_max)
        q.put((rank, ms_max, value))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_max_over_ranks_and_aggregate_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(world))
    for rank, ms_max, value in res:
        assert ms_max == 30.25                       # slowest rank decides the time
        assert value == pytest.approx(65536 * 2 * 4 / 0.03025)   # all ranks' tokens


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.0, 1, torch.device("cpu")) == 7.0
    assert bench.aggregate_throughput(100, 1, 2, 1000.0) == pytest.approx(200.0)


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True,
                       timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
