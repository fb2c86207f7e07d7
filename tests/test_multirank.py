"""Multi-rank host logic of bench.py on CPU: two gloo ranks, as the torchrun
replicas of `bench.py --gpus 2` would run (the path needs no data exchange;
only the device time is reduced with a max over ranks)."""
from __future__ import annotations

import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # Each rank "measured" a different device time; everyone must agree on the max.
        mine = 10.0 + 5.0 * rank
        got = bench.max_over_ranks(mine, world)
        bench.barrier(world)
        value = bench.whole_job_tflops(world, 1e12, 4, got)
        q.put((rank, got, value))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_time_and_whole_job_value():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, got, value in res:
        assert got == 15.0
        # 2 ranks x 1e12 FLOP x 4 steps / 15 ms
        assert abs(value - 2 * 1e12 * 4 / 15e-3 / 1e12) < 1e-9


def test_whole_job_value_single_rank():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert abs(bench.whole_job_tflops(1, 2e12, 10, 20.0) - 1000.0) < 1e-9


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""
