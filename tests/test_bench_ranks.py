"""The multi-rank host logic of bench.py on CPU: two gloo ranks (spawned
processes, rendezvous on 127.0.0.1).  With N ranks the benchmark runs N
independent replicas, takes the slowest rank's time (all_reduce MAX) and
reports the whole job's throughput; the reference arm runs on rank 0 only."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, q):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        ms = bench.max_over_ranks(times[rank], world)
        q.put((rank, ms, bench.job_rate(16384, 10, world, ms)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time_and_sum_the_work():
    world, port = 2, _free_port()
    times = [400.0, 523.5]  # ms of 10 steps on each rank
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, times, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms, rate in got:
        assert ms == max(times)
        # 2 ranks x 10 steps x 16384 tokens over the slowest rank's 523.5 ms
        assert rate == pytest.approx(2 * 10 * 16384 / 0.5235)


def test_single_rank_helpers_need_no_process_group():
    import bench
    assert bench.max_over_ranks(12.5, 1) == 12.5
    assert bench.job_rate(1000, 4, 1, 2000.0) == pytest.approx(2000.0)


def test_reference_arm_runs_on_rank_zero_only():
    import argparse
    import bench
    args = argparse.Namespace(config="c5", steps=1, warmup=1)
    # rank 1 returns at once without touching the oracle
    assert bench.run_reference(args, 1) is None
