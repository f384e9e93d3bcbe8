"""Host logic of the replicated multi-GPU benchmark, run as two gloo ranks on the CPU.

The canvas step has no exchange between sequences, so N GPUs run N independent batch-1 replicas:
each rank draws its own weights, prompt and sampler stream, and the job's rate is the units all
ranks processed over the slowest rank's time.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, q):
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        t = bench.max_over_ranks(times[rank], torch.device("cpu"), world)
        seeds = [None] * world
        dist.all_gather_object(seeds, bench.replica_seed(rank))
        q.put((rank, t, bench.whole_job_rate(world, 24, t), seeds))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_replicas_max_over_ranks_and_rate(world):
    times = [0.30 + 0.05 * r for r in range(world)][::-1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, times, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    t_max = max(times)
    for rank, t, rate, seeds in out:
        assert t == pytest.approx(t_max, rel=0, abs=0)
        assert rate == pytest.approx(world * 24 / t_max)
        assert len(set(seeds)) == world          # every replica has its own stream


def test_single_rank_needs_no_process_group():
    import torch

    import bench
    assert bench.max_over_ranks(0.25, torch.device("cpu"), 1) == 0.25
    assert bench.whole_job_rate(1, 24, 0.25) == 96.0
