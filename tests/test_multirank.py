"""The N > 1 host logic of bench.py on CPU: two gloo ranks reduce their
timings (max) and their work (sum) the way the GPU run does over NCCL, and
the reference arm runs on rank 0 only."""
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


def _rank_main(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        times, work = bench.reduce_over_ranks([10.0 + rank, 5.0 - rank, 1.5], [100.0 * (rank + 1)])
        q.put((rank, times, work))
    finally:
        dist.destroy_process_group()


def test_reduce_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=5) for _ in range(2))
    for rank, times, work in got:
        assert times == [11.0, 5.0, 1.5]          # max over ranks
        assert work == [300.0]                    # sum over ranks


def test_reduce_over_ranks_single_process_is_identity():
    import bench
    assert bench.reduce_over_ranks([3.0, 4.0], [7.0]) == ([3.0, 4.0], [7.0])


def test_reference_arm_runs_on_rank_zero_only():
    import argparse

    import bench
    args = argparse.Namespace(config=0, steps=1, warmup=3, ref_rows=8)
    assert bench.run_reference(args, rank=1) is None
