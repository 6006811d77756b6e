"""The bench's multi-process plumbing (one process per GPU; here gloo on CPU,
world size 2): the slowest rank's time reaches every rank, barriers line the
ranks up, and the whole-job value counts the work of every replica."""
import datetime
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(True, cuda=False)
        slowest = bench.max_over_ranks(times[rank], True, device="cpu")
        bench.barrier(True, cuda=False)
        out.put((rank, slowest))
    finally:
        torch.distributed.destroy_process_group()


def test_max_over_ranks_and_barrier_gloo():
    world, times = 2, [0.75, 1.25]
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, times, out)) for r in range(world)]
    for p in procs:
        p.start()
    try:
        got = dict(out.get(timeout=120) for _ in range(world))
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    assert got == {0: 1.25, 1: 1.25}


def test_single_process_needs_no_group():
    assert bench.max_over_ranks(3.5, False) == 3.5


def test_whole_job_value_counts_every_replica():
    # 58 GOP per rank in 0.075 ms on the slowest of 4 ranks
    one = bench.whole_job_tops(58e9, 1, 0.075)
    assert one == pytest.approx(773.33, rel=1e-4)
    assert bench.whole_job_tops(58e9, 4, 0.075) == pytest.approx(4 * one)
