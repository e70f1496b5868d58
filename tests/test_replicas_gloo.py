"""The multi-rank form of the benchmark: one independent replica per rank, no collective on
the data path; the only cross-rank steps are barriers and one MAX all-reduce of the device
times.  Two `gloo` ranks on the CPU check that reduction, the whole-job rate built on it and
that the reference arm works on rank 0 alone."""
import argparse
import datetime
import os
import socket
import sys

import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        # device times of this rank (ms): rank 1 is slower in the first, rank 0 in the second
        mine = [10.0 + rank, 5.0 - rank, 7.5]
        got = bench.max_over_ranks(mine, torch.device("cpu"), world)
        rate = bench.job_rate(1000, 4, world, got[0])
        # the reference arm: every rank but 0 returns at once, without work
        ref = bench.run_reference(argparse.Namespace(warmup=0, steps=0), rank, world) if rank else None
        torch.distributed.barrier()
        out.put((rank, got, rate, ref))
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks_reduce_to_the_slowest_rank():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    try:
        for _ in range(world):
            rank, got, rate, ref = out.get(timeout=120)
            res[rank] = (got, rate, ref)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    for rank in range(world):
        got, rate, ref = res[rank]
        assert got == [11.0, 5.0, 7.5]               # elementwise max over the two ranks
        assert rate == 1000 * 4 * world / (11.0 / 1e3)  # all ranks' units over the slowest time
    assert res[1][2] is None


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks([3.0, 4.0], torch.device("cpu"), 1) == [3.0, 4.0]
    assert bench.job_rate(128, 5, 1, 250.0) == 128 * 5 / 0.25
