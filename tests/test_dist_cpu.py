"""Multi-rank plumbing of bench.py on CPU (gloo, world size 2).

The indexer shards by independent rows and sequences, so each of N GPUs
indexes its own batch with no data-path collective; what needs testing is
the plumbing: every rank joins the same collectives, the slowest rank's time
is the job's time, the whole-job rate counts every rank's units, the ranks'
batches differ, and only rank 0 of the reference arm does any work."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime

    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench._barrier(dist)
        local_ms = 10.0 + 5.0 * rank          # rank 1 is the slow one
        slowest = bench._max_over_ranks(dist, local_ms, device="cpu")
        rate = bench.whole_job_rate(1000, world, 4, slowest)
        # reference arm: ranks other than 0 return at once, before any work
        ref = None
        if rank != 0:
            class A:
                config = "no-such-workload"   # would raise if rank 1 tried to build it
                T = None
                steps = 1
                warmup = 3
            ref = bench.run_reference(A())
        # each rank's own batch: a checksum of its queries, gathered
        bench.SHARD = rank
        wl = bench.Dense("cpu", size=64)
        mine = torch.tensor([float(wl.inp.q.float().sum())], dtype=torch.float64)
        sums = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(sums, mine)
        bench._barrier(dist)
        out.put((rank, slowest, rate, ref, [float(x) for x in sums]))
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_and_whole_job_rate():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    try:
        for _ in range(world):
            r, slowest, rate, ref, sums = q.get(timeout=120)
            res[r] = (slowest, rate, ref, sums)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    for r in range(world):
        slowest, rate, ref, sums = res[r]
        assert slowest == pytest.approx(15.0)                  # max over ranks, seen by every rank
        assert rate == pytest.approx(1000 * 2 * 4 / 0.015)     # all ranks' units / slowest time
        assert ref is None
        assert sums[0] != sums[1]                              # two ranks, two different batches
