"""The multi-rank benchmark logic on two gloo ranks (CPU): each rank runs its
own replica of the workload with disjoint clip seeds (weak scaling, no
collective on the data path), the step time is the maximum over ranks and
the throughput counts every rank's audio."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = synth.WORKLOADS["moss_16x30s"]
        seeds = bench.rank_clip_seeds(w, rank)
        gathered = [None] * world
        dist.all_gather_object(gathered, seeds)
        ms = bench.reduce_max(10.0 + 5.0 * rank)            # rank 1 is the slower one
        value = bench.job_throughput(w.batch * w.seconds, world, ms)
        q.put((rank, gathered, ms, value))
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    seeds0, seeds1 = res[0][1]
    assert not set(seeds0) & set(seeds1) and len(seeds0) == 16
    for rank, _, ms, value in res:
        assert ms == 15.0                                   # max over ranks
        assert value == pytest.approx(16 * 30 * 2 / 0.015)  # all ranks' audio / slowest time


def test_single_process_identity():
    assert bench.reduce_max(3.5) == 3.5
    assert bench.job_throughput(480, 1, 15.0) == pytest.approx(32000.0)
