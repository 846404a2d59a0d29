"""bench.py's multi-rank host logic on CPU with world_size 2 over gloo.

The block has no exchange step, so N GPUs run N independent replicas: each
rank times its own replica, the job time is the slowest rank's, and the value
counts every rank's FLOPs.  These tests run that logic in two gloo processes.
"""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w, lr = bench.dist_env()
        ms_local = [3.0, 5.0][rank]           # rank 1 is the slow replica
        ms_max = bench.max_over_ranks(ms_local, torch.device("cpu"), w)
        value = bench.replica_throughput(1e12, 10, w, ms_max)
        ref = bench.run_reference(type("A", (), {"workload": "tiny", "steps": 1, "warmup": 0})()) if rank else None
        q.put((r, w, lr, ms_max, value, ref))
    finally:
        dist.destroy_process_group()


def test_two_rank_replicas_take_the_slowest_rank_and_sum_the_work():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, (r, w, lr, ms_max, value, ref) in enumerate(out):
        assert (r, w, lr) == (rank, 2, rank)
        assert ms_max == 5.0                       # both ranks see the slowest rank's time
        assert value == pytest.approx(1e12 * 10 * 2 / 5e-3 / 1e12)
        assert ref is None                         # the reference arm does no work off rank 0


def test_single_process_defaults():
    assert bench.max_over_ranks(2.5, torch.device("cpu"), 1) == 2.5
    assert bench.replica_throughput(2e12, 4, 1, 8.0) == pytest.approx(1000.0)
