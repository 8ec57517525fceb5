"""World-size-2 checks (gloo, CPU) of the benchmark's multi-rank host logic:
every rank decodes its own replica, the job's throughput is all ranks'
tokens over the slowest rank's device time, and only rank 0 reports."""
import os
import socket
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


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from tree_indexed_sparse_02_b200.inputs import DEEP_256K
        ms_local = 10.0 * (rank + 1)                 # rank 1 is the slower one
        value, ms = bench.job_throughput(4.0 * 20, ms_local, world)
        w = bench.replica(DEEP_256K, rank)
        seeds = [None] * world
        dist.all_gather_object(seeds, w.seed)
        out[rank] = (value, ms, tuple(seeds), w.batch, w.context)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_rank_throughput_and_replicas():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    for rank in range(world):
        value, ms, seeds, batch, ctx = out[rank]
        assert ms == 20.0                            # the slowest rank's time
        assert value == pytest.approx(2 * 80 / 0.020)
        assert len(set(seeds)) == world              # independent problems
        assert (batch, ctx) == (4, 262144)           # same shapes everywhere
