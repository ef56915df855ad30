"""World-size-2 checks of bench.py's multi-rank logic on CPU (gloo): each rank
runs an independent replica of the workload (weak scaling, no collective on
the data path), the job's time is the max over ranks, and throughput counts
every rank's tokens."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 + 5.0 * rank
        m = bench.max_over_ranks(local_ms, dist)
        w = bench.rank_workload(1, rank, chunk=16)
        digest = float(np.asarray(w.q, np.float64).sum())
        sums = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(sums, torch.tensor([digest], dtype=torch.float64))
        out[rank] = (m, [float(x) for x in sums], w.q.shape)
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_distinct_replicas():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    for r in range(world):
        m, sums, shape = out[r]
        assert m == 15.0                         # slowest rank decides the job time
        assert sums[0] != sums[1]                # independent inputs per rank
        assert shape == out[0][2]                # same workload shape on every rank
    assert bench.job_throughput(256, 2, 15.0) == 256 * 2 / 0.015


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.5, None) == 3.5
    assert bench.rank_workload(2, 0).seed != bench.rank_workload(2, 1).seed
