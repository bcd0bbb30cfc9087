"""Multi-rank host logic of bench.py on CPU: two gloo ranks (replicas).  Each rank owns an
independent problem (distinct seeds), the job time is the max over ranks, and the job
value counts every rank's tokens."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        r, lr, w = bench.rank_env()
        local_ms = 1.0 + rank                      # rank 1 is the slow one
        job_ms = bench.max_over_ranks(local_ms, w)
        bench.barrier(w)
        seeds = [None] * w
        dist.all_gather_object(seeds, bench.rank_seed(1001, r))
        results[rank] = (r, w, job_ms, seeds)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_independent_problems():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    mp.start_processes(_worker, args=(world, port, results), nprocs=world, join=True,
                       start_method="spawn")
    assert sorted(results.keys()) == [0, 1]
    for rank in range(world):
        r, w, job_ms, seeds = results[rank]
        assert (r, w) == (rank, world)
        assert job_ms == 2.0                       # max over ranks, seen by every rank
        assert len(set(seeds)) == world            # each replica draws its own problem
    # weak scaling: the job value counts all ranks' tokens over the slowest rank's time
    T = 8192
    assert world * T / (2.0 * 1e-3) == pytest.approx(8.192e6)
