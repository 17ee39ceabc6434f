"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): the job time is
the slowest rank's, throughput aggregates every rank's replica, ranks get
distinct seeds."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        t = bench.max_over_ranks(10.0 + 5.0 * rank)
        results[rank] = (t, bench.rank_seed(rank))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_gloo():
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    results = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, results)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert results[0][0] == 15.0 and results[1][0] == 15.0
    assert results[0][1] != results[1][1]
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.job_throughput(1e9, 2, 1000.0) == pytest.approx(2.0)
    assert bench.max_over_ranks(3.5) == 3.5          # single process: identity
