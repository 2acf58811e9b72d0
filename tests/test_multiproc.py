"""The multi-GPU path of the benchmark is replicas only: each rank runs the same
workload, the job time is the maximum over ranks and the job throughput sums the
ranks' bytes over it.  Exercised here with world_size 2 on the gloo backend (CPU)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world)})
    import datetime
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        local_ms = 1.0 + rank * 0.5            # rank 1 is the slow one
        m = bench.max_over_ranks(world, local_ms)
        v = bench.job_throughput(world, 1e9, m)
        q.put((rank, m, v))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_replicas_max_over_ranks_gloo():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, m, v in res:
        assert m == pytest.approx(1.5)
        assert v == pytest.approx(2 * 1e9 / 1.5e-3 / 1e12)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(1, 3.25) == 3.25
    assert bench.job_throughput(1, 2e9, 1.0) == pytest.approx(2.0)
