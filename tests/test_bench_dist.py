"""The bench's multi-rank plumbing on CPU: two gloo ranks, max-over-ranks timing
and the whole-job rate of independent replicas (the path itself has no exchange)."""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import datetime
    import sys

    import torch.distributed as dist

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    t_local = 1.0 + rank  # rank 1 is the slow one
    t_max = bench.reduce_max(t_local)
    out[rank] = (t_max, bench.whole_job_rate(100.0, world, t_max))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_max_and_rate():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == out[1] == (2.0, 100.0)


def test_single_process_identity():
    import bench

    assert bench.reduce_max(3.5) == 3.5
    assert bench.whole_job_rate(10.0, 1, 2.0) == pytest.approx(5.0)
