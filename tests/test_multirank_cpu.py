"""Multi-rank host logic of bench.py on CPU: two gloo ranks, one slow.

The layer runs as independent replicas (no collective on the data path); the
bench times every rank on its device and reports the whole job's throughput
against the slowest rank.  Here the ranks are plain processes on 127.0.0.1.
"""
import multiprocessing as mp
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    from datetime import timedelta

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench
    t = bench.max_over_ranks(10.0 + 5.0 * rank)            # rank 1 is the slow one
    v = bench.job_throughput(world, 1e12, 4, t)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, t, v))


def test_two_rank_max_and_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [o[1] for o in out] == [15.0, 15.0]              # both see the slowest rank
    assert out[0][2] == pytest.approx(2 * 1e12 * 4 / 15e-3 / 1e12)


def test_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.job_throughput(1, 2e12, 10, 20.0) == pytest.approx(1000.0)
