"""Multi-rank host logic of bench.py on CPU: two gloo ranks.

Each rank of `bench.py --gpus N` runs independent replicas of the decode
step (weak scaling, no data-path collective); the only collectives are the
ones that turn per-rank timings into the job's figures: the slowest rank's
time and the sum of the bytes every rank processed.  These tests run those
helpers in two processes with per-rank values that differ, so that a max
taken where a sum belongs (or the reverse) fails.
"""
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


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import datetime

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ws, r, local = bench.dist_info()
        bench.barrier()
        out = dict(
            info=(ws, r, local),
            mx=bench.max_over_ranks(1.5 + rank),            # 1.5, 2.5 -> 2.5
            sm=bench.sum_over_ranks(10.0 * (rank + 1)),     # 10, 20 -> 30
            # rank 0: 6e9 bytes in 2 ms, rank 1: 2e9 bytes in 4 ms:
            # (6e9 + 2e9) B / 4 ms = 2 TB/s
            rate=bench.aggregate_rate([6e9, 2e9][rank], [2.0, 4.0][rank]),
        )
        bench.barrier()
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


def test_two_rank_aggregation():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(2):
        rank, out = q.get(timeout=120)
        res[rank] = out
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in (0, 1):
        assert res[rank]["info"] == (2, rank, rank)
        assert res[rank]["mx"] == pytest.approx(2.5)
        assert res[rank]["sm"] == pytest.approx(30.0)
        assert res[rank]["rate"] == pytest.approx(2.0)


def test_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert not dist.is_initialized()
    assert bench.max_over_ranks(3.25) == 3.25
    assert bench.sum_over_ranks(7.0) == 7.0
    assert bench.aggregate_rate(4e9, 2.0) == pytest.approx(2.0)
