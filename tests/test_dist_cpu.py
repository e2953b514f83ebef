"""Multi-rank host logic of the benchmark on CPU: two gloo ranks.

The path shards by independent (batch, head) problems, so the only
cross-rank steps are the barrier and the max-over-ranks timing reduction;
both are exercised here, plus the whole-job aggregation.
"""
import datetime
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w, r, l = bench.rank_env()
        dist.barrier()
        t = bench.max_over_ranks(dist, 10.0 + 5.0 * r, "cpu")
        q.put((r, w, l, t))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_env():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert res == [(0, 2, 0, 15.0), (1, 2, 1, 15.0)]


def test_single_process_identity_and_aggregate():
    assert bench.max_over_ranks(None, 3.5, "cpu") == 3.5
    # two ranks, 1e12 flops each, 1 ms per step -> 2000 TFLOPS
    assert bench.aggregate_value(1e12, 2, 1.0) == pytest.approx(2000.0)
