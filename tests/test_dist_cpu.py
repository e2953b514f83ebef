"""Multi-rank host logic on CPU: two gloo ranks.

The path shards by independent (batch, head) problems, so the only
cross-rank steps are the barrier and the max-over-ranks timing reduction;
both are exercised here, plus the whole-job aggregation, and the split of one
seeded batch's heads over the ranks (head_range): every rank takes its
contiguous share, and gathering the shares in rank order gives back the
batch, every head once, in order. Splitting one batch needs one exchange for
NVFP4 Q/K, the tensor amax (one float, max-reduced); with it every rank's
share quantizes (oracle, on the CPU) exactly as the whole tensor would.
"""
import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import precision_attention_nvfp4_b200 as fp
import workloads


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


def _split_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w = workloads.Workload("t", B=3, H=5, N=64, d=64, causal=False, qk_format="fp8", seed=21)
        x, _, _ = workloads.make_qkv(w)              # the global batch, drawn identically on each rank
        flat = x.reshape(w.B * w.H, w.N, w.d)
        a, b = fp.head_range(w.B * w.H, world, rank)
        mine = flat[a:b].contiguous()
        # shares differ in size: pad to the largest before the gather
        cap = -(-w.B * w.H // world)
        buf = torch.zeros(cap, w.N, w.d, dtype=x.dtype)
        buf[:b - a] = mine
        ids = torch.full((cap,), -1, dtype=torch.int64)
        ids[:b - a] = torch.arange(a, b)
        bufs = [torch.zeros_like(buf) for _ in range(world)]
        idss = [torch.zeros_like(ids) for _ in range(world)]
        dist.all_gather(bufs, buf)
        dist.all_gather(idss, ids)
        got_ids = torch.cat(idss)
        keep = got_ids >= 0
        got = torch.cat(bufs)[keep]
        q.put((rank, a, b, got_ids[keep].tolist() == list(range(w.B * w.H)), bool(torch.equal(got, flat))))
    finally:
        dist.destroy_process_group()


def test_two_rank_head_split_reassembles_the_batch():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_split_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    # 15 heads over 2 ranks: 8 + 7, contiguous, in rank order
    assert res == [(0, 0, 8, True, True), (1, 8, 15, True, True)]


@pytest.mark.parametrize("n,world", [(15, 2), (32, 8), (3, 4), (0, 3), (128, 7)])
def test_head_range_covers_each_head_once(n, world):
    spans = [fp.head_range(n, world, r) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == n
    assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
    sizes = [b - a for a, b in spans]
    assert max(sizes) - min(sizes) <= 1 and sizes == sorted(sizes, reverse=True)


def _amax_worker(rank, world, port, q):
    import numpy as np
    from oracle import quant as oq
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w = workloads.Workload("t", B=2, H=3, N=64, d=64, causal=False, qk_format="nvfp4", seed=22, outliers=True)
        x, _, _ = workloads.make_qkv(w)
        flat = x.reshape(w.B * w.H, w.N, w.d).float().numpy()
        a, b = fp.head_range(w.B * w.H, world, rank)
        # the one exchange a head-sharded batch needs: the NVFP4 tensor amax,
        # one float per tensor, max-reduced over the ranks
        local = torch.tensor([float(np.abs(flat[a:b]).max()) if b > a else 0.0])
        dist.all_reduce(local, op=dist.ReduceOp.MAX)
        codes, sf, st = oq.quantize_nvfp4(flat[a:b], static_amax=float(local))
        whole_codes, whole_sf, whole_st = oq.quantize_nvfp4(flat)
        q.put((rank, float(local) == float(np.abs(flat).max()), bool(np.array_equal(codes, whole_codes[a:b])),
               bool(np.array_equal(sf, whole_sf[a:b])), float(st) == float(whole_st)))
    finally:
        dist.destroy_process_group()


def test_two_rank_nvfp4_amax_exchange_gives_the_whole_tensor_codes():
    """Sharding one batch's heads over ranks: the max-reduced amax makes every
    rank quantize its share exactly as the whole tensor would be quantized."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_amax_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert res == [(0, True, True, True, True), (1, True, True, True, True)]
