"""Input generator and benchmark bookkeeping (CPU only).

* The generator's tile-major permutation (workloads.video_tile_major_perm,
  which arranges the sliding-tile workload's inputs) equals the oracle's own
  index (oracle.sta.raster_index_of_tile_major), so inputs and parity checks
  agree on the token order.
* make_qkv is deterministic, and its raster and tile-major outputs of the
  sliding-tile workload are the same tokens, permuted.
* The benchmark's algorithmic quantize bytes and aggregate throughput follow
  the per-element counts of the scope table.
"""
import numpy as np
import pytest
import torch

import bench
import workloads
from oracle import sta


@pytest.mark.parametrize("grid,tile", [((18, 48, 80), (6, 8, 8)), ((12, 16, 24), (6, 8, 8)),
                                       ((8, 16, 24), (4, 8, 8)), ((6, 32, 48), (6, 16, 16))])
def test_generator_permutation_equals_oracle_index(grid, tile):
    perm = workloads.video_tile_major_perm(grid, tile).numpy()
    assert np.array_equal(perm, sta.raster_index_of_tile_major(grid, tile))


def test_make_qkv_deterministic_and_shaped():
    w = workloads.get("llm_prefill_causal")
    a = workloads.make_qkv(w, heads=2, batch=1, N=300)
    b = workloads.make_qkv(w, heads=2, batch=1, N=300)
    for x, y in zip(a, b):
        assert x.shape == (1, 2, 300, 128) and x.dtype == torch.bfloat16
        assert torch.equal(x, y)


def test_sta_workload_raster_and_tile_major_are_the_same_tokens():
    w = workloads.get("video_sta_fp8")
    tm = workloads.make_qkv(w, heads=1)
    ra = workloads.make_qkv(w, heads=1, tile_major=False)
    perm = torch.from_numpy(sta.raster_index_of_tile_major(w.video, w.sta_tile))
    for x, y in zip(tm, ra):
        assert x.shape == (1, 1, w.N, w.d)
        assert torch.equal(x, y[:, :, perm])


def test_quant_bytes_and_aggregate():
    w = workloads.get("llm_prefill_causal")
    n = 4 * 32 * 4096 * 128
    # NVFP4 Q and K: amax read 2 + quantize read 2 + codes 0.5 + scales 1/16; FP8 V: 2 + 2 + 1
    assert bench.quant_bytes(w) == pytest.approx(2 * n * 4.5625 + n * 5)
    assert bench.quant_bytes(w, "nvfp4") == pytest.approx(2 * n * 4.5625 + n * 4.5625)
    v = workloads.get("video_dense_fp8")
    nv = 1 * 40 * 75600 * 128
    assert bench.quant_bytes(v) == pytest.approx(2 * nv * 3 + nv * 5)
    # weak scaling: every rank does the per-rank flops in the (max over ranks) step time
    assert bench.aggregate_value(1e12, 4, 2.0) == pytest.approx(4 * 1e12 / 2e-3 / 1e12)
