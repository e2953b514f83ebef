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


def test_one_pass_bound_and_alu_roofline():
    w = workloads.get("llm_prefill_causal")
    n = 4 * 32 * 4096 * 128
    # every input read once, every code and scale written once
    assert bench.quant_bytes_one_pass(w) == pytest.approx(2 * n * 2.5625 + n * 3)
    assert bench.quant_bytes_one_pass(w, "nvfp4") == pytest.approx(3 * n * 2.5625)
    v = workloads.get("video_dense_fp8")
    nv = 1 * 40 * 75600 * 128
    assert bench.quant_bytes_one_pass(v) == pytest.approx(3 * nv * 3)
    # the ALU bound: 4*128*128*d flops per block over SOFTMAX_CYCLES_PER_BLOCK cycles on 148 SMs
    r = bench.alu_roofline(w, 1000.0, {"sm_max_mhz": 1965.0})
    expect = 4 * 128 * 128 * 128 * 148 * 1965e6 / bench.SOFTMAX_CYCLES_PER_BLOCK / 1e12
    assert r["bound"] == "alu" and r["peak"] == pytest.approx(expect) and r["frac"] == pytest.approx(1000 / expect)
    d64 = workloads.Workload("t", B=1, H=1, N=128, d=64, causal=False, qk_format="nvfp4", seed=0)
    assert bench.alu_roofline(d64, 1.0, {"sm_max_mhz": 1965.0})["peak"] == pytest.approx(expect / 2)


def test_code_hash_ignores_comments_only():
    src = 'int a = 1; // note\n/* block\n note */ int b = 2;\n\nconst char* s = "// kept";\n'
    reworded = 'int a = 1; // other words\n/* another\n block */ int b = 2;\nconst char* s = "// kept";  \n'
    assert bench.strip_comments(src) == bench.strip_comments(reworded)
    assert bench.strip_comments(src) != bench.strip_comments(src.replace("b = 2", "b = 3"))
    assert '"// kept"' in bench.strip_comments(src)


def test_peak_choice_follows_the_clock_record():
    peaks = {"bf16_tflops": 1655.8, "bf16_tflops_sustained": 1416.8, "hbm_gbs": 6538.3}
    full = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    capped = {"sm_mhz": 1357.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    # mixed NVFP4-QK + FP8-PV: harmonic mean of 4x and 2x the bf16 figure
    peak, burst, bf16, sus, cap = bench.choose_peak(peaks, full, 5.0, "nvfp4", "fp8")
    assert not sus and not cap and bf16 == 1655.8
    assert peak == pytest.approx(2 / (1 / (4 * 1655.8) + 1 / (2 * 1655.8))) == pytest.approx(burst)
    peak, burst, bf16, sus, cap = bench.choose_peak(peaks, capped, 5.0, "fp8", "fp8")
    assert sus and cap and peak == pytest.approx(2 * 1416.8) and burst == pytest.approx(2 * 1655.8)
    # a short region is a burst even when capped
    peak, _, _, sus, _ = bench.choose_peak(peaks, capped, 0.2, "nvfp4", "nvfp4")
    assert not sus and peak == pytest.approx(4 * 1655.8)


def test_clock_sampler_keeps_the_timed_window():
    cs = bench.ClockSampler(0)

    class _P:
        def terminate(self):
            pass

        def wait(self, timeout=None):
            return 0

    cs.proc = _P()
    line = "{sm}, 1965, 700.0, Active, Not Active, Not Active, Not Active, {cap}"
    cs.samples = [(1.0, line.format(sm=1200, cap="Active")), (2.0, line.format(sm=1965, cap="Not Active")),
                  (3.0, line.format(sm=1965, cap="Not Active")), (9.0, line.format(sm=900, cap="Active"))]
    r = cs.stop(1.5, 3.5)
    assert r["samples"] == 2 and r["sm_mhz"] == 1965.0 and r["reasons"] == [] and r["window"] == "timed region"
    r = cs.stop(4.0, 4.01)     # no sample inside: all samples, said so
    assert r["samples"] == 4 and "sw_power_cap" in r["reasons"] and r["window"].startswith("warm-up")


def test_oracle_sample_rows_and_rate():
    w = workloads.get("long_seq_128k_nvfp4")
    rows = bench.sample_rows(w, [0, 1023])
    assert [r[0] for r in rows] == [0, 1023 * 128] and all(8 <= len(r) <= 128 for r in rows)
    small = workloads.get("llm_prefill_causal")
    assert all(len(r) == 128 for r in bench.sample_rows(small, [0, 31]))
    # rate: flops over attention time plus the rows' share of the quantization time
    res = {"flops": 4e9, "attn_s": 1.0, "quant_s": 8.0, "done": [(0, np.arange(64)), (0, np.arange(64))]}
    assert bench.oracle_rate(res, 1024) == pytest.approx(4e9 / (1.0 + 8.0 * 128 / 1024) / 1e12)
