"""GPU fused attention vs the fp64 oracle.

The oracle quantizes the same seeded inputs itself (its codes equal the GPU's,
which test_quant_gpu pins bit for bit) and runs its tiled online softmax.
Tolerances: max-abs <= 2e-2 * max|V_hat|, relative L2 <= 5e-3, lse within
1e-3 + 1e-5 |lse| (see tests/parity.py). Reduced cases span several tiles and
a ragged tail; full-size workloads are checked on sampled query blocks (first,
last, middle, causal diagonal, STA edge tiles) in the launch configuration the
benchmark uses.
"""

import numpy as np
import pytest
import torch

import precision_attention_nvfp4_b200 as fp
import workloads
from oracle import sta
import parity

pytestmark = pytest.mark.gpu


def _run_gpu(q, k, v, fmt, causal=False, tile_mask=None):
    out, lse = fp.attention(q.cuda(), k.cuda(), v.cuda(), qk_format=fmt, causal=causal, tile_mask=tile_mask)
    torch.cuda.synchronize()
    err = fp.device_error()
    assert err == 0, f"device wait expired: {err:#x}"
    return out.float().cpu().numpy(), lse.cpu().numpy()


def _check_case(q, k, v, fmt, causal=False, key_blocks=None, tile_mask=None, qblocks=None, heads=None,
                min_cos=None, outliers=False):
    B, H, N, d = q.shape
    out, lse = _run_gpu(q, k, v, fmt, causal, tile_mask)
    out = out.reshape(B * H, N, d)
    lse = lse.reshape(B * H, N)
    heads = list(range(B * H)) if heads is None else heads
    qh, kh, vh = parity.oracle_operands(q, k, v, fmt, heads)
    nblk = (N + 127) // 128
    qblocks = list(range(nblk)) if qblocks is None else qblocks
    for i, bh in enumerate(heads):
        rows = np.concatenate([np.arange(b * 128, min(N, b * 128 + 128)) for b in qblocks])
        res = parity.compare_attention(out[bh], lse[bh], qh[i], kh[i], vh[i], rows, causal=causal,
                                       key_blocks=key_blocks)
        parity.assert_close(res, f"{fmt} bh={bh}")
        if min_cos is not None:
            # Cosine against unquantized fp64 attention. With x20 outlier
            # channels the scores are so peaked that quantizing Q/K moves the
            # argmax of many rows, for the oracle as much as for the kernel, so
            # there the kernel must track the oracle's own cosine instead.
            qe, ke, ve = (t.reshape(B * H, N, d)[bh].double().numpy() for t in (q, k, v))
            cos = parity.cosine_vs_exact(out[bh][rows], qe, ke, ve, rows, causal=causal, key_blocks=key_blocks)
            if outliers:
                ref, _ = parity.oatt.attention_rows(qh[i], kh[i], vh[i], rows, causal=causal, key_blocks=key_blocks)
                cos_oracle = parity.cosine_vs_exact(ref, qe, ke, ve, rows, causal=causal, key_blocks=key_blocks)
                assert cos >= cos_oracle - 0.01, f"cosine vs exact {cos} (oracle {cos_oracle})"
            else:
                assert cos >= min_cos, f"cosine vs exact {cos}"


@pytest.mark.parametrize("fmt", ["fp8", "nvfp4"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [128, 300, 1000])
@pytest.mark.parametrize("outliers", [False, True])
def test_reduced(fmt, d, causal, N, outliers):
    w = workloads.Workload("t", B=1, H=2, N=N, d=d, causal=causal, qk_format=fmt, seed=N + d, outliers=outliers)
    q, k, v = workloads.make_qkv(w)
    _check_case(q, k, v, fmt, causal=causal, min_cos=0.99 if fmt == "fp8" else 0.98, outliers=outliers)


def test_tiny_nvfp4_workload():
    w = workloads.get("tiny_nvfp4")
    q, k, v = workloads.make_qkv(w)
    _check_case(q, k, v, "nvfp4", min_cos=0.98)


def test_batch_heads_and_softmax_scale():
    w = workloads.Workload("t", B=3, H=5, N=257, d=128, causal=False, qk_format="fp8", seed=11)
    q, k, v = workloads.make_qkv(w)
    _check_case(q, k, v, "fp8", heads=[0, 7, 14])


def test_identical_keys_give_mean_of_v():
    """Degenerate case: all keys equal -> every P is 1 -> output = mean(V_hat)."""
    g = torch.Generator().manual_seed(12)
    B, H, N, d = 1, 1, 384, 128
    q = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    k = torch.randn(1, 1, 1, d, generator=g).expand(B, H, N, d).contiguous().to(torch.bfloat16)
    v = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    for fmt in ("fp8", "nvfp4"):
        _check_case(q, k, v, fmt)


@pytest.mark.parametrize("fmt", ["fp8", "nvfp4"])
def test_sta_reduced(fmt):
    grid, tile, window = (12, 16, 24), (6, 8, 8), (3, 3, 5)
    N = 12 * 16 * 24
    w = workloads.Workload("t", B=1, H=2, N=N, d=128, causal=False, qk_format=fmt, seed=13)
    q, k, v = workloads.make_qkv(w)
    tg = tuple(a // b for a, b in zip(grid, tile))
    plan = fp.sta_plan(tg, tile, window)
    kb = sta.block_lists(grid, tile, window)
    _check_case(q, k, v, fmt, key_blocks=kb, tile_mask=plan.to("cuda"))


def test_sta_causal_combined():
    grid, tile, window = (12, 16, 16), (6, 8, 8), (3, 3, 3)
    N = 12 * 16 * 16
    w = workloads.Workload("t", B=1, H=1, N=N, d=64, causal=True, qk_format="fp8", seed=14)
    q, k, v = workloads.make_qkv(w)
    tg = tuple(a // b for a, b in zip(grid, tile))
    plan = fp.sta_plan(tg, tile, window)
    kb = sta.block_lists(grid, tile, window)
    _check_case(q, k, v, "fp8", causal=True, key_blocks=kb, tile_mask=plan.to("cuda"))


def test_empty_mask_rows():
    """A user mask with empty rows: those rows get out = 0, lse = -inf."""
    w = workloads.Workload("t", B=1, H=1, N=384, d=128, causal=False, qk_format="fp8", seed=15)
    q, k, v = workloads.make_qkv(w)
    row_ptr = np.array([0, 2, 2, 3], dtype=np.int32)
    col_idx = np.array([0, 2, 1], dtype=np.int32)
    mask = fp.StaPlan(row_ptr, col_idx, np.array([0, 2, 1], dtype=np.int32)).to("cuda")
    out, lse = _run_gpu(q, k, v, "fp8", tile_mask=mask)
    assert np.all(out[0, 0, 128:256] == 0) and np.all(np.isneginf(lse[0, 0, 128:256]))
    kb = [[0, 2], [], [1]]
    qh, kh, vh = parity.oracle_operands(q, k, v, "fp8")
    for blk in (0, 2):
        rows = np.arange(blk * 128, blk * 128 + 128)
        parity.assert_close(parity.compare_attention(out[0, 0], lse[0, 0], qh[0], kh[0], vh[0], rows,
                                                     key_blocks=kb))


# ---------------------------------------------------------------- full size
def _full(name, qblocks_fn, heads_fn, fmt=None, tile_mask=None, key_blocks=None, min_cos=None):
    w = workloads.get(name)
    q, k, v = parity.workload_qkv(name)
    B, H, N, d = q.shape
    nblk = (N + 127) // 128
    _check_case(q, k, v, fmt or w.qk_format, causal=w.causal, key_blocks=key_blocks, tile_mask=tile_mask,
                qblocks=qblocks_fn(nblk), heads=heads_fn(B * H), min_cos=min_cos, outliers=w.outliers)


def test_full_llm_prefill_causal():
    # x20 outlier channels: the cosine against exact attention is held to the
    # oracle's own (within 0.01), not to 0.98
    _full("llm_prefill_causal", lambda n: [0, 1, n // 2, n - 1], lambda bh: [0, bh - 1], min_cos=0.98)


def test_full_video_dense_fp8():
    _full("video_dense_fp8", lambda n: [0, n - 1], lambda bh: [0, bh - 1], min_cos=0.99)


def test_full_video_sta_fp8():
    w = workloads.get("video_sta_fp8")
    tg = tuple(a // b for a, b in zip(w.video, w.sta_tile))
    plan = fp.sta_plan(tg, w.sta_tile, w.sta_window)
    kb = sta.block_lists(w.video, w.sta_tile, w.sta_window)
    # corner tile (fewest neighbours), an interior tile, the last tile
    _full("video_sta_fp8", lambda n: [0, 3 * (1 * 60 + 2 * 10 + 5), n - 1], lambda bh: [bh // 2],
          tile_mask=plan.to("cuda"), key_blocks=kb, min_cos=0.99)


@pytest.mark.parametrize("name", ["long_seq_128k_nvfp4", "long_seq_128k_fp8"])
def test_full_long_sequence_as_benchmarked(name):
    """The benchmark's default workload (B=1, H=32, N=131072, d=128, dense,
    x20 outliers) in the launch configuration bench.py times: inputs drawn
    on the device, Q, K, V through the fused quantizer, one attention launch
    over all 32 heads. Sampled: one head, query blocks first / middle / last,
    each against the oracle on the same inputs (copied to the host)."""
    w = workloads.get(name)
    q, k, v = workloads.make_qkv(w, device="cuda")
    qq, kq, vq = fp.quantize_qkv(q, k, v, w.qk_format)
    out, lse = fp.attention_fwd(qq, kq, vq, causal=w.causal)
    torch.cuda.synchronize()
    assert fp.device_error() == 0
    h = 21
    nblk = w.N // 128
    o = out.reshape(w.B * w.H, w.N, w.d)[h].float().cpu().numpy()
    ls = lse.reshape(w.B * w.H, w.N)[h].cpu().numpy()
    qc, kc, vc = q.cpu(), k.cpu(), v.cpu()
    del q, k, v, qq, kq, vq, out, lse
    qh, kh, vh = parity.oracle_operands(qc, kc, vc, w.qk_format, [h])
    for qb in (0, nblk // 2, nblk - 1):
        rows = np.arange(qb * 128, qb * 128 + 128)
        parity.assert_close(parity.compare_attention(o, ls, qh[0], kh[0], vh[0], rows), f"{name} qb={qb}")


# ----------------------------------------------------- sequence-sweep shapes
# The sweep's configurations differ from one another only in N, d, the mask,
# the QK format and the batch count (B * H * N = 2^22); each head is an
# independent problem, so two heads at the sweep's full N, drawn with the
# sweep's recipe, cover a configuration. Sampled query blocks: first, middle,
# last.
@pytest.mark.parametrize("N,d,causal,fmt", [(16384, 64, True, "fp8"), (16384, 64, False, "nvfp4"),
                                            (131072, 128, False, "nvfp4"), (131072, 128, True, "fp8")])
def test_sweep_shape_sampled(N, d, causal, fmt):
    w = next(x for x in workloads.sweep_workloads() if x.N == N and x.d == d and x.causal == causal
             and x.qk_format == fmt)
    q, k, v = workloads.make_qkv(w, heads=2, batch=1)
    nblk = (N + 127) // 128
    _check_case(q, k, v, fmt, causal=causal, qblocks=[0, nblk // 2, nblk - 1], heads=[0, 1])
