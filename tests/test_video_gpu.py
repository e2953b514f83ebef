"""GPU fused video token permutation vs the oracle.

The _video entry points read raster-order (time-major) activations, quantize
them into tile-major codes and write the attention output back in raster
order. The oracle permutes with its own index map
(oracle.sta.raster_index_of_tile_major) and runs the plain quantizers and
attention on the tile-major tensors. Codes and scales must match bit for bit;
the attention output, permuted back, to the tolerances of tests/parity.py.

Layouts cover the three shapes a 32-row chunk of a tile can take in the grid:
part of one w-row (tile (1,4,32)), whole w-rows of one t-slice (tiles
(6,8,8), (6,16,16)), and whole t-slices (tile (8,2,8)).
"""
import numpy as np
import pytest
import torch

import precision_attention_nvfp4_b200 as fp
import workloads
from oracle import codec, quant, sta
import parity

pytestmark = pytest.mark.gpu

LAYOUTS = [
    ((12, 16, 24), (6, 8, 8)),     # chunk = 4 w-rows of 8
    ((6, 32, 32), (6, 16, 16)),    # chunk = 2 w-rows of 16
    ((2, 8, 64), (1, 4, 32)),      # chunk = one w-row of 32
    ((16, 4, 16), (8, 2, 8)),      # chunk = 2 t-slices of 2 x 8
]


def _raster(shape, seed, outliers=True):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(shape, generator=g)
    if outliers:
        x[..., ::shape[-1] // 4] *= 20
    return x.to(torch.bfloat16)


def _perm(grid, tile):
    return torch.from_numpy(sta.raster_index_of_tile_major(grid, tile))


@pytest.mark.parametrize("grid,tile", LAYOUTS)
@pytest.mark.parametrize("d", [64, 128])
def test_quantize_video_codes_bit_exact(grid, tile, d):
    N = grid[0] * grid[1] * grid[2]
    lay = fp.VideoLayout(grid, tile)
    x = _raster((1, 2, N, d), seed=N + d)
    perm = _perm(grid, tile)
    xt = x[:, :, perm].contiguous()
    xf = xt.float().numpy()
    # FP8 per tile and per channel
    for gran in ("tile128", "channel"):
        r = fp.quantize_fp8(x.cuda(), gran, video=lay)
        torch.cuda.synchronize()
        codes, s = quant.quantize_fp8_tile(xf) if gran == "tile128" else quant.quantize_fp8_channel(xf)
        assert np.array_equal(r.scales.cpu().numpy().view(np.uint32), s.view(np.uint32)), gran
        got = r.codes.cpu().numpy()
        assert np.array_equal(got, codes), f"{gran}: {np.count_nonzero(got != codes)} codes differ"
    # NVFP4
    r = fp.quantize_nvfp4(x.cuda(), video=lay)
    torch.cuda.synchronize()
    codes, sb, s_t = quant.quantize_nvfp4(xf)
    assert r.tensor_scale.cpu().numpy().view(np.uint32)[0] == np.float32(s_t).view(np.uint32)
    assert np.array_equal(r.codes.cpu().numpy(), codec.pack_e2m1(codes))
    B, H = x.shape[:2]
    ref_sf = quant.nvfp4_sf_swizzle(sb.reshape(B * H, N, d // 16), N, d).reshape(-1)
    assert np.array_equal(r.block_sf.cpu().numpy(), ref_sf)


def _check_video_attention(q, k, v, grid, tile, fmt, *, window=None, causal=False, heads=None, qblocks=None,
                           tile_major=None):
    """Fused path on raster q, k, v vs the oracle on the tile-major tensors.
    ``tile_major`` may pass the tile-major inputs when they were generated
    separately (the workload generator permutes on its own)."""
    B, H, N, d = q.shape
    lay = fp.VideoLayout(grid, tile)
    mask, kb = None, None
    if window is not None:
        tg = tuple(a // b for a, b in zip(grid, tile))
        mask = fp.sta_plan(tg, tile, window).to("cuda")
        kb = sta.block_lists(grid, tile, window)
    out, lse = fp.attention(q.cuda(), k.cuda(), v.cuda(), qk_format=fmt, causal=causal, tile_mask=mask,
                            video=lay)
    torch.cuda.synchronize()
    assert fp.device_error() == 0
    perm = _perm(grid, tile)
    # raster rows -> tile-major rows
    out_t = out.float().cpu()[:, :, perm].numpy().reshape(B * H, N, d)
    lse_t = lse.cpu()[:, :, perm].numpy().reshape(B * H, N)
    if tile_major is None:
        tile_major = tuple(t[:, :, perm].contiguous() for t in (q, k, v))
    heads = list(range(B * H)) if heads is None else heads
    qh, kh, vh = parity.oracle_operands(*tile_major, fmt, heads)
    nblk = N // 128
    qblocks = list(range(nblk)) if qblocks is None else qblocks
    rows = np.concatenate([np.arange(b * 128, b * 128 + 128) for b in qblocks])
    for i, bh in enumerate(heads):
        res = parity.compare_attention(out_t[bh], lse_t[bh], qh[i], kh[i], vh[i], rows, causal=causal,
                                       key_blocks=kb)
        parity.assert_close(res, f"video {fmt} {grid} {tile} bh={bh}")


@pytest.mark.parametrize("grid,tile", LAYOUTS)
@pytest.mark.parametrize("fmt", ["fp8", "nvfp4"])
def test_video_attention_dense(grid, tile, fmt):
    N = grid[0] * grid[1] * grid[2]
    q, k, v = (_raster((1, 2, N, 128), seed=s) for s in (21, 22, 23))
    _check_video_attention(q, k, v, grid, tile, fmt)


@pytest.mark.parametrize("fmt", ["fp8", "nvfp4"])
def test_video_attention_sta(fmt):
    grid, tile, window = (12, 16, 24), (6, 8, 8), (3, 3, 5)
    N = grid[0] * grid[1] * grid[2]
    q, k, v = (_raster((1, 2, N, 128), seed=s) for s in (31, 32, 33))
    _check_video_attention(q, k, v, grid, tile, fmt, window=window)


def test_video_attention_sta_causal_d64():
    grid, tile, window = (6, 32, 32), (6, 16, 16), (1, 3, 1)
    N = grid[0] * grid[1] * grid[2]
    q, k, v = (_raster((2, 1, N, 64), seed=s, outliers=False) for s in (41, 42, 43))
    _check_video_attention(q, k, v, grid, tile, "fp8", window=window, causal=True)


def test_full_video_sta_fused():
    """The sliding-tile workload at full size, raster in and out, as the
    benchmark runs it: sampled heads and query blocks (corner tile, an
    interior tile, the last tile)."""
    w = workloads.get("video_sta_fp8")
    q, k, v = workloads.make_qkv(w, tile_major=False)
    tm = parity.workload_qkv("video_sta_fp8")  # the generator's own tile-major permutation
    n = w.N // 128
    _check_video_attention(q, k, v, w.video, w.sta_tile, "fp8", window=w.sta_window,
                           heads=[0, w.B * w.H - 1], qblocks=[0, 3 * (1 * 60 + 2 * 10 + 5), n - 1],
                           tile_major=tm)
