"""GPU denoising-step-aware configurations vs the oracle.

The FPSAttention page (section 3.2) switches the Q/K quantization granularity
and the sliding-tile window by denoising phase. Here:

* grouped FP8 scales (one scale per group of 128-token tiles) are bit-exact
  against oracle.quant.quantize_fp8_group, in kernel order and fused with the
  video token permutation;
* attention on grouped scales meets the tolerances of tests/parity.py;
* one reduced video run per phase of a 50-step schedule, with the phase from
  the library's fpattn_step_phase: early = one scale per head with a sparse
  window, middle = per-tile scales and dense attention, late = one scale per
  video tile with a medium window; also the tile variants (4,8,8) and
  (6,16,16) the page reports for fast-motion and static scenes.
"""
import numpy as np
import pytest
import torch

import precision_attention_nvfp4_b200 as fp
from oracle import quant, sta
import parity

pytestmark = pytest.mark.gpu


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(shape, generator=g)
    x[..., ::max(1, shape[-1] // 4)] *= 20
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("shape,group", [((1, 2, 600, 64), 2), ((1, 2, 600, 64), 3), ((1, 2, 600, 64), 7),
                                         ((2, 1, 1000, 128), 8), ((2, 1, 1000, 128), 100),
                                         ((1, 1, 129, 128), 2)])
def test_group_scales_bit_exact(shape, group):
    x = _rand(shape, seed=sum(shape) + group)
    r = fp.quantize_fp8(x.cuda(), "group", group_tiles=group)
    torch.cuda.synchronize()
    codes, s = quant.quantize_fp8_group(x.float().numpy(), group)
    assert np.array_equal(r.scales.cpu().numpy().view(np.uint32), s.view(np.uint32))
    got = r.codes.cpu().numpy()
    assert np.array_equal(got, codes), f"{np.count_nonzero(got != codes)} codes differ"


def test_group_scales_video_order_bit_exact():
    grid, tile = (12, 16, 24), (6, 8, 8)
    N = 12 * 16 * 24
    x = _rand((1, 2, N, 128), seed=3)
    perm = torch.from_numpy(sta.raster_index_of_tile_major(grid, tile))
    r = fp.quantize_fp8(x.cuda(), "group", group_tiles=3, video=fp.VideoLayout(grid, tile))
    torch.cuda.synchronize()
    codes, s = quant.quantize_fp8_group(x[:, :, perm].float().numpy(), 3)
    assert np.array_equal(r.scales.cpu().numpy().view(np.uint32), s.view(np.uint32))
    assert np.array_equal(r.codes.cpu().numpy(), codes)


def _oracle_grouped(q, k, v, group, heads):
    B, H, N, d = q.shape
    idx = torch.tensor(heads)
    qf, kf, vf = (t.reshape(B * H, N, d)[idx].float().numpy() for t in (q, k, v))
    cq, sq = quant.quantize_fp8_group(qf, group)
    ck, sk = quant.quantize_fp8_group(kf, group)
    cv, sv = quant.quantize_fp8_channel(vf)
    return (quant.dequantize_fp8_tile(cq, sq), quant.dequantize_fp8_tile(ck, sk),
            quant.dequantize_fp8_channel(cv, sv))


def _check(q, k, v, group, *, causal=False, grid=None, tile=None, window=None):
    """Fused attention with group-scaled FP8 Q/K; video inputs (grid given)
    are raster order and compared after the oracle's permutation."""
    B, H, N, d = q.shape
    video = mask = kb = None
    if grid is not None:
        video = fp.VideoLayout(grid, tile)
        if window is not None:
            tg = tuple(a // b for a, b in zip(grid, tile))
            mask = fp.sta_plan(tg, tile, window).to("cuda")
            kb = sta.block_lists(grid, tile, window)
    out, lse = fp.attention(q.cuda(), k.cuda(), v.cuda(), qk_format="fp8", causal=causal, tile_mask=mask,
                            video=video, qk_group_tiles=group)
    torch.cuda.synchronize()
    assert fp.device_error() == 0
    out, lse = out.float().cpu(), lse.cpu()
    if grid is not None:
        perm = torch.from_numpy(sta.raster_index_of_tile_major(grid, tile))
        q, k, v, out, lse = (t[:, :, perm].contiguous() for t in (q, k, v, out, lse))
    out = out.numpy().reshape(B * H, N, d)
    lse = lse.numpy().reshape(B * H, N)
    heads = list(range(B * H))
    qh, kh, vh = _oracle_grouped(q, k, v, group, heads)
    rows = np.arange(N)
    for i, bh in enumerate(heads):
        res = parity.compare_attention(out[bh], lse[bh], qh[i], kh[i], vh[i], rows, causal=causal,
                                       key_blocks=kb)
        parity.assert_close(res, f"group={group} bh={bh}")


@pytest.mark.parametrize("group", [3, 8])
@pytest.mark.parametrize("causal", [False, True])
def test_attention_group_scales(group, causal):
    q, k, v = (_rand((1, 2, 1000, 128), seed=s) for s in (11, 12, 13))
    _check(q, k, v, group, causal=causal)


SCHEDULE = {  # phase -> (Q/K scale group in tiles: None = one per head, window in tiles or None = dense)
    0: (None, (1, 3, 3)),   # early: coarse granularity, sparse window
    1: (1, None),           # middle: fine granularity, dense
    2: (3, (3, 3, 5)),      # late: one scale per (6,8,8) video tile, medium window
}


@pytest.mark.parametrize("t", [1, 10, 11, 35, 36, 50])
def test_schedule_phase_configs(t):
    grid, tile = (12, 16, 24), (6, 8, 8)
    N = 12 * 16 * 24
    phase = fp.step_phase(t, 50)
    assert phase == (0 if t <= 10 else 1 if t <= 35 else 2)
    group, window = SCHEDULE[phase]
    group = N // 128 if group is None else group
    q, k, v = (_rand((1, 1, N, 128), seed=100 + t + s) for s in range(3))
    _check(q, k, v, group, grid=grid, tile=tile, window=window)


@pytest.mark.parametrize("grid,tile,window", [((8, 16, 24), (4, 8, 8), (3, 3, 3)),
                                              ((6, 32, 48), (6, 16, 16), (1, 3, 3))])
def test_tile_variants_fused(grid, tile, window):
    N = grid[0] * grid[1] * grid[2]
    q, k, v = (_rand((1, 1, N, 128), seed=200 + s) for s in range(3))
    per_tile = tile[0] * tile[1] * tile[2] // 128
    _check(q, k, v, per_tile, grid=grid, tile=tile, window=window)
