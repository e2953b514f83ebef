"""GPU all-NVFP4 attention (P and V in NVFP4, P V on block-scaled FP4 tensor
cores) vs the oracle.

* The NVFP4 V quantizer (16-token blocks, channel-major, tensor-core scale
  layout with channels as rows) is bit-exact against
  oracle.quant.quantize_nvfp4_tokens, also fused with the video permutation.
* Attention with p_format "nvfp4" in the oracle (P in 16-key NVFP4 blocks with
  the tensor amax fixed at 2^tau) meets the tolerances of tests/parity.py, with
  NVFP4 or FP8 Q/K, causal and dense, d 64 and 128, a ragged tail, the
  threshold rescale, the sliding-tile mask and the full LLM workload.
"""
import numpy as np
import pytest
import torch

import precision_attention_nvfp4_b200 as fp
from oracle import codec, quant, sta
import parity

pytestmark = pytest.mark.gpu


def _rand(shape, seed, outliers=True):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(shape, generator=g)
    if outliers:
        x[..., ::max(1, shape[-1] // 4)] *= 20
    return x.to(torch.bfloat16)


def _check_v(x, video=None, perm=None):
    B, H, N, d = x.shape
    r = fp.quantize_nvfp4_v(x.cuda(), video=video)
    torch.cuda.synchronize()
    xf = (x if perm is None else x[:, :, perm]).float().numpy().reshape(B * H, N, d)
    codes, sb, s_t = quant.quantize_nvfp4_tokens(xf)
    assert r.tensor_scale.cpu().numpy().view(np.uint32)[0] == np.float32(s_t).view(np.uint32)
    got = r.codes.cpu().numpy().reshape(B * H, d, -1)
    ref = codec.pack_e2m1(codes)
    assert np.array_equal(got, ref), f"{np.count_nonzero(got != ref)} code bytes differ"
    Np = codes.shape[-1]
    ref_sf = quant.nvfp4_sf_swizzle(sb, d, Np).reshape(-1)
    got_sf = r.block_sf.cpu().numpy()
    assert np.array_equal(got_sf, ref_sf), f"{np.count_nonzero(got_sf != ref_sf)} scale bytes differ"


@pytest.mark.parametrize("shape", [(1, 2, 300, 128), (2, 1, 256, 64), (1, 1, 129, 128), (1, 3, 1000, 64)])
def test_nvfp4_v_bit_exact(shape):
    _check_v(_rand(shape, seed=sum(shape)))


def test_nvfp4_v_video_order_bit_exact():
    grid, tile = (12, 16, 24), (6, 8, 8)
    x = _rand((1, 2, 12 * 16 * 24, 128), seed=7)
    perm = torch.from_numpy(sta.raster_index_of_tile_major(grid, tile))
    _check_v(x, video=fp.VideoLayout(grid, tile), perm=perm)


def _check(q, k, v, fmt, *, causal=False, tau=0.0, heads=None, qblocks=None, tile_mask=None, key_blocks=None):
    B, H, N, d = q.shape
    out, lse = fp.attention(q.cuda(), k.cuda(), v.cuda(), qk_format=fmt, causal=causal, tile_mask=tile_mask,
                            rescale_threshold=tau, pv_format="nvfp4")
    torch.cuda.synchronize()
    assert fp.device_error() == 0
    out = out.float().cpu().numpy().reshape(B * H, N, d)
    lse = lse.cpu().numpy().reshape(B * H, N)
    heads = list(range(B * H)) if heads is None else heads
    qh, kh, vh = parity.oracle_operands(q, k, v, fmt, heads, pv_format="nvfp4")
    nblk = (N + 127) // 128
    qblocks = list(range(nblk)) if qblocks is None else qblocks
    rows = np.concatenate([np.arange(b * 128, min(N, b * 128 + 128)) for b in qblocks])
    for i, bh in enumerate(heads):
        res = parity.compare_attention(out[bh], lse[bh], qh[i], kh[i], vh[i], rows, causal=causal,
                                       key_blocks=key_blocks, rescale_threshold=tau, p_format="nvfp4")
        parity.assert_close(res, f"pv nvfp4 {fmt} bh={bh}")


@pytest.mark.parametrize("fmt", ["nvfp4", "fp8"])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,d", [(300, 64), (1000, 128), (128, 128)])
def test_all_nvfp4_reduced(fmt, causal, N, d):
    q, k, v = (_rand((1, 2, N, d), seed=N + d + s) for s in range(3))
    _check(q, k, v, fmt, causal=causal)


def test_all_nvfp4_threshold_and_batch():
    q, k, v = (_rand((2, 3, 700, 128), seed=40 + s, outliers=False) for s in range(3))
    _check(q, k, v, "nvfp4", causal=True, tau=8.0, heads=[0, 5])


def test_all_nvfp4_sta():
    grid, tile, window = (12, 16, 24), (6, 8, 8), (3, 3, 5)
    N = 12 * 16 * 24
    q, k, v = (_rand((1, 2, N, 128), seed=50 + s) for s in range(3))
    tg = tuple(a // b for a, b in zip(grid, tile))
    _check(q, k, v, "fp8", tile_mask=fp.sta_plan(tg, tile, window).to("cuda"),
           key_blocks=sta.block_lists(grid, tile, window))


def test_all_nvfp4_full_llm_prefill_sampled():
    q, k, v = parity.workload_qkv("llm_prefill_causal")
    B, H, N, d = q.shape
    _check(q, k, v, "nvfp4", causal=True, heads=[0, B * H - 1], qblocks=[0, 1, N // 256, N // 128 - 1])
