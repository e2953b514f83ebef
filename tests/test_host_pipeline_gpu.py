"""attention() on host (pinned) inputs: the chunked pipeline that overlaps
the copies with the kernels returns the same bits as the call on device
inputs, for every format pair, for the default and for uneven groups of
heads, with the sliding-tile mask on a raster-order video, and with the
tensor-amax pass run piece by piece (the NVFP4 tensor scale of the whole
tensor)."""
import numpy as np
import pytest
import torch

import precision_attention_nvfp4_b200 as fp
import workloads

pytestmark = pytest.mark.gpu


def _pinned(*ts):
    return [t.contiguous().pin_memory() for t in ts]


@pytest.mark.parametrize("qk,pv", [("nvfp4", "fp8"), ("fp8", "fp8"), ("nvfp4", "nvfp4"), ("fp8", "nvfp4")])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("chunks", [None, 4])
def test_host_pipeline_equals_device_call(qk, pv, causal, chunks):
    w = workloads.Workload("t", B=1, H=5, N=700, d=128, causal=causal, qk_format=qk, seed=31, outliers=True)
    q, k, v = workloads.make_qkv(w)
    ref_out, ref_lse = fp.attention(q.cuda(), k.cuda(), v.cuda(), qk_format=qk, causal=causal, pv_format=pv)
    torch.cuda.synchronize()
    qh, kh, vh = _pinned(q, k, v)
    out, lse = fp.attention(qh, kh, vh, qk_format=qk, causal=causal, pv_format=pv, host_chunks=chunks)
    assert not out.is_cuda and out.is_pinned()
    assert torch.equal(out.view(torch.int16), ref_out.cpu().view(torch.int16))
    assert torch.equal(lse.view(torch.int32), ref_lse.cpu().view(torch.int32))
    assert fp.device_error() == 0


def test_host_pipeline_video_sta_and_reused_buffers():
    grid, tile, window = (12, 16, 24), (6, 8, 8), (3, 3, 5)
    w = workloads.Workload("t", B=1, H=3, N=12 * 16 * 24, d=64, causal=False, qk_format="fp8", seed=32)
    q, k, v = workloads.make_qkv(w)
    video = fp.VideoLayout(grid, tile)
    mask = fp.sta_plan(tuple(a // b for a, b in zip(grid, tile)), tile, window).to("cuda")
    ref_out, ref_lse = fp.attention(q.cuda(), k.cuda(), v.cuda(), qk_format="fp8", tile_mask=mask, video=video)
    torch.cuda.synchronize()
    qh, kh, vh = _pinned(q, k, v)
    out_h = torch.empty(q.shape, dtype=torch.bfloat16, pin_memory=True)
    lse_h = torch.empty(q.shape[:3], dtype=torch.float32, pin_memory=True)
    for _ in range(2):
        out, lse = fp.attention(qh, kh, vh, qk_format="fp8", tile_mask=mask, video=video, out_host=out_h,
                                lse_host=lse_h, host_chunks=3)
        assert out.data_ptr() == out_h.data_ptr()
        assert torch.equal(out.view(torch.int16), ref_out.cpu().view(torch.int16))
        assert torch.equal(lse.view(torch.int32), ref_lse.cpu().view(torch.int32))


def test_tensor_amax_in_pieces_equals_whole():
    """Accumulating the amax over pieces of a tensor gives the whole-tensor
    amax, and NVFP4 quantization with it as the static amax reproduces the
    dynamic call bit for bit."""
    g = torch.Generator().manual_seed(33)
    x = (torch.randn(2, 3, 260, 64, generator=g) * 3).to(torch.bfloat16).cuda()
    x[1, 2, 5, 7] = -97.0
    flat = x.reshape(6, 260, 64)
    acc = torch.empty(1, dtype=torch.float32, device="cuda")
    for i, (a, b) in enumerate([(0, 2), (2, 3), (3, 6)]):
        fp.tensor_amax(flat[a:b].view(1, b - a, 260, 64), acc, accumulate=i > 0)
    assert float(acc) == float(x.float().abs().max()) == 97.0
    whole = fp.quantize_nvfp4(x)
    parts = fp.quantize_nvfp4(x, static_amax=acc)
    for f in ("codes", "block_sf", "tensor_scale"):
        assert torch.equal(getattr(whole, f).view(torch.uint8), getattr(parts, f).view(torch.uint8)), f
    np.testing.assert_equal(fp.tensor_amax(x).item(), 97.0)


@pytest.mark.parametrize("scale", [1.0, 2.0])
def test_host_pipeline_with_caller_amax(scale):
    """A caller's Q/K amax (the static form of the NVFP4 recipe): the host
    pipeline quantizes each group as it lands and returns the bits of the
    device call with the same amax; with the true amax, those of the dynamic
    call."""
    w = workloads.Workload("t", B=2, H=3, N=520, d=128, causal=True, qk_format="nvfp4", seed=34, outliers=True)
    q, k, v = workloads.make_qkv(w)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    amax = (fp.tensor_amax(qc) * scale, fp.tensor_amax(kc) * scale)
    ref_out, ref_lse = fp.attention(qc, kc, vc, causal=True, qk_amax=amax)
    if scale == 1.0:
        dyn_out, _ = fp.attention(qc, kc, vc, causal=True)
        assert torch.equal(dyn_out.view(torch.int16), ref_out.view(torch.int16))
    torch.cuda.synchronize()
    qh, kh, vh = _pinned(q, k, v)
    out, lse = fp.attention(qh, kh, vh, causal=True, qk_amax=amax, host_chunks=4)
    assert torch.equal(out.view(torch.int16), ref_out.cpu().view(torch.int16))
    assert torch.equal(lse.view(torch.int32), ref_lse.cpu().view(torch.int32))
    assert fp.device_error() == 0
