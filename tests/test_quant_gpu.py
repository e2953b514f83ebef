"""GPU quantize kernels vs the oracle: codes and scales bit-exact.

Cases span several 128-token tiles and a ragged tail, d in {64, 128}, the
workload shapes (reduced head counts), outlier channels, all-zero tiles, exact
rounding ties, saturation and denormal-range block scales.
"""
import numpy as np
import pytest
import torch

import precision_attention_nvfp4_b200 as fp
import workloads
from oracle import codec, quant
import parity

pytestmark = pytest.mark.gpu


def _rand(shape, seed, scale=1.0, outliers=False):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(shape, generator=g) * scale
    if outliers:
        x[..., :: max(1, shape[-1] // 4)] *= 20
    return x.to(torch.bfloat16)


def _f32(x):
    return x.float().numpy()


def _ties_fp8(B, H, N, d, seed):
    """Tiles whose amax is 448 (scale exactly 1) filled with E4M3 midpoints."""
    rng = np.random.default_rng(seed)
    grid = codec.e4m3_decode(np.arange(0, 127))
    mids = (grid[1:] + grid[:-1]) / 2
    vals = rng.choice(np.concatenate([mids, grid]), (B, H, N, d)) * rng.choice([-1, 1], (B, H, N, d))
    vals[..., 0, 0] = 448.0
    for t in range(0, N, 128):
        vals[..., t, 0] = 448.0
    return torch.from_numpy(vals.astype(np.float32)).to(torch.bfloat16)


def _ties_nvfp4(B, H, N, d, seed):
    """Tensor amax 2688 (s_t = 1), blocks of E2M1 midpoints times exact scales."""
    rng = np.random.default_rng(seed)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 0.5, 1.0, 6.0, 0.0])
    sb = codec.e4m3_decode(rng.integers(0x08, 0x70, (B, H, N, d // 16)))
    vals = rng.choice(mids, (B, H, N, d)) * rng.choice([-1, 1], (B, H, N, d))
    x = vals * np.repeat(sb, 16, axis=-1)
    x[0, 0, 0, 0] = 2688.0
    return torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)


def _check_nvfp4(x, static_amax=None):
    B, H, N, d = x.shape
    amax_t = None if static_amax is None else torch.tensor([static_amax], dtype=torch.float32, device="cuda")
    r = fp.quantize_nvfp4(x.cuda(), static_amax=amax_t)
    torch.cuda.synchronize()
    codes, sb, s_t = quant.quantize_nvfp4(_f32(x), static_amax=static_amax)
    assert r.tensor_scale.cpu().numpy().view(np.uint32)[0] == np.float32(s_t).view(np.uint32)
    got_codes = r.codes.cpu().numpy()
    ref_codes = codec.pack_e2m1(codes)
    bad = np.argwhere(got_codes != ref_codes)
    assert bad.size == 0, f"{len(bad)} code bytes differ, first {bad[:3]}"
    ref_sf = quant.nvfp4_sf_swizzle(sb.reshape(B * H, N, d // 16), N, d).reshape(-1)
    got_sf = r.block_sf.cpu().numpy()
    assert np.array_equal(got_sf, ref_sf), f"{np.count_nonzero(got_sf != ref_sf)} scale bytes differ"


def _check_fp8(x, granularity):
    r = fp.quantize_fp8(x.cuda(), granularity)
    torch.cuda.synchronize()
    if granularity == "tile128":
        codes, s = quant.quantize_fp8_tile(_f32(x))
    else:
        codes, s = quant.quantize_fp8_channel(_f32(x))
    got_s = r.scales.cpu().numpy()
    assert np.array_equal(got_s.view(np.uint32), s.view(np.uint32)), "scales differ"
    got = r.codes.cpu().numpy()
    assert np.array_equal(got, codes), f"{np.count_nonzero(got != codes)} codes differ"


SHAPES = [(1, 2, 256, 64), (2, 3, 300, 128), (1, 1, 75, 64), (1, 2, 129, 128), (1, 1, 1, 128)]


@pytest.mark.parametrize("shape", SHAPES)
def test_nvfp4_random(shape):
    _check_nvfp4(_rand(shape, 1, outliers=True))


@pytest.mark.parametrize("shape", [(1, 2, 256, 64), (1, 2, 200, 128)])
def test_nvfp4_ties_and_static_amax(shape):
    x = _ties_nvfp4(*shape, seed=2)
    _check_nvfp4(x)
    _check_nvfp4(x, static_amax=2688.0)
    _check_nvfp4(_rand(shape, 3), static_amax=1.5)  # static amax below the data: saturation


def test_nvfp4_zero_and_tiny():
    x = torch.zeros(1, 1, 130, 64, dtype=torch.bfloat16)
    _check_nvfp4(x)
    y = _rand((1, 1, 130, 64), 4)
    y[0, 0, :64] *= 1e-6   # blocks whose E4M3 scale is subnormal or zero
    y[0, 0, 64:70] = 0
    _check_nvfp4(y)


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("gran", ["tile128", "channel"])
def test_fp8_random(shape, gran):
    _check_fp8(_rand(shape, 5, scale=3.0, outliers=True), gran)


@pytest.mark.parametrize("gran", ["tile128", "channel"])
def test_fp8_ties_zero_tiny(gran):
    _check_fp8(_ties_fp8(1, 2, 300, 128, seed=6), gran)
    x = _rand((1, 1, 260, 64), 7)
    x[0, 0, 128:256] = 0          # an all-zero tile / zero rows
    x[0, 0, :128] *= 1e-30        # values reaching E4M3 subnormals after scaling
    _check_fp8(x, gran)


def test_nonfinite_flag():
    x = _rand((1, 1, 256, 64), 8).cuda()
    x[0, 0, 17, 3] = float("inf")
    for run in (lambda f: fp.quantize_fp8(x, "tile128", nonfinite_flag=f),
                lambda f: fp.quantize_fp8(x, "channel", nonfinite_flag=f),
                lambda f: fp.quantize_nvfp4(x, nonfinite_flag=f)):
        flag = torch.zeros(1, dtype=torch.int32, device="cuda")
        run(flag)
        assert int(flag.item()) == 1
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    fp.quantize_fp8(_rand((1, 1, 256, 64), 9).cuda(), "tile128", nonfinite_flag=flag)
    assert int(flag.item()) == 0


@pytest.mark.parametrize("name", ["tiny_nvfp4", "llm_prefill_causal"])
def test_workload_nvfp4_full_tensor(name):
    """Full-size workload tensor on the GPU; every code and scale compared on a
    sample of heads (the tensor scale is over the whole tensor)."""
    w = workloads.get(name)
    q, k, v = parity.workload_qkv(name)
    B, H, N, d = q.shape
    for x in (q, k):
        r = fp.quantize_nvfp4(x.cuda())
        torch.cuda.synchronize()
        xf = _f32(x).reshape(B * H, N, d)
        amax = np.abs(xf).max()
        heads = np.unique(np.array([0, B * H // 2, B * H - 1]))
        codes, sb, s_t = quant.quantize_nvfp4(xf[heads], static_amax=amax)
        assert r.tensor_scale.cpu().numpy().view(np.uint32)[0] == np.float32(s_t).view(np.uint32)
        got = r.codes.cpu().numpy().reshape(B * H, N, d // 2)[heads]
        assert np.array_equal(got, codec.pack_e2m1(codes))
        nb = (N + 127) // 128
        got_sf = r.block_sf.cpu().numpy().reshape(B * H, nb, d // 64, 512)[heads]
        assert np.array_equal(got_sf, quant.nvfp4_sf_swizzle(sb, N, d))


@pytest.mark.parametrize("name", ["video_dense_fp8", "video_sta_fp8"])
def test_workload_fp8_heads(name):
    """Video workload shapes (N = 75600 with an 80-token tail, N = 69120) on a
    subset of heads: per-tile Q/K and per-channel V, bit-exact."""
    w = workloads.get(name)
    q, k, v = parity.workload_qkv(name)
    sub = slice(0, 3)
    _check_fp8(q[:, sub].contiguous(), "tile128")
    _check_fp8(v[:, sub].contiguous(), "channel")


# ---------------------------------------------- Q, K, V in four fused launches
def _same_bits(a: torch.Tensor, b: torch.Tensor, what: str):
    a, b = a.contiguous().view(torch.uint8).cpu(), b.contiguous().view(torch.uint8).cpu()
    n = int((a != b).sum())
    assert a.shape == b.shape and n == 0, f"{what}: {n} bytes differ"


@pytest.mark.parametrize("fmt", ["nvfp4", "fp8"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [128, 300, 1000])
def test_quantize_qkv_equals_separate_calls(fmt, d, N):
    """quantize_qkv (zero, one amax pass over Q, K and V, one conversion pass,
    one finalize) gives bit for bit the codes and scales of the per-tensor
    calls, which the tests above pin to the oracle."""
    q = _rand((2, 3, N, d), 40 + N + d, outliers=True).cuda()
    k = _rand((2, 3, N, d), 41 + N + d, scale=3.0).cuda()
    v = _rand((2, 3, N, d), 42 + N + d, scale=0.5, outliers=True).cuda()
    qq, kq, vq = fp.quantize_qkv(q, k, v, fmt)
    if fmt == "nvfp4":
        for got, ref in ((qq, fp.quantize_nvfp4(q)), (kq, fp.quantize_nvfp4(k))):
            _same_bits(got.codes, ref.codes, "codes")
            _same_bits(got.block_sf, ref.block_sf, "block scales")
            _same_bits(got.tensor_scale, ref.tensor_scale, "tensor scale")
    else:
        for got, ref in ((qq, fp.quantize_fp8(q, "tile128")), (kq, fp.quantize_fp8(k, "tile128"))):
            _same_bits(got.codes, ref.codes, "codes")
            _same_bits(got.scales, ref.scales, "tile scales")
    ref = fp.quantize_fp8(v, "channel")
    _same_bits(vq.codes, ref.codes, "V codes")
    _same_bits(vq.scales, ref.scales, "V channel scales")
    torch.cuda.synchronize()


def test_quantize_qkv_against_oracle_and_video_order():
    """The fused call against the oracle directly (NVFP4 Q, FP8 V), and with a
    raster-order video layout against the separate _video calls."""
    x = _rand((1, 2, 300, 128), 77, outliers=True)
    qq, _, vq = fp.quantize_qkv(x.cuda(), x.cuda(), x.cuda(), "nvfp4")
    torch.cuda.synchronize()
    codes, sb, s_t = quant.quantize_nvfp4(_f32(x))
    assert qq.tensor_scale.cpu().numpy().view(np.uint32)[0] == np.float32(s_t).view(np.uint32)
    assert np.array_equal(qq.codes.cpu().numpy(), codec.pack_e2m1(codes))
    assert np.array_equal(qq.block_sf.cpu().numpy(), quant.nvfp4_sf_swizzle(sb.reshape(2, 300, 8), 300, 128).reshape(-1))
    vc, vs = quant.quantize_fp8_channel(_f32(x))
    assert np.array_equal(vq.codes.cpu().numpy(), vc)
    assert np.array_equal(vq.scales.cpu().numpy().view(np.uint32), vs.view(np.uint32))
    grid, tile = (4, 16, 16), (2, 8, 8)
    video = fp.VideoLayout(grid, tile)
    xs = [_rand((1, 2, 1024, 64), 80 + i, outliers=(i == 0)).cuda() for i in range(3)]
    for fmt in ("nvfp4", "fp8"):
        qq, kq, vq = fp.quantize_qkv(*xs, fmt, video=video)
        if fmt == "nvfp4":
            rq = fp.quantize_nvfp4(xs[0], video=video)
            _same_bits(qq.codes, rq.codes, "video codes")
            _same_bits(qq.block_sf, rq.block_sf, "video scales")
        else:
            rq = fp.quantize_fp8(xs[1], "tile128", video=video)
            _same_bits(kq.codes, rq.codes, "video codes")
            _same_bits(kq.scales, rq.scales, "video tile scales")
        rv = fp.quantize_fp8(xs[2], "channel", video=video)
        _same_bits(vq.codes, rv.codes, "video V codes")
        _same_bits(vq.scales, rv.scales, "video V scales")
