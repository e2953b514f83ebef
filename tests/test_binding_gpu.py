"""The Python binding refuses, before any launch, buffers the kernels would
read or write out of place: outputs, amax and flag words and tile-mask
arrays that are on the host, on another dtype, too small or not contiguous."""
import pytest
import torch

import precision_attention_nvfp4_b200 as fp

pytestmark = pytest.mark.gpu


def _qkv(N=256, d=128):
    g = torch.Generator(device="cuda").manual_seed(41)
    return [torch.randn(1, 2, N, d, device="cuda", generator=g).to(torch.bfloat16) for _ in range(3)]


def test_attention_fwd_refuses_bad_outputs():
    q, k, v = _qkv()
    qq, kq, vq = fp.quantize_qkv(q, k, v, "nvfp4")
    for bad in (torch.empty(1, 2, 256, 128, dtype=torch.bfloat16),                   # host
                torch.empty(1, 2, 255, 128, dtype=torch.bfloat16, device="cuda"),    # too small
                torch.empty(1, 2, 256, 128, dtype=torch.float32, device="cuda"),     # dtype
                torch.empty(1, 2, 128, 256, dtype=torch.bfloat16, device="cuda").transpose(2, 3)):  # strided
        with pytest.raises(ValueError, match="out"):
            fp.attention_fwd(qq, kq, vq, out=bad)
    with pytest.raises(ValueError, match="lse"):
        fp.attention_fwd(qq, kq, vq, lse=torch.empty(1, 2, 256, dtype=torch.float16, device="cuda"))
    with pytest.raises(ValueError, match="lse"):
        fp.attention_fwd(qq, kq, vq, lse=torch.empty(1, 2, 256))
    out, lse = fp.attention_fwd(qq, kq, vq)     # the well-formed call still runs
    torch.cuda.synchronize()
    assert fp.device_error() == 0 and torch.isfinite(out.float()).all()


def test_quantizers_refuse_bad_words():
    q, k, v = _qkv()
    with pytest.raises(ValueError, match="static_amax"):
        fp.quantize_nvfp4(q, static_amax=torch.ones(1))                                  # host
    with pytest.raises(ValueError, match="static_amax"):
        fp.quantize_nvfp4(q, static_amax=torch.ones(1, dtype=torch.float64, device="cuda"))
    with pytest.raises(ValueError, match="nonfinite_flag"):
        fp.quantize_fp8(q, "tile128", nonfinite_flag=torch.zeros(1, dtype=torch.int64, device="cuda"))
    with pytest.raises(ValueError, match="nonfinite_flag"):
        fp.quantize_qkv(q, k, v, "nvfp4", nonfinite_flag=torch.zeros(1, dtype=torch.int32))
    with pytest.raises(ValueError, match="out"):
        fp.tensor_amax(q, out=torch.empty(0, dtype=torch.float32, device="cuda"))
    with pytest.raises(ValueError, match="static_amax"):
        fp.quantize_nvfp4_v(v, static_amax=torch.ones(2))
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    fp.quantize_nvfp4(q, nonfinite_flag=flag)     # the well-formed call still runs
    torch.cuda.synchronize()
    assert int(flag) == 0


def test_attention_fwd_refuses_host_tile_mask():
    q, k, v = _qkv(N=384)
    plan = fp.sta_plan((1, 1, 3), (2, 8, 8), (1, 1, 3))   # three 128-token tiles in a row
    qq, kq = fp.quantize_fp8(q, "tile128"), fp.quantize_fp8(k, "tile128")
    vq = fp.quantize_fp8(v, "channel")
    with pytest.raises(ValueError, match="tile_mask"):
        fp.attention_fwd(qq, kq, vq, tile_mask=plan.to("cpu"))
    out, _ = fp.attention_fwd(qq, kq, vq, tile_mask=plan.to("cuda"))
    torch.cuda.synchronize()
    assert fp.device_error() == 0 and torch.isfinite(out.float()).all()
