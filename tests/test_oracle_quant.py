"""Pins for the oracle's NVFP4 and FP8 quantizers (CPU only).

Checks: hand-worked examples, exactly representable inputs surviving, the
amax element mapping to the format maximum, zero blocks, the error bound of
half a grid step, quantize(dequantize(quantize(x))) == quantize(x), the FP8
element conversion against torch's float8 cast, and the swizzled scale layout
against byte positions worked by hand from NVIDIA's published tensor-core
scale-factor layout (tests/golden/nvfp4_sf_layout.json).
"""
import json
import os

import numpy as np
import pytest
import torch

from oracle import codec, quant

F32 = np.float32


GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _bf16(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).float().numpy()


def test_nvfp4_hand_example():
    # static amax 2688 -> s_t = 1 exactly; block amax 3 -> 3/6 = 0.5 -> E4M3 0x30
    x = np.zeros(16, dtype=F32)
    x[:6] = [3.0, -1.2, 0.74, 0.26, 2.2, -3.0]
    codes, sb, s_t = quant.quantize_nvfp4(x[None], static_amax=2688.0)
    assert s_t == F32(1.0)
    assert sb[0, 0] == 0x30 and codec.e4m3_decode(0x30) == 0.5
    # x / 0.5 = [6, -2.4, 1.48, 0.52, 4.4, -6] -> [6, -2, 1.5, 0.5, 4, -6]
    assert list(codes[0, :6]) == [7, 8 | 4, 3, 1, 6, 8 | 7]
    assert list(codes[0, 6:]) == [0] * 10


def test_nvfp4_grid_points_survive_and_amax_maps_to_6():
    rng = np.random.default_rng(0)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    # blocks whose values are e2m1 grid values times an exact E4M3 scale, max 6
    scales = codec.e4m3_decode(rng.integers(0x20, 0x60, 32))
    vals = rng.choice(grid, (32, 16)) * rng.choice([-1, 1], (32, 16))
    vals[:, 3] = 6.0
    x = (vals * scales[:, None]).astype(F32)
    codes, sb, s_t = quant.quantize_nvfp4(x, static_amax=2688.0)
    assert s_t == F32(1.0)
    assert np.array_equal(codec.e4m3_decode(sb[:, 0]), scales)
    assert np.array_equal(codec.e2m1_decode(codes), vals)
    assert np.all(codes[:, 3] == 7)


def test_nvfp4_zero_block_and_tensor():
    x = np.zeros((2, 32), dtype=F32)
    x[1, :16] = 1.0
    codes, sb, s_t = quant.quantize_nvfp4(x)
    assert np.all(codes[0] == 0) and np.all(sb[0] == 0)
    assert np.all(codes[1, 16:] == 0) and sb[1, 1] == 0
    c0, sb0, st0 = quant.quantize_nvfp4(np.zeros((4, 16), dtype=F32))
    assert st0 == F32(1.0) and np.all(c0 == 0) and np.all(sb0 == 0)


def test_nvfp4_tensor_scale_and_block_max():
    rng = np.random.default_rng(3)
    x = _bf16(rng.standard_normal((8, 128)) * 3)
    codes, sb, s_t = quant.quantize_nvfp4(x)
    A = F32(np.abs(x).max())
    assert s_t == F32(A / F32(2688.0))
    # the tensor-amax element sits in a block whose scale is (nearly) 448,
    # and it maps to +-6
    i, j = np.unravel_index(np.abs(x).argmax(), x.shape)
    assert codec.e4m3_decode(sb[i, j // 16]) == 448.0
    assert codes[i, j] & 7 == 7


def test_nvfp4_error_bound():
    rng = np.random.default_rng(4)
    x = _bf16(rng.standard_normal((64, 128)))
    x[:, 5] *= 20
    codes, sb, s_t = quant.quantize_nvfp4(x)
    xh = quant.dequantize_nvfp4(codes, sb, s_t)
    den = np.repeat(codec.e4m3_decode(sb), 16, axis=-1) * float(s_t)
    y = np.abs(x / den)
    gap = np.where(y < 2, 0.5, np.where(y < 4, 1.0, 2.0))
    assert np.all(np.abs(x - xh) <= (gap / 2) * den * (1 + 1e-5))


def test_nvfp4_roundtrip_idempotent():
    rng = np.random.default_rng(5)
    x = _bf16(rng.standard_normal((16, 64)))
    amax = np.abs(x).max()
    c1, sb1, st1 = quant.quantize_nvfp4(x)
    xh = quant.dequantize_nvfp4(c1, sb1, st1).astype(F32)
    c2, sb2, st2 = quant.quantize_nvfp4(xh, static_amax=amax)
    assert st1 == st2
    assert np.array_equal(sb1, sb2)
    assert np.array_equal(codec.e2m1_decode(c1), codec.e2m1_decode(c2))


def test_nvfp4_sf_swizzle_golden_positions():
    """The scale layout against byte positions worked by hand from NVIDIA's
    published tensor-core scale-factor layout (tests/golden/nvfp4_sf_layout.json):
    a single marked scale must land at exactly that byte, nowhere else."""
    gold = json.load(open(os.path.join(GOLDEN, "nvfp4_sf_layout.json")))
    for case in gold["cases"]:
        N, d = case["N"], case["d"]
        sf = np.zeros((1, N, d // 16), dtype=np.uint8)
        sf[0, case["row"], case["col"]] = 0xAB
        sw = quant.nvfp4_sf_swizzle(sf, N, d).reshape(-1)
        assert sw.size == -(-N // 128) * (d // 64) * 512
        hit = np.flatnonzero(sw)
        assert hit.tolist() == [case["byte"]], (case, hit)


def test_nvfp4_sf_swizzle_is_a_bijection_with_zero_padding():
    """Every (row, column) scale of a ragged tensor lands at its own byte,
    and the bytes of the rows past N that pad the last 128-row block are 0."""
    N, d = 200, 128
    ncol = d // 16
    seen = np.zeros((-(-N // 128)) * (d // 64) * 512, dtype=np.int64)
    for col in range(ncol):  # one column at a time: a uint8 cannot label every scale
        sf = np.zeros((1, N, ncol), dtype=np.uint8)
        sf[0, :, col] = 1
        seen += quant.nvfp4_sf_swizzle(sf, N, d).reshape(-1)
    assert seen.max() == 1 and seen.sum() == N * ncol
    rng = np.random.default_rng(6)
    sf = rng.integers(1, 256, (3, N, ncol)).astype(np.uint8)
    sw = quant.nvfp4_sf_swizzle(sf, N, d)
    assert np.count_nonzero(sw) == np.count_nonzero(sf)
    # the 56 padding rows of the second block (200..255) hold no scale
    pad = np.zeros_like(seen, dtype=bool)
    pad[np.flatnonzero(seen == 0)] = True
    assert np.all(sw.reshape(3, -1)[:, pad] == 0) and pad.sum() == (256 - N) * ncol


def test_fp8_tile_amax_maps_to_448_and_matches_torch_cast():
    rng = np.random.default_rng(7)
    x = _bf16(rng.standard_normal((2, 3, 300, 64)) * 5)   # ragged: 300 = 2*128 + 44
    codes, s = quant.quantize_fp8_tile(x)
    assert s.shape == (2, 3, 3)
    for t in range(3):
        blk = x[:, :, t * 128:(t + 1) * 128]
        A = np.abs(blk).max(axis=(-2, -1)).astype(F32)
        assert np.array_equal(s[:, :, t], F32(448.0) / A)
    s_tok = np.repeat(s, 128, axis=-1)[..., :300]
    prod = (x * s_tok[..., None]).astype(F32)
    ref = torch.from_numpy(np.clip(prod, -448, 448)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codes, ref)
    # every tile has its amax element at +-448
    dec = np.abs(codec.e4m3_decode(codes))
    for t in range(3):
        assert np.all(dec[:, :, t * 128:(t + 1) * 128].max(axis=(-2, -1)) == 448.0)


def test_fp8_channel_scales_and_bound():
    rng = np.random.default_rng(8)
    x = _bf16(rng.standard_normal((1, 2, 257, 64)))
    x[..., 7] *= 30
    codes, s = quant.quantize_fp8_channel(x)
    A = np.abs(x).max(axis=-2).astype(F32)
    assert np.array_equal(s, F32(448.0) / A)
    xh = quant.dequantize_fp8_channel(codes, s)
    y = np.abs(x * s[..., None, :]).astype(np.float64)
    # half an E4M3 step at y: subnormal step 2^-9, else 2^(floor(log2 y) - 3)
    e = np.floor(np.log2(np.maximum(y, 2.0 ** -6)))
    half = np.where(y < 2.0 ** -6, 2.0 ** -10, 2.0 ** (e - 4))
    assert np.all(np.abs(x * s[..., None, :] - codec.e4m3_decode(codes)) <= half * (1 + 1e-6))
    assert np.all(np.abs(codec.e4m3_decode(codes)).max(axis=-2) == 448.0)


def test_fp8_roundtrip_idempotent_and_zero():
    rng = np.random.default_rng(9)
    x = _bf16(rng.standard_normal((1, 1, 256, 128)))
    c1, s1 = quant.quantize_fp8_tile(x)
    xh = quant.dequantize_fp8_tile(c1, s1).astype(F32)
    c2, s2 = quant.quantize_fp8_tile(xh)
    assert np.array_equal(c1, c2)
    assert np.allclose(s1, s2, rtol=3e-7, atol=0)
    cz, sz = quant.quantize_fp8_channel(np.zeros((1, 1, 10, 16), dtype=F32))
    assert np.all(cz == 0) and np.all(sz == 1.0)


@pytest.mark.parametrize("group", [1, 2, 3, 5])
def test_fp8_group_scales_and_torch_cast(group):
    # N = 600: 5 tiles, the last one ragged (88 tokens). Each group's scale is
    # 448 / amax over exactly its tokens, repeated for its tiles; codes equal
    # torch's E4M3 cast of x * s.
    rng = np.random.default_rng(10 + group)
    x = _bf16(rng.standard_normal((2, 2, 600, 64)) * 3)
    x[0, 1, 590, 5] = 40.0                       # an outlier in the ragged tail
    codes, s = quant.quantize_fp8_group(x, group)
    assert s.shape == (2, 2, 5)
    for t in range(5):
        g0 = (t // group) * group
        tokens = x[:, :, g0 * 128:min(600, (g0 + group) * 128)]
        A = np.abs(tokens).max(axis=(-2, -1)).astype(F32)
        assert np.array_equal(s[:, :, t], F32(448.0) / A), t
    s_tok = np.repeat(s, 128, axis=-1)[..., :600]
    prod = (x * s_tok[..., None]).astype(F32)
    ref = torch.from_numpy(np.clip(prod, -448, 448)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codes, ref)
    # the amax element of every group maps to +-448
    dec = np.abs(codec.e4m3_decode(codes))
    for g0 in range(0, 5, group):
        assert np.all(dec[:, :, g0 * 128:(g0 + group) * 128].max(axis=(-2, -1)) == 448.0)


def test_fp8_group_of_one_tile_is_per_tile_and_whole_head_is_one_scale():
    rng = np.random.default_rng(12)
    x = _bf16(rng.standard_normal((1, 3, 300, 128)))
    c1, s1 = quant.quantize_fp8_group(x, 1)
    c0, s0 = quant.quantize_fp8_tile(x)
    assert np.array_equal(c1, c0) and np.array_equal(s1, s0)
    ch, sh = quant.quantize_fp8_group(x, 3)
    A = np.abs(x).max(axis=(-2, -1)).astype(F32)
    assert np.all(sh == (F32(448.0) / A)[..., None])


def test_step_phase_worked_example():
    # D = 50 steps with the page's alpha1 = 0.2, alpha2 = 0.7: t1 = 10, t2 = 35
    from oracle import schedule
    got = [schedule.step_phase(t, 50) for t in range(1, 51)]
    assert got == [schedule.EARLY] * 10 + [schedule.MIDDLE] * 25 + [schedule.LATE] * 15
    # D = 7: t1 = 1.4, t2 = 4.9 -> steps 1 | 2..4 | 5..7
    assert [schedule.step_phase(t, 7) for t in range(1, 8)] == [0, 1, 1, 1, 2, 2, 2]


def test_nvfp4_tokens_grid_values_survive_and_padding_is_zero():
    # V [N = 40, d = 32]: in channel c, token block b (16 tokens) holds E2M1
    # grid values times a scale that E4M3 represents exactly, with one element
    # at 6 * scale so the block's amax is 6 * scale. Channel 0, block 0 has
    # scale 448, which puts the tensor amax at 2688 and s_t at exactly 1. Then
    # every block scale encodes exactly and dequantize(quantize(v)) == v.
    # Tokens 40..127 are padding: zero codes and zero scales.
    rng = np.random.default_rng(21)
    grid = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    N, d = 40, 32
    v = np.zeros((N, d), dtype=np.float64)
    scale = np.zeros((d, 3))
    for c in range(d):
        for b in range(3):
            t0, t1 = 16 * b, min(N, 16 * b + 16)
            vals = rng.choice(grid, t1 - t0) * rng.choice([-1, 1], t1 - t0)
            vals[0] = 6.0
            scale[c, b] = 448.0 if (c, b) == (0, 0) else 2.0 ** -(c % 5) * (b + 1)
            v[t0:t1, c] = vals * scale[c, b]
    codes, sb, s_t = quant.quantize_nvfp4_tokens(v.astype(np.float32))
    assert codes.shape == (d, 128) and sb.shape == (d, 8)
    assert s_t == np.float32(1.0)
    back = quant.dequantize_nvfp4_tokens(codes, sb, s_t, N)
    assert np.array_equal(back, v)
    assert np.all(codes[:, 48:] == 0) and np.all(sb[:, 3:] == 0)
    # blocks run along tokens: (channel c, token block b) has scale[c, b]
    assert np.array_equal(codec.e4m3_decode(sb[:, :3]), scale)
