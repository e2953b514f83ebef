"""Block-scaled quantizers for Q, K and V: TEST INFRASTRUCTURE ONLY.

Arrays are float32 numpy arrays shaped [..., N, d] (bf16 inputs widen to
float32 exactly). Every scale computation is one correctly rounded float32
operation in the order written below, with no fused multiply-add, so that the
codes and scales are fixed bit for bit.

NVFP4 (Blackwell FP4 practice page, section 1 "micro-scaling": a block of
values is divided by a scale, rounded to FP4, and the scale is kept in FP8).
The pages leave the two-level arithmetic open; the reading used here is:
  A_t  = max |x| over the whole tensor (or a caller-supplied static amax)
  s_t  = A_t / 2688            (2688 = 6 * 448; s_t = 1 when A_t = 0)
  per 16-element block along d:
    A_b  = max |x| over the block
    sb   = E4M3( A_b / (6 * s_t) )           (E4M3 block scale, RNE, saturating)
    den  = dec(sb) * s_t
    code = E2M1( x * (1 / den) )             (all codes 0 when den == 0)
  dequantized value: E2M1val * dec(sb) * s_t.

FP8 E4M3 (FPSAttention page, section 2.1 conversion formula
X_hat = dequantize(FP8_convert(X * s_g)) / s_g, and section 3.1 "staged
quantization": Q/K per block, V per channel):
  s    = 448 / A    (A = amax of the block or channel; s = 1 when A = 0)
  code = E4M3( x * s ),   dequantized value dec(code) / s.
Q/K blocks are 128-token tiles of one (batch, head) spanning all d channels; a
last partial tile takes its amax over its valid tokens only. V channels take
their amax over all N tokens of one (batch, head).
"""
from __future__ import annotations

import numpy as np

from . import codec

F32 = np.float32
NVFP4_BLOCK = 16
FP8_TILE = 128


def _f32(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float32)


# ----------------------------------------------------------------------------
# NVFP4
# ----------------------------------------------------------------------------

def nvfp4_tensor_scale(amax) -> np.float32:
    """s_t = A_t / 2688 in float32, 1 when A_t == 0."""
    a = F32(amax)
    return F32(1.0) if a == 0 else F32(a / F32(2688.0))


def quantize_nvfp4(x, static_amax=None):
    """Quantize ``x`` [..., d] to NVFP4.

    Returns (codes, block_scales, s_t):
      codes         uint8 [..., d]      4-bit E2M1 codes, one per element
      block_scales  uint8 [..., d/16]   E4M3 codes of the block scales
      s_t           float32             tensor scale (a decode multiplier)
    """
    x = _f32(x)
    d = x.shape[-1]
    assert d % NVFP4_BLOCK == 0
    amax = F32(np.max(np.abs(x))) if static_amax is None else F32(static_amax)
    s_t = nvfp4_tensor_scale(amax)
    blocks = x.reshape(x.shape[:-1] + (d // NVFP4_BLOCK, NVFP4_BLOCK))
    a_b = np.max(np.abs(blocks), axis=-1).astype(F32)
    sb = codec.e4m3_encode(a_b / (F32(6.0) * s_t))
    den = codec.e4m3_decode(sb).astype(F32) * s_t
    with np.errstate(divide="ignore", over="ignore", invalid="ignore"):
        inv = F32(1.0) / den
        y = blocks * inv[..., None]
    usable = (den != 0) & np.isfinite(inv)
    y = np.where(usable[..., None], y, F32(0.0))
    codes = codec.e2m1_encode(y).reshape(x.shape)
    # A zero block (or an unusable scale) gives +0 codes, whatever the signs.
    codes = np.where(np.repeat(usable, NVFP4_BLOCK, axis=-1), codes, np.uint8(0))
    return codes.astype(np.uint8), sb, s_t


def dequantize_nvfp4(codes, block_scales, s_t) -> np.ndarray:
    """E2M1val * dec(sb) * s_t, exact in float64."""
    v = codec.e2m1_decode(codes)
    d = v.shape[-1]
    sbv = np.repeat(codec.e4m3_decode(block_scales), NVFP4_BLOCK, axis=-1)
    return v * sbv * float(s_t)


def quantize_nvfp4_tokens(v, pad_to: int = 128):
    """NVFP4 for V as the second operand of a block-scaled P V product: the
    same recipe as quantize_nvfp4 (tensor amax over all of ``v``), with the
    16-element blocks running along the sequence (the contraction axis of
    P V) instead of along d.

    ``v`` [..., N, d]. The sequence is zero-padded to a multiple of
    ``pad_to`` tokens. Returns (codes uint8 [..., d, Np], block_scales uint8
    [..., d, Np/16], s_t): channel-major, tokens along the last axis.
    """
    v = _f32(v)
    N = v.shape[-2]
    Np = -(-N // pad_to) * pad_to
    vt = np.zeros(v.shape[:-2] + (v.shape[-1], Np), dtype=F32)
    vt[..., :N] = np.swapaxes(v, -1, -2)
    return quantize_nvfp4(vt)


def dequantize_nvfp4_tokens(codes, block_scales, s_t, N: int) -> np.ndarray:
    """Inverse arrangement of quantize_nvfp4_tokens: float64 [..., N, d]."""
    return np.swapaxes(dequantize_nvfp4(codes, block_scales, s_t), -1, -2)[..., :N, :]


def nvfp4_sf_swizzle(block_scales: np.ndarray, N: int, d: int) -> np.ndarray:
    """Arrange logical block scales [BH, N, d/16] into the tensor-core layout.

    Layout (per 128-row block of one (batch, head), per group of four scale
    columns): 512 bytes where the scale of row r = 32*j + i (i < 32, j < 4) and
    column 4*a + c (c < 4) sits at byte 16*i + 4*j + c of group a. Rows past N
    are zero. Shape of the result: [BH, ceil(N/128), d/64, 512] uint8.
    """
    bh = block_scales.shape[0]
    nb = -(-N // 128)
    ga = d // 64
    out = np.zeros((bh, nb, ga, 512), dtype=np.uint8)
    for r in range(N):
        blk, rr = divmod(r, 128)
        j, i = divmod(rr, 32)
        for col in range(d // 16):
            a, c = divmod(col, 4)
            out[:, blk, a, 16 * i + 4 * j + c] = block_scales[:, r, col]
    return out


# ----------------------------------------------------------------------------
# FP8 E4M3
# ----------------------------------------------------------------------------

def fp8_scale(amax) -> np.ndarray:
    """s = 448 / A in float32 (1 where A == 0)."""
    a = _f32(amax)
    with np.errstate(divide="ignore"):
        s = F32(448.0) / a
    return np.where(a == 0, F32(1.0), s).astype(F32)


def quantize_fp8_tile(x, tile: int = FP8_TILE):
    """Per-(batch, head) 128-token-tile quantization of ``x`` [..., N, d].

    Returns (codes uint8 [..., N, d], scales float32 [..., ceil(N/tile)]).
    """
    x = _f32(x)
    N = x.shape[-2]
    nt = -(-N // tile)
    amax = np.zeros(x.shape[:-2] + (nt,), dtype=F32)
    for t in range(nt):
        amax[..., t] = np.max(np.abs(x[..., t * tile:(t + 1) * tile, :]), axis=(-2, -1))
    s = fp8_scale(amax)
    s_tok = np.repeat(s, tile, axis=-1)[..., :N]
    codes = codec.e4m3_encode(x * s_tok[..., None])
    return codes, s


def quantize_fp8_group(x, group: int, tile: int = FP8_TILE):
    """Q/K quantization with one scale per group of ``group`` consecutive
    128-token tiles of one (batch, head): the coarser granularities of the
    FPSAttention page's denoising-step-aware schedule (section 3.2: coarse,
    intermediate and fine granularities by phase). group = 1 is the per-tile
    quantization; a group of all tiles is one scale per (batch, head); a
    group of the tiles of one 3D video tile is one scale per video tile.
    A is the amax over the group's tokens (a last partial group over its
    valid tokens); s = 448 / A; code = E4M3(x * s).

    Returns (codes uint8 [..., N, d], scales float32 [..., ceil(N/tile)]): the
    scale of each tile, i.e. its group's scale repeated, so the result
    dequantizes with dequantize_fp8_tile.
    """
    assert group >= 1
    x = _f32(x)
    N = x.shape[-2]
    nt = -(-N // tile)
    span = group * tile
    s = np.zeros(x.shape[:-2] + (nt,), dtype=F32)
    for g0 in range(0, nt, group):
        a = np.max(np.abs(x[..., g0 * tile:g0 * tile + span, :]), axis=(-2, -1)).astype(F32)
        s[..., g0:g0 + group] = fp8_scale(a)[..., None]
    s_tok = np.repeat(s, tile, axis=-1)[..., :N]
    codes = codec.e4m3_encode(x * s_tok[..., None])
    return codes, s


def quantize_fp8_channel(x):
    """Per-(batch, head) per-channel quantization of ``x`` [..., N, d].

    Returns (codes uint8 [..., N, d], scales float32 [..., d]).
    """
    x = _f32(x)
    amax = np.max(np.abs(x), axis=-2).astype(F32)
    s = fp8_scale(amax)
    codes = codec.e4m3_encode(x * s[..., None, :])
    return codes, s


def dequantize_fp8_tile(codes, scales, tile: int = FP8_TILE) -> np.ndarray:
    N = codes.shape[-2]
    s_tok = np.repeat(np.asarray(scales, dtype=np.float64), tile, axis=-1)[..., :N]
    return codec.e4m3_decode(codes) / s_tok[..., None]


def dequantize_fp8_channel(codes, scales) -> np.ndarray:
    return codec.e4m3_decode(codes) / np.asarray(scales, dtype=np.float64)[..., None, :]
