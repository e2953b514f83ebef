"""Seeded synthetic inputs for the quantized-attention workloads.

This module only draws random numbers and arranges them into tensors. It holds
none of the method's arithmetic (no quantization, no attention), so both the
CPU oracle and the CUDA path can take their inputs from here without sharing
any computation.

The workloads restate the ones the pages study:
  * an LLM prefill with a causal mask (FlashAttention-4 article on the
    Blackwell tensor memory design; "LLM prefill" usage),
  * video-DiT attention over time x height x width tokens (FPSAttention page,
    section 1: Wan2.1-14B 720p, 3D attention over video tokens),
  * sliding-tile sparse attention over (6,8,8)-token tiles (FPSAttention page,
    section 2.2, "STA"),
  * a sequence-length sweep, and its longest single-GPU point (N = 128K,
    d = 128, 32 heads) as a workload of its own.

Recipe (all CPU torch.Generator, fp32 draws cast to bf16):
  * one generator per workload, seeded with the workload's seed; Q, then K,
    then V are drawn from the same stream, ~N(0,1);
  * outlier channels: per head, ``randperm(d)[:4]`` from the same stream, the
    same channels for Q and K, multiplied by 20;
  * smooth spatial bias for video workloads: for each channel c a frequency
    triple f in {1,2}^3 and a phase phi_c ~ U[0, 2pi); the bias
    ``sin(2pi(f_t t/T + f_h h/Hs + f_w w/W) + phi_c)`` is added to Q, K and V.
  * ``make_qkv(..., device="cuda")`` draws the same recipe from a seeded CUDA
    generator on the device (other bits than the CPU stream, same
    distributions). The long-sequence workloads are defined by that device
    stream: their three 1 GiB tensors take seconds on the device and about
    half a minute on host cores.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Tuple

import torch

__all__ = [
    "Workload", "WORKLOADS", "get", "make_qkv", "video_tile_major_perm",
    "sweep_workloads",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    """One attention problem: shapes, dtypes and input recipe."""
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    qk_format: str            # "nvfp4" or "fp8"
    seed: int
    outliers: bool = False
    video: Optional[Tuple[int, int, int]] = None       # (T, Hs, W) token grid
    sta_tile: Optional[Tuple[int, int, int]] = None    # tile size in tokens
    sta_window: Optional[Tuple[int, int, int]] = None  # window size in tiles
    device_draw: bool = False  # the recipe is drawn on the CUDA device (see make_qkv)

    @property
    def sparse(self) -> bool:
        return self.sta_tile is not None

    def dense_flops(self) -> float:
        """Dense-equivalent flops of QK^T and PV: 4*B*H*N^2*d, halved if causal."""
        f = 4.0 * self.B * self.H * self.N * self.N * self.d
        return f / 2 if self.causal else f

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    # 1: tiny NVFP4 attention
    "tiny_nvfp4": Workload("tiny_nvfp4", B=1, H=2, N=256, d=64, causal=False,
                           qk_format="nvfp4", seed=0),
    # 2: LLM prefill, causal, outlier channels
    "llm_prefill_causal": Workload("llm_prefill_causal", B=4, H=32, N=4096, d=128,
                                   causal=True, qk_format="nvfp4", seed=2,
                                   outliers=True),
    # 3: video DiT dense, 21x45x80 tokens, time-major
    "video_dense_fp8": Workload("video_dense_fp8", B=1, H=40, N=21 * 45 * 80, d=128,
                                causal=False, qk_format="fp8", seed=3,
                                video=(21, 45, 80)),
    # 4: sliding-tile sparse video, 18x48x80 tokens in (6,8,8) tiles
    "video_sta_fp8": Workload("video_sta_fp8", B=1, H=40, N=18 * 48 * 80, d=128,
                              causal=False, qk_format="fp8", seed=4,
                              video=(18, 48, 80), sta_tile=(6, 8, 8),
                              sta_window=(3, 3, 5)),
    # 5: the sequence sweep's longest single-GPU point, dense, x20 outliers;
    # NVFP4 Q/K with FP8 P/V, and the all-FP8 variant. Drawn on the device.
    "long_seq_128k_nvfp4": Workload("long_seq_128k_nvfp4", B=1, H=32, N=131072, d=128, causal=False,
                                    qk_format="nvfp4", seed=5, outliers=True, device_draw=True),
    "long_seq_128k_fp8": Workload("long_seq_128k_fp8", B=1, H=32, N=131072, d=128, causal=False,
                                  qk_format="fp8", seed=5, outliers=True, device_draw=True),
}


def sweep_workloads():
    """Sequence sweep: N in {1K..128K}, d in {64,128}, B*H*N = 2^22, H = 32."""
    out = []
    for N in (1024, 4096, 16384, 32768, 65536, 131072):
        B = (1 << 22) // (32 * N)
        for d in (64, 128):
            for causal in (False, True):
                for fmt in ("nvfp4", "fp8"):
                    out.append(Workload(f"sweep_N{N}_d{d}_{'c' if causal else 'nc'}_{fmt}",
                                        B=B, H=32, N=N, d=d, causal=causal,
                                        qk_format=fmt, seed=5, outliers=True))
    return out


def get(name: str) -> Workload:
    return WORKLOADS[name]


def video_tile_major_perm(grid: Tuple[int, int, int], tile: Tuple[int, int, int]) -> torch.Tensor:
    """Index map from tile-major position to time-major (raster) position.

    Tokens of a T x Hs x W video are numbered t*Hs*W + h*W + w in raster order.
    Tile-major order lists the tiles in raster order over the tile grid and,
    inside each tile, its tokens in raster order. ``perm[i]`` is the raster
    index of the i-th token in tile-major order, so ``x_tile = x_raster[perm]``.
    """
    T, Hs, W = grid
    tt, th, tw = tile
    assert T % tt == 0 and Hs % th == 0 and W % tw == 0
    t = torch.arange(T).view(T // tt, tt, 1, 1, 1, 1)
    h = torch.arange(Hs).view(1, 1, Hs // th, th, 1, 1)
    w = torch.arange(W).view(1, 1, 1, 1, W // tw, tw)
    raster = (t * Hs * W + h * W + w)                       # [nt,tt,nh,th,nw,tw]
    raster = raster.permute(0, 2, 4, 1, 3, 5).contiguous()  # [nt,nh,nw,tt,th,tw]
    return raster.reshape(-1)


def _video_bias(gen: torch.Generator, grid, d: int) -> torch.Tensor:
    T, Hs, W = grid
    dev = gen.device
    f = torch.randint(1, 3, (3, d), generator=gen, device=dev).to(torch.float32).cpu()
    phi = torch.rand(d, generator=gen, device=dev).cpu() * (2 * math.pi)
    t = torch.arange(T, dtype=torch.float32).view(T, 1, 1, 1) / T
    h = torch.arange(Hs, dtype=torch.float32).view(1, Hs, 1, 1) / Hs
    w = torch.arange(W, dtype=torch.float32).view(1, 1, W, 1) / W
    arg = 2 * math.pi * (f[0] * t + f[1] * h + f[2] * w) + phi
    return torch.sin(arg).reshape(T * Hs * W, d)


def make_qkv(w: Workload, *, heads: Optional[int] = None, batch: Optional[int] = None,
             N: Optional[int] = None, tile_major: bool = True, device=None):
    """Return bf16 tensors q, k, v of shape [B, H, N, d] for workload ``w``.

    ``heads``/``batch``/``N`` override the sizes for reduced parity cases; the
    seed and recipe stay the workload's. Sliding-tile workloads come in
    tile-major token order unless ``tile_major`` is False (raster order, as a
    video model holds its tokens). ``device`` None draws from a CPU
    generator and returns CPU tensors; a CUDA device draws from a CUDA
    generator seeded the same way and returns tensors on that device.
    """
    B = w.B if batch is None else batch
    H = w.H if heads is None else heads
    n = w.N if N is None else N
    d = w.d
    dev = torch.device("cpu") if device is None else torch.device(device)
    gen = torch.Generator(device=dev).manual_seed(w.seed)
    q = torch.randn(B, H, n, d, generator=gen, device=dev)
    k = torch.randn(B, H, n, d, generator=gen, device=dev)
    v = torch.randn(B, H, n, d, generator=gen, device=dev)
    if w.outliers:
        for hh in range(H):
            ch = torch.randperm(d, generator=gen, device=dev)[:4]
            q[:, hh, :, ch] *= 20.0
            k[:, hh, :, ch] *= 20.0
    if w.video is not None and n == w.N:
        bias = _video_bias(gen, w.video, d).to(dev)
        q += bias
        k += bias
        v += bias
        if w.sta_tile is not None and tile_major:
            perm = video_tile_major_perm(w.video, w.sta_tile).to(dev)
            q, k, v = q[:, :, perm], k[:, :, perm], v[:, :, perm]
    return (q.to(torch.bfloat16).contiguous(), k.to(torch.bfloat16).contiguous(),
            v.to(torch.bfloat16).contiguous())
