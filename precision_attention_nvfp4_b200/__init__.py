"""Quantized attention forward (NVFP4 / FP8) for B200, Python binding.

Every function marshals torch tensors into the C ABI of ``libfpattn.so``
(include/fpattn.h) and enqueues the library's CUDA kernels on the current
torch stream; torch only provides device memory and streams. Nothing here
computes any part of the method on the host.

Public calls
  quantize_nvfp4(x)            -> Nvfp4Tensor(codes, block_sf, tensor_scale)
  quantize_fp8(x, granularity) -> Fp8Tensor(codes, scales); granularity
                                  "tile128", "channel", or "group" with
                                  group_tiles tiles per scale
                                  (with video=VideoLayout: x in raster order,
                                  codes and scales in tile-major order)
  quantize_qkv(q, k, v, fmt)   -> (q, k, v) quantized together: Q/K NVFP4 or
                                  FP8 per tile, V FP8 per channel, in four
                                  fused launches (same bits as the calls above)
  quantize_nvfp4_v(x)          -> Nvfp4VTensor: V in NVFP4 with 16-token
                                  blocks, channel-major (all-NVFP4 attention)
  sta_plan(grid, tile, window) -> StaPlan (host CSR over 128-token blocks)
  step_phase(t, num_steps)     -> 0 early / 1 middle / 2 late denoising phase
  attention_fwd(q, k, v, ...)  -> (out, lse) on quantized operands
  attention(q, k, v, ...)      -> (out, lse) from bf16 inputs: quantize + fwd;
                                  host (pinned) inputs are copied in and the
                                  result copied back. With video=VideoLayout,
                                  inputs and outputs are in raster order and
                                  the tile-major permutation happens inside
                                  the quantize and attention kernels.
"""
from __future__ import annotations

import ctypes
import dataclasses
from typing import Optional, Sequence, Tuple

import numpy as np
import torch

from . import _lib
from ._lib import FpattnError

__all__ = ["Nvfp4Tensor", "Nvfp4VTensor", "Fp8Tensor", "StaPlan", "VideoLayout", "quantize_nvfp4", "quantize_qkv",
           "quantize_nvfp4_v", "quantize_fp8", "sta_plan",
           "step_phase", "attention_fwd", "attention", "device_error", "library", "FpattnError",
           "head_range", "tensor_amax", "causal_plan", "attention_sharded"]


def library() -> ctypes.CDLL:
    return _lib.load()


def _stream() -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _aux(t: Optional[torch.Tensor], dev: torch.device, dtype: torch.dtype, n: int, name: str) -> Optional[int]:
    """Device pointer of an optional buffer the kernels read or write (an
    amax, a flag, an output), after checking that it is a contiguous tensor
    of ``dtype`` on ``dev`` with at least ``n`` elements: anything else is
    refused before a launch could touch it."""
    if t is None:
        return None
    if (not isinstance(t, torch.Tensor) or not t.is_cuda or t.device != dev or t.dtype != dtype
            or not t.is_contiguous() or t.numel() < n):
        raise ValueError(f"{name}: expected a contiguous {dtype} tensor on {dev} with at least {n} elements")
    return t.data_ptr()


def _desc(t: torch.Tensor, dtype: int, B: int, H: int, N: int, d: int) -> _lib.Tensor:
    return _lib.Tensor(t.data_ptr(), dtype, B, H, N, d)


def _check_bf16(x: torch.Tensor) -> Tuple[int, int, int, int]:
    if x.dim() != 4 or x.dtype != torch.bfloat16 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("expected a contiguous CUDA bf16 tensor [B, H, N, d]")
    return tuple(x.shape)


@dataclasses.dataclass(frozen=True)
class VideoLayout:
    """A T x Hs x W video token grid cut into tt x th x tw tiles.

    Raster order holds token (t, h, w) in row (t*Hs + h)*W + w; tile-major
    order lists tiles in raster order and each tile's tokens in raster order.
    """
    grid: Tuple[int, int, int]
    tile: Tuple[int, int, int]

    def c(self) -> _lib.VideoLayout:
        return _lib.VideoLayout(*(int(v) for v in self.grid), *(int(v) for v in self.tile))


def _video_ref(video: Optional[VideoLayout]):
    return None if video is None else ctypes.byref(video.c())


@dataclasses.dataclass
class Nvfp4Tensor:
    codes: torch.Tensor         # uint8 [B, H, N, d/2], packed E2M1
    block_sf: torch.Tensor      # uint8 [B*H*ceil(N/128)*(d/64)*512], tensor-core scale layout
    tensor_scale: torch.Tensor  # float32 [1]
    shape: Tuple[int, int, int, int]


@dataclasses.dataclass
class Nvfp4VTensor:
    codes: torch.Tensor         # uint8 [B, H, d, 64*ceil(N/128)], packed E2M1 along tokens
    block_sf: torch.Tensor      # uint8 [B*H*ceil(N/128)*1024], tensor-core layout, channels as rows
    tensor_scale: torch.Tensor  # float32 [1]
    shape: Tuple[int, int, int, int]


@dataclasses.dataclass
class Fp8Tensor:
    codes: torch.Tensor         # uint8 [B, H, N, d] (E4M3 bits)
    scales: torch.Tensor        # float32 [B, H, ceil(N/128)] or [B, H, d]
    granularity: str            # "tile128" or "channel"
    shape: Tuple[int, int, int, int]


def quantize_nvfp4(x: torch.Tensor, static_amax: Optional[torch.Tensor] = None,
                   nonfinite_flag: Optional[torch.Tensor] = None,
                   video: Optional[VideoLayout] = None) -> Nvfp4Tensor:
    B, H, N, d = _check_bf16(x)
    lib = library()
    codes = torch.empty((B, H, N, d // 2), dtype=torch.uint8, device=x.device)
    sf = torch.empty(lib.fpattn_nvfp4_sf_bytes(B, H, N, d), dtype=torch.uint8, device=x.device)
    ts = torch.empty(1, dtype=torch.float32, device=x.device)
    xd = ctypes.byref(_desc(x, _lib.BF16, B, H, N, d))
    amax_p = _aux(static_amax, x.device, torch.float32, 1, "static_amax")
    flag_p = _aux(nonfinite_flag, x.device, torch.int32, 1, "nonfinite_flag")
    if video is None:
        st = lib.fpattn_quantize_nvfp4(xd, amax_p, codes.data_ptr(), sf.data_ptr(), ts.data_ptr(), flag_p,
                                       _stream())
    else:
        st = lib.fpattn_quantize_nvfp4_video(xd, _video_ref(video), amax_p, codes.data_ptr(),
                                             sf.data_ptr(), ts.data_ptr(), flag_p, _stream())
    _lib.check(st, "fpattn_quantize_nvfp4" + ("_video" if video is not None else ""))
    return Nvfp4Tensor(codes, sf, ts, (B, H, N, d))


def tensor_amax(x: torch.Tensor, out: Optional[torch.Tensor] = None, accumulate: bool = False,
                nonfinite_flag: Optional[torch.Tensor] = None) -> torch.Tensor:
    """max|x| of a bf16 tensor folded into ``out`` (a device float32 [1],
    zeroed first unless ``accumulate``): the amax pass of quantize_nvfp4, for
    a tensor that arrives in pieces."""
    B, H, N, d = _check_bf16(x)
    if out is None:
        out = torch.empty(1, dtype=torch.float32, device=x.device)
    out_p = _aux(out, x.device, torch.float32, 1, "out")
    flag_p = _aux(nonfinite_flag, x.device, torch.int32, 1, "nonfinite_flag")
    st = library().fpattn_tensor_amax(ctypes.byref(_desc(x, _lib.BF16, B, H, N, d)), 1 if accumulate else 0,
                                      out_p, flag_p, _stream())
    _lib.check(st, "fpattn_tensor_amax")
    return out


def quantize_nvfp4_v(x: torch.Tensor, static_amax: Optional[torch.Tensor] = None,
                     nonfinite_flag: Optional[torch.Tensor] = None,
                     video: Optional[VideoLayout] = None) -> Nvfp4VTensor:
    """V for the all-NVFP4 attention: NVFP4 blocks of 16 tokens, channel-major."""
    B, H, N, d = _check_bf16(x)
    lib = library()
    sfb = ctypes.c_size_t(0)
    nbytes = lib.fpattn_nvfp4_v_bytes(B, H, N, d, ctypes.byref(sfb))
    codes = torch.empty((B, H, d, nbytes // (B * H * d)), dtype=torch.uint8, device=x.device)
    sf = torch.empty(sfb.value, dtype=torch.uint8, device=x.device)
    ts = torch.empty(1, dtype=torch.float32, device=x.device)
    st = lib.fpattn_quantize_nvfp4_v(ctypes.byref(_desc(x, _lib.BF16, B, H, N, d)), _video_ref(video),
                                     _aux(static_amax, x.device, torch.float32, 1, "static_amax"), codes.data_ptr(),
                                     sf.data_ptr(), ts.data_ptr(),
                                     _aux(nonfinite_flag, x.device, torch.int32, 1, "nonfinite_flag"), _stream())
    _lib.check(st, "fpattn_quantize_nvfp4_v")
    return Nvfp4VTensor(codes, sf, ts, (B, H, N, d))


def quantize_fp8(x: torch.Tensor, granularity: str = "tile128",
                 nonfinite_flag: Optional[torch.Tensor] = None,
                 video: Optional[VideoLayout] = None, group_tiles: int = 1) -> Fp8Tensor:
    B, H, N, d = _check_bf16(x)
    lib = library()
    codes = torch.empty((B, H, N, d), dtype=torch.uint8, device=x.device)
    if granularity == "tile128":
        g, scales = _lib.FP8_TILE128, torch.empty((B, H, (N + 127) // 128), dtype=torch.float32, device=x.device)
    elif granularity == "channel":
        g, scales = _lib.FP8_CHANNEL, torch.empty((B, H, d), dtype=torch.float32, device=x.device)
    elif granularity == "group":
        g, scales = None, torch.empty((B, H, (N + 127) // 128), dtype=torch.float32, device=x.device)
    else:
        raise ValueError("granularity must be 'tile128', 'channel' or 'group'")
    xd = ctypes.byref(_desc(x, _lib.BF16, B, H, N, d))
    flag_p = _aux(nonfinite_flag, x.device, torch.int32, 1, "nonfinite_flag")
    if g is None:
        st = lib.fpattn_quantize_fp8_group(xd, _video_ref(video), int(group_tiles), codes.data_ptr(),
                                           scales.data_ptr(), flag_p, _stream())
        _lib.check(st, "fpattn_quantize_fp8_group")
        return Fp8Tensor(codes, scales, "tile128", (B, H, N, d))
    if video is None:
        st = lib.fpattn_quantize_fp8(xd, g, codes.data_ptr(), scales.data_ptr(), flag_p, _stream())
    else:
        st = lib.fpattn_quantize_fp8_video(xd, _video_ref(video), g, codes.data_ptr(), scales.data_ptr(),
                                           flag_p, _stream())
    _lib.check(st, "fpattn_quantize_fp8" + ("_video" if video is not None else ""))
    return Fp8Tensor(codes, scales, granularity, (B, H, N, d))


def quantize_qkv(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, qk_format: str = "nvfp4",
                 nonfinite_flag: Optional[torch.Tensor] = None, video: Optional[VideoLayout] = None):
    """Q and K (NVFP4, or FP8 per 128-token tile) and V (FP8 per channel) in
    four fused launches; returns (q, k, v) quantized exactly as the separate
    quantize_nvfp4 / quantize_fp8 calls would."""
    B, H, N, d = _check_bf16(q)
    if _check_bf16(k) != (B, H, N, d) or _check_bf16(v) != (B, H, N, d):
        raise ValueError("q, k, v must have one shape")
    if k.device != q.device or v.device != q.device:
        raise ValueError("q, k, v must be on one device")
    lib = library()
    dev = q.device
    flag_p = _aux(nonfinite_flag, dev, torch.int32, 1, "nonfinite_flag")
    nblk = (N + 127) // 128
    if qk_format == "nvfp4":
        dt = _lib.NVFP4
        qc, kc = (torch.empty((B, H, N, d // 2), dtype=torch.uint8, device=dev) for _ in range(2))
        qsf, ksf = (torch.empty(lib.fpattn_nvfp4_sf_bytes(B, H, N, d), dtype=torch.uint8, device=dev)
                    for _ in range(2))
        qs, ks = (torch.empty(1, dtype=torch.float32, device=dev) for _ in range(2))
    elif qk_format == "fp8":
        dt = _lib.E4M3
        qc, kc = (torch.empty((B, H, N, d), dtype=torch.uint8, device=dev) for _ in range(2))
        qsf = ksf = None
        qs, ks = (torch.empty((B, H, nblk), dtype=torch.float32, device=dev) for _ in range(2))
    else:
        raise ValueError("qk_format must be 'nvfp4' or 'fp8'")
    vc = torch.empty((B, H, N, d), dtype=torch.uint8, device=dev)
    vs = torch.empty((B, H, d), dtype=torch.float32, device=dev)
    st = lib.fpattn_quantize_qkv(ctypes.byref(_desc(q, _lib.BF16, B, H, N, d)),
                                 ctypes.byref(_desc(k, _lib.BF16, B, H, N, d)),
                                 ctypes.byref(_desc(v, _lib.BF16, B, H, N, d)), dt, _video_ref(video),
                                 qc.data_ptr(), _ptr(qsf), qs.data_ptr(), kc.data_ptr(), _ptr(ksf), ks.data_ptr(),
                                 vc.data_ptr(), vs.data_ptr(), flag_p, _stream())
    _lib.check(st, "fpattn_quantize_qkv")
    if qk_format == "nvfp4":
        qq, kq = Nvfp4Tensor(qc, qsf, qs, (B, H, N, d)), Nvfp4Tensor(kc, ksf, ks, (B, H, N, d))
    else:
        qq, kq = Fp8Tensor(qc, qs, "tile128", (B, H, N, d)), Fp8Tensor(kc, ks, "tile128", (B, H, N, d))
    return qq, kq, Fp8Tensor(vc, vs, "channel", (B, H, N, d))


@dataclasses.dataclass
class StaPlan:
    row_ptr: np.ndarray    # int32 [nblk + 1]
    col_idx: np.ndarray    # int32 [nnz]
    row_order: Optional[np.ndarray]  # int32 [nblk], longest rows first, or None

    @property
    def nblk(self) -> int:
        return len(self.row_ptr) - 1

    @property
    def nnz(self) -> int:
        return len(self.col_idx)

    def check(self) -> None:
        """Raises FpattnError unless the CSR is well formed (fpattn_tile_mask_check)."""
        rp = np.ascontiguousarray(self.row_ptr, dtype=np.int32)
        ci = np.ascontiguousarray(self.col_idx, dtype=np.int32)
        ro = None if self.row_order is None else np.ascontiguousarray(self.row_order, dtype=np.int32)
        if len(rp) < 1 or (ro is not None and len(ro) != len(rp) - 1):
            raise FpattnError(_lib.ERR_INVALID_ARG, "fpattn_tile_mask_check")
        _lib.check(library().fpattn_tile_mask_check(len(rp) - 1, len(ci), rp.ctypes.data,
                                                    ci.ctypes.data if len(ci) else None,
                                                    None if ro is None else ro.ctypes.data),
                   "fpattn_tile_mask_check")

    def to(self, device) -> "DeviceTileMask":
        """Checks the mask on the host, then copies it to ``device``."""
        self.check()
        return DeviceTileMask(self.nblk, self.nnz,
                              torch.from_numpy(self.row_ptr).to(device),
                              torch.from_numpy(self.col_idx).to(device),
                              None if self.row_order is None else torch.from_numpy(self.row_order).to(device))


@dataclasses.dataclass
class DeviceTileMask:
    nblk: int
    nnz: int
    row_ptr: torch.Tensor
    col_idx: torch.Tensor
    row_order: Optional[torch.Tensor]

    def desc(self, dev: Optional[torch.device] = None) -> _lib.TileMask:
        """The C descriptor; with ``dev``, after checking that the arrays are
        int32 tensors on that device, sized as nblk and nnz say."""
        if dev is not None:
            _aux(self.row_ptr, dev, torch.int32, self.nblk + 1, "tile_mask.row_ptr")
            _aux(self.col_idx, dev, torch.int32, self.nnz, "tile_mask.col_idx")
            _aux(self.row_order, dev, torch.int32, self.nblk, "tile_mask.row_order")
        return _lib.TileMask(self.nblk, self.nnz, self.row_ptr.data_ptr(), self.col_idx.data_ptr(),
                             _ptr(self.row_order))


def sta_plan(tile_grid: Sequence[int], tile: Sequence[int], window: Sequence[int]) -> StaPlan:
    """Block CSR of the 3D sliding-tile pattern (host-only planner)."""
    lib = library()
    nblk, nnz = ctypes.c_int32(0), ctypes.c_int32(0)
    args = [int(v) for v in (*tile_grid, *tile, *window)]
    _lib.check(lib.fpattn_sta_plan(*args, None, None, None, 0, ctypes.byref(nblk), ctypes.byref(nnz)),
               "fpattn_sta_plan")
    row_ptr = np.zeros(nblk.value + 1, dtype=np.int32)
    col_idx = np.zeros(max(nnz.value, 1), dtype=np.int32)
    row_order = np.zeros(nblk.value, dtype=np.int32)
    _lib.check(lib.fpattn_sta_plan(*args, row_ptr.ctypes.data, col_idx.ctypes.data, row_order.ctypes.data,
                                   nnz.value, ctypes.byref(nblk), ctypes.byref(nnz)), "fpattn_sta_plan")
    return StaPlan(row_ptr, col_idx[:nnz.value], row_order)


def causal_plan(num_heads: int, N: int, d: int, qk_format: str = "nvfp4", pv_format: str = "fp8",
                sm_count: int = 148) -> dict:
    """Schedule of a causal attention launch over num_heads (batch, head)
    problems (host-only): heads per group and schedule positions of a full
    group (longest-first order), pairs of query blocks per head (paired
    order, else 0), all positions of the launch, and the CTA count. Either
    order keeps the K/V in flight within the L2; the output does not depend
    on it."""
    fmt = {"nvfp4": 2, "fp8": 1, "e4m3": 1}
    vals = [ctypes.c_int32(0) for _ in range(5)]
    _lib.check(library().fpattn_causal_plan(int(num_heads), int(N), int(d), fmt[qk_format], fmt[pv_format],
                                            int(sm_count), *(ctypes.byref(v) for v in vals)),
               "fpattn_causal_plan")
    return dict(zip(("heads_per_group", "group_positions", "pairs_per_head", "positions", "ctas"),
                    (v.value for v in vals)))


def step_phase(t: int, num_steps: int, alpha1: float = 0.2, alpha2: float = 0.7) -> int:
    """Denoising phase of step t (1-based): 0 early, 1 middle, 2 late."""
    ph = ctypes.c_int32(0)
    _lib.check(library().fpattn_step_phase(int(t), int(num_steps), float(alpha1), float(alpha2), ctypes.byref(ph)),
               "fpattn_step_phase")
    return ph.value


def _check_operands(q, k, v) -> None:
    """Refuses, before any launch, operands the kernel would read past: q and
    k both NVFP4 or both FP8 with per-tile scales, v FP8 with per-channel
    scales or NVFP4 V, one shape [B, H, N, d] for all three, every buffer
    sized for that shape and on one CUDA device."""
    if isinstance(q, Nvfp4Tensor) and isinstance(k, Nvfp4Tensor):
        pass
    elif isinstance(q, Fp8Tensor) and isinstance(k, Fp8Tensor):
        if q.granularity != "tile128" or k.granularity != "tile128":
            raise ValueError("FP8 q and k need per-tile scales (granularity 'tile128' or 'group')")
    else:
        raise TypeError("q and k must both be Nvfp4Tensor or both Fp8Tensor")
    if isinstance(v, Fp8Tensor):
        if v.granularity != "channel":
            raise ValueError("FP8 v needs per-channel scales (granularity 'channel')")
    elif not isinstance(v, Nvfp4VTensor):
        raise TypeError("v must be an Fp8Tensor (per channel) or an Nvfp4VTensor")
    if not (tuple(q.shape) == tuple(k.shape) == tuple(v.shape)):
        raise ValueError(f"q, k, v shapes differ: {q.shape}, {k.shape}, {v.shape}")
    B, H, N, d = q.shape
    nblk = (N + 127) // 128
    dev = v.codes.device
    for name, t in (("q", q), ("k", k)):
        if isinstance(t, Nvfp4Tensor):
            need = {"codes": B * H * N * d // 2, "block_sf": B * H * nblk * (d // 64) * 512, "tensor_scale": 1}
        else:
            need = {"codes": B * H * N * d, "scales": B * H * nblk}
        _check_buffers(name, t, need, dev)
    if isinstance(v, Nvfp4VTensor):
        need = {"codes": B * H * d * 64 * nblk, "block_sf": B * H * nblk * 1024, "tensor_scale": 1}
    else:
        need = {"codes": B * H * N * d, "scales": B * H * d}
    _check_buffers("v", v, need, dev)


def _check_buffers(name, t, need, dev) -> None:
    for field, n in need.items():
        buf = getattr(t, field)
        if not buf.is_cuda or buf.device != dev or not buf.is_contiguous():
            raise ValueError(f"{name}.{field}: expected a contiguous tensor on {dev}")
        if buf.numel() < n:
            raise ValueError(f"{name}.{field}: {buf.numel()} elements, the shape {tuple(t.shape)} needs {n}")


def attention_fwd(q, k, v, *, causal: bool = False, tile_mask: Optional[DeviceTileMask] = None,
                  softmax_scale: float = 0.0, out: Optional[torch.Tensor] = None,
                  lse: Optional[torch.Tensor] = None, return_lse: bool = True,
                  video: Optional[VideoLayout] = None, rescale_threshold: float = 0.0):
    """Fused attention on quantized operands.

    q, k: both Nvfp4Tensor or both Fp8Tensor (tile128); v: Fp8Tensor
    (channel), or Nvfp4VTensor for the all-NVFP4 attention (P and V in NVFP4).
    Returns (out bf16 [B,H,N,d], lse float32 [B,H,N] or None). With ``video``
    the operands are in tile-major order and out / lse come back in raster
    order. ``rescale_threshold`` (tau, log2 units, 0..8) skips the O / l
    rescale until a row's max has grown by more than tau; 0 is exact.
    """
    _check_operands(q, k, v)
    B, H, N, d = v.shape
    lib = library()
    if isinstance(v, Nvfp4VTensor):
        vd, v_scale, v_sf = _desc(v.codes, _lib.NVFP4, *v.shape), v.tensor_scale.data_ptr(), v.block_sf.data_ptr()
    else:
        vd, v_scale, v_sf = _desc(v.codes, _lib.E4M3, *v.shape), v.scales.data_ptr(), None
    if isinstance(q, Nvfp4Tensor):
        qd = _desc(q.codes, _lib.NVFP4, *q.shape)
        kd = _desc(k.codes, _lib.NVFP4, *k.shape)
        sc = _lib.Scales(q.tensor_scale.data_ptr(), k.tensor_scale.data_ptr(), v_scale,
                         q.block_sf.data_ptr(), k.block_sf.data_ptr(), 1.0 / 448.0, softmax_scale,
                         rescale_threshold, v_sf)
    else:
        qd = _desc(q.codes, _lib.E4M3, *q.shape)
        kd = _desc(k.codes, _lib.E4M3, *k.shape)
        sc = _lib.Scales(q.scales.data_ptr(), k.scales.data_ptr(), v_scale, None, None,
                         1.0 / 448.0, softmax_scale, rescale_threshold, v_sf)
    dev = v.codes.device
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev)
    if lse is None and return_lse:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    # the kernel writes every row of out and lse: a caller's buffers must hold them
    _aux(out, dev, torch.bfloat16, B * H * N * d, "out")
    _aux(lse, dev, torch.float32, B * H * N, "lse")
    mask = ctypes.byref(tile_mask.desc(dev)) if tile_mask is not None else None
    if video is None:
        st = lib.fpattn_fwd(ctypes.byref(qd), ctypes.byref(kd), ctypes.byref(vd), ctypes.byref(sc), mask,
                            1 if causal else 0, out.data_ptr(), _ptr(lse), _stream())
    else:
        st = lib.fpattn_fwd_video(ctypes.byref(qd), ctypes.byref(kd), ctypes.byref(vd), ctypes.byref(sc), mask,
                                  1 if causal else 0, _video_ref(video), out.data_ptr(), _ptr(lse), _stream())
    _lib.check(st, "fpattn_fwd" + ("_video" if video is not None else ""))
    return out, lse


def attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, qk_format: str = "nvfp4",
              causal: bool = False, tile_mask: Optional[DeviceTileMask] = None, softmax_scale: float = 0.0,
              return_lse: bool = True, device: Optional[torch.device] = None,
              out_host: Optional[torch.Tensor] = None, lse_host: Optional[torch.Tensor] = None,
              video: Optional[VideoLayout] = None, rescale_threshold: float = 0.0,
              qk_group_tiles: int = 1, pv_format: str = "fp8", host_chunks: Optional[int] = None,
              qk_amax: Optional[Tuple[torch.Tensor, torch.Tensor]] = None):
    """softmax(Q K^T * scale) V with quantized operands, from bf16 inputs.

    ``qk_group_tiles`` > 1 (FP8 Q/K only) shares one Q/K scale across that
    many consecutive 128-token tiles (the coarser granularities of the
    denoising-step schedule). ``pv_format="nvfp4"`` quantizes P and V to
    NVFP4 and runs P V on the block-scaled FP4 tensor cores.

    CUDA inputs stay where they are. Host inputs (ideally pinned) are copied
    to ``device`` (default cuda:0) and the output (and lse) copied back to
    host memory, into ``out_host`` / ``lse_host`` when given (pinned buffers
    the caller reuses), else into new pinned tensors; the copies of one group
    of heads overlap the kernels of another (see _attention_host), and the
    call returns once the results are in host memory. ``host_chunks`` sets
    the number of head groups of that pipeline (default: about 8 MiB of V a
    group, at most 16); the results do not depend on it.

    ``qk_amax`` (NVFP4 Q/K only): device float32 [1] tensors with the amax of
    Q and of K, e.g. from calibration or ``tensor_amax``, used for the tensor
    scales instead of the amax of these inputs (the static-amax form of the
    NVFP4 recipe). With it, host inputs are quantized group by group as they
    land, so the copies back start before all of Q and K are in.
    """
    if qk_format not in ("nvfp4", "fp8"):
        raise ValueError("qk_format must be 'nvfp4' or 'fp8'")
    if pv_format not in ("fp8", "nvfp4"):
        raise ValueError("pv_format must be 'fp8' or 'nvfp4'")
    if qk_amax is not None:
        if qk_format != "nvfp4":
            raise ValueError("qk_amax applies to NVFP4 Q/K only")
        if len(qk_amax) != 2 or not all(isinstance(a, torch.Tensor) and a.is_cuda and a.dtype == torch.float32
                                        and a.numel() >= 1 for a in qk_amax):
            raise ValueError("qk_amax must be two CUDA float32 tensors (amax of Q, amax of K)")
    if not q.is_cuda:
        return _attention_host(q, k, v, qk_format=qk_format, causal=causal, tile_mask=tile_mask,
                               softmax_scale=softmax_scale, return_lse=return_lse, device=device,
                               out_host=out_host, lse_host=lse_host, video=video,
                               rescale_threshold=rescale_threshold, qk_group_tiles=qk_group_tiles,
                               pv_format=pv_format, chunks=host_chunks, qk_amax=qk_amax)
    if qk_format not in ("nvfp4", "fp8"):
        raise ValueError("qk_format must be 'nvfp4' or 'fp8'")
    if pv_format not in ("fp8", "nvfp4"):
        raise ValueError("pv_format must be 'fp8' or 'nvfp4'")
    if pv_format == "fp8" and qk_group_tiles <= 1 and qk_amax is None:
        qq, kq, vq = quantize_qkv(q, k, v, qk_format, video=video)   # four fused launches
    else:
        if qk_format == "nvfp4":
            aq, ak = qk_amax if qk_amax is not None else (None, None)
            qq, kq = quantize_nvfp4(q, static_amax=aq, video=video), quantize_nvfp4(k, static_amax=ak, video=video)
        else:
            gran = "group" if qk_group_tiles > 1 else "tile128"
            qq = quantize_fp8(q, gran, video=video, group_tiles=qk_group_tiles)
            kq = quantize_fp8(k, gran, video=video, group_tiles=qk_group_tiles)
        vq = quantize_fp8(v, "channel", video=video) if pv_format == "fp8" else quantize_nvfp4_v(v, video=video)
    return attention_fwd(qq, kq, vq, causal=causal, tile_mask=tile_mask, softmax_scale=softmax_scale,
                         return_lse=return_lse, video=video, rescale_threshold=rescale_threshold)


_COPY_STREAMS = {}


def _copy_streams(dev: torch.device):
    """The host pipeline's two copy streams of a device, created once: every
    call orders them after the caller's stream itself, so reusing them adds
    no dependency between calls beyond the caller's own stream order."""
    key = dev.index if dev.index is not None else torch.cuda.current_device()
    if key not in _COPY_STREAMS:
        _COPY_STREAMS[key] = (torch.cuda.Stream(dev), torch.cuda.Stream(dev))
    return _COPY_STREAMS[key]


def _attention_host(q, k, v, *, qk_format, causal, tile_mask, softmax_scale, return_lse, device, out_host,
                    lse_host, video, rescale_threshold, qk_group_tiles, pv_format, chunks: Optional[int] = None,
                    qk_amax=None):
    """attention() for host inputs: the (batch, head) problems are split into
    ``chunks`` contiguous groups, and the copies in, the kernels and the
    copies out of different groups overlap on three streams. Q and K are
    copied first: an NVFP4 tensor scale needs the amax over every head, so
    their amax pass runs as each group lands, and every group's Q and K are
    quantized as soon as the amax is complete (the bits of the one-shot
    call). V is copied after them, group by group, and each group's V
    quantize + attention + copy back starts as soon as its V has landed; the
    copies back then run while the rest of V comes in, so small groups keep
    the tail after the last input byte short. With FP8 Q/K and V, or a
    caller's Q/K amax (no tensor-wide amax to wait for), each group's Q, K, V
    are copied together and the group is quantized as it lands. By default a
    group holds about 8 MiB of V (at most 16 groups): enough groups to keep
    the tail short, few enough that the host's enqueue work stays hidden
    behind the Q/K copies."""
    dev = torch.device(device or "cuda:0")
    B, H, N, d = q.shape
    if tuple(k.shape) != (B, H, N, d) or tuple(v.shape) != (B, H, N, d):
        raise ValueError("q, k, v must have one shape")
    BH = B * H
    if chunks is None:
        chunks = max(1, min(16, (BH * N * d * 2) >> 23))
    chunks = max(1, min(int(chunks), BH))
    spans = [s for s in (head_range(BH, chunks, r) for r in range(chunks)) if s[1] > s[0]]
    flat = [t.reshape(BH, N, d) for t in (q, k, v)]
    cur = torch.cuda.current_stream(dev)
    s_in, s_out = _copy_streams(dev)
    qd, kd, vd = (torch.empty((BH, N, d), dtype=torch.bfloat16, device=dev) for _ in range(3))
    out_d = torch.empty((BH, N, d), dtype=torch.bfloat16, device=dev)
    lse_d = torch.empty((BH, N), dtype=torch.float32, device=dev) if return_lse else None
    out_h = out_host if out_host is not None else torch.empty((B, H, N, d), dtype=torch.bfloat16, pin_memory=True)
    lse_h = None
    if return_lse:
        lse_h = lse_host if lse_host is not None else torch.empty((B, H, N), dtype=torch.float32, pin_memory=True)
    out_hf, lse_hf = out_h.view(BH, N, d), (lse_h.view(BH, N) if lse_h is not None else None)
    s_in.wait_stream(cur)     # the device buffers were allocated on the current stream
    ev_qk, ev_v = [torch.cuda.Event() for _ in spans], [torch.cuda.Event() for _ in spans]
    # with no tensor-wide amax to wait for (FP8 Q/K and V), group i's Q, K, V
    # are copied together so its kernels can start right after them
    interleave = pv_format == "fp8" and (qk_format == "fp8" or qk_amax is not None)
    with torch.cuda.stream(s_in):
        for i, (a, b) in enumerate(spans):
            qd[a:b].copy_(flat[0][a:b], non_blocking=True)
            kd[a:b].copy_(flat[1][a:b], non_blocking=True)
            ev_qk[i].record(s_in)
            if interleave:
                vd[a:b].copy_(flat[2][a:b], non_blocking=True)
                ev_v[i].record(s_in)
        if not interleave:
            for i, (a, b) in enumerate(spans):
                vd[a:b].copy_(flat[2][a:b], non_blocking=True)
                ev_v[i].record(s_in)

    def part(t, a, b):
        return t[a:b].view(1, b - a, N, d)

    amax_q = amax_k = amax_v = None
    if qk_amax is not None:
        amax_q, amax_k = (a.to(dev) for a in qk_amax)
    elif qk_format == "nvfp4":
        amax_q, amax_k = (torch.empty(1, dtype=torch.float32, device=dev) for _ in range(2))
        for i, (a, b) in enumerate(spans):
            cur.wait_event(ev_qk[i])
            tensor_amax(part(qd, a, b), amax_q, accumulate=i > 0)
            tensor_amax(part(kd, a, b), amax_k, accumulate=i > 0)
    if pv_format == "nvfp4":
        amax_v = torch.empty(1, dtype=torch.float32, device=dev)
        for i, (a, b) in enumerate(spans):
            cur.wait_event(ev_v[i])
            tensor_amax(part(vd, a, b), amax_v, accumulate=i > 0)
    s_out.wait_stream(cur)

    def quantize_qk(i, a, b):
        qc, kc = part(qd, a, b), part(kd, a, b)
        if qk_format == "nvfp4":
            return (quantize_nvfp4(qc, static_amax=amax_q, video=video),
                    quantize_nvfp4(kc, static_amax=amax_k, video=video))
        gran = "group" if qk_group_tiles > 1 else "tile128"
        return (quantize_fp8(qc, gran, video=video, group_tiles=qk_group_tiles),
                quantize_fp8(kc, gran, video=video, group_tiles=qk_group_tiles))

    # with a tensor-wide Q/K amax every group's Q/K can be quantized as soon
    # as the amax is done, ahead of the V copies; otherwise group by group
    qk_ready = ([quantize_qk(i, a, b) for i, (a, b) in enumerate(spans)]
                if qk_format == "nvfp4" and qk_amax is None else None)
    for i, (a, b) in enumerate(spans):
        cur.wait_event(ev_qk[i])
        cur.wait_event(ev_v[i])
        qq, kq = qk_ready[i] if qk_ready is not None else quantize_qk(i, a, b)
        vc = part(vd, a, b)
        if pv_format == "fp8":
            vq = quantize_fp8(vc, "channel", video=video)
        else:
            vq = quantize_nvfp4_v(vc, static_amax=amax_v, video=video)
        attention_fwd(qq, kq, vq, causal=causal, tile_mask=tile_mask, softmax_scale=softmax_scale,
                      out=out_d[a:b].view(1, b - a, N, d),
                      lse=None if lse_d is None else lse_d[a:b].view(1, b - a, N), return_lse=return_lse,
                      video=video, rescale_threshold=rescale_threshold)
        done = torch.cuda.Event()
        done.record(cur)
        s_out.wait_event(done)
        with torch.cuda.stream(s_out):
            out_hf[a:b].copy_(out_d[a:b], non_blocking=True)
            if lse_hf is not None:
                lse_hf[a:b].copy_(lse_d[a:b], non_blocking=True)
    cur.wait_stream(s_out)
    for t in (qd, kd, vd, out_d) + ((lse_d,) if lse_d is not None else ()):
        t.record_stream(s_in)
        t.record_stream(s_out)
    cur.synchronize()
    return out_h, lse_h


def attention_sharded(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, group=None,
                      qk_format: str = "nvfp4", **kwargs):
    """attention() on this rank's share of one batch's (batch, head)
    problems (device bf16 [B_r, H_r, N, d], e.g. the heads head_range gives
    the rank), with P and V in FP8. NVFP4 Q/K take their tensor scale from
    the amax of the whole batch: the ranks' Q and K amax (two floats) are
    max-reduced over ``group`` (torch.distributed) before quantizing, so every
    share is quantized exactly as the whole batch would be. FP8 Q/K and V
    have per-head scales and need no exchange. Every rank of the group must
    call it, with its own share."""
    import torch.distributed as dist
    if kwargs.get("pv_format", "fp8") != "fp8":
        raise ValueError("attention_sharded takes FP8 P/V (an NVFP4 V would need its tensor amax too)")
    if qk_format != "nvfp4":
        return attention(q, k, v, qk_format=qk_format, **kwargs)
    _check_bf16(q)
    _check_bf16(k)
    amax = torch.cat([tensor_amax(q), tensor_amax(k)])
    if dist.get_backend(group) == "gloo":
        host = amax.cpu()
        dist.all_reduce(host, op=dist.ReduceOp.MAX, group=group)
        amax = host.to(q.device)
    else:
        dist.all_reduce(amax, op=dist.ReduceOp.MAX, group=group)
    return attention(q, k, v, qk_format="nvfp4", qk_amax=(amax[0:1], amax[1:2]), **kwargs)


def head_range(num_heads: int, world: int, rank: int) -> Tuple[int, int]:
    """Rank ``rank``'s share [start, stop) of ``num_heads`` independent
    (batch, head) problems split over ``world`` ranks: contiguous ranges in
    rank order, the first ``num_heads % world`` ranks taking one more. The
    flattened [B*H, N, d] view of a contiguous [B, H, N, d] tensor makes each
    share one contiguous slice."""
    if world < 1 or not 0 <= rank < world or num_heads < 0:
        raise ValueError("need world >= 1, 0 <= rank < world, num_heads >= 0")
    base, extra = divmod(num_heads, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def device_error(clear: bool = True) -> int:
    """Raw device error word (0 = no bounded wait expired). Synchronizes."""
    code = ctypes.c_int32(0)
    library().fpattn_device_error(_stream(), 1 if clear else 0, ctypes.byref(code))
    return code.value
