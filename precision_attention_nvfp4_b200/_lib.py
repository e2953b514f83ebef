"""ctypes declarations of the C ABI in include/fpattn.h (argument marshalling only)."""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfpattn.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_ALIGNMENT, ERR_CUDA, ERR_TIMEOUT = range(6)
BF16, E4M3, NVFP4 = 0, 1, 2
FP8_TILE128, FP8_CHANNEL = 0, 1


class Tensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("B", ctypes.c_int32),
                ("H", ctypes.c_int32), ("N", ctypes.c_int32), ("d", ctypes.c_int32)]


class Scales(ctypes.Structure):
    _fields_ = [("q_scale", ctypes.c_void_p), ("k_scale", ctypes.c_void_p), ("v_scale", ctypes.c_void_p),
                ("q_block_sf", ctypes.c_void_p), ("k_block_sf", ctypes.c_void_p),
                ("p_scale", ctypes.c_float), ("softmax_scale", ctypes.c_float),
                ("rescale_threshold", ctypes.c_float), ("v_block_sf", ctypes.c_void_p)]


class TileMask(ctypes.Structure):
    _fields_ = [("nblk_q", ctypes.c_int32), ("nnz", ctypes.c_int32), ("row_ptr", ctypes.c_void_p),
                ("col_idx", ctypes.c_void_p), ("row_order", ctypes.c_void_p)]


class VideoLayout(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("Hs", ctypes.c_int32), ("W", ctypes.c_int32),
                ("tt", ctypes.c_int32), ("th", ctypes.c_int32), ("tw", ctypes.c_int32)]


_P = ctypes.POINTER
_SIGNATURES = {
    "fpattn_nvfp4_sf_bytes": (ctypes.c_size_t, [ctypes.c_int32] * 4),
    "fpattn_quantize_nvfp4": (ctypes.c_int, [_P(Tensor), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                             ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "fpattn_quantize_fp8": (ctypes.c_int, [_P(Tensor), ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
                                           ctypes.c_void_p, ctypes.c_void_p]),
    "fpattn_video_layout_check": (ctypes.c_int, [_P(VideoLayout), ctypes.c_int32]),
    "fpattn_quantize_nvfp4_video": (ctypes.c_int, [_P(Tensor), _P(VideoLayout), ctypes.c_void_p, ctypes.c_void_p,
                                                   ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                                   ctypes.c_void_p]),
    "fpattn_quantize_fp8_video": (ctypes.c_int, [_P(Tensor), _P(VideoLayout), ctypes.c_int32, ctypes.c_void_p,
                                                 ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "fpattn_nvfp4_v_bytes": (ctypes.c_size_t, [ctypes.c_int32] * 4 + [_P(ctypes.c_size_t)]),
    "fpattn_quantize_nvfp4_v": (ctypes.c_int, [_P(Tensor), _P(VideoLayout), ctypes.c_void_p, ctypes.c_void_p,
                                               ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "fpattn_quantize_fp8_group": (ctypes.c_int, [_P(Tensor), _P(VideoLayout), ctypes.c_int32, ctypes.c_void_p,
                                                 ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "fpattn_quantize_qkv": (ctypes.c_int, [_P(Tensor), _P(Tensor), _P(Tensor), ctypes.c_int32, _P(VideoLayout)] +
                            [ctypes.c_void_p] * 10),
    "fpattn_tensor_amax": (ctypes.c_int, [_P(Tensor), ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
                                          ctypes.c_void_p]),
    "fpattn_step_phase": (ctypes.c_int, [ctypes.c_int32, ctypes.c_int32, ctypes.c_double, ctypes.c_double,
                                         _P(ctypes.c_int32)]),
    "fpattn_sta_plan": (ctypes.c_int, [ctypes.c_int32] * 9 + [ctypes.c_void_p] * 3 +
                        [ctypes.c_size_t, _P(ctypes.c_int32), _P(ctypes.c_int32)]),
    "fpattn_causal_plan": (ctypes.c_int, [ctypes.c_int64, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                          ctypes.c_int32, ctypes.c_int32] + [_P(ctypes.c_int32)] * 5),
    "fpattn_tile_mask_check": (ctypes.c_int, [ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
                                              ctypes.c_void_p]),
    "fpattn_fwd": (ctypes.c_int, [_P(Tensor), _P(Tensor), _P(Tensor), _P(Scales), _P(TileMask),
                                  ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "fpattn_fwd_video": (ctypes.c_int, [_P(Tensor), _P(Tensor), _P(Tensor), _P(Scales), _P(TileMask),
                                        ctypes.c_int32, _P(VideoLayout), ctypes.c_void_p, ctypes.c_void_p,
                                        ctypes.c_void_p]),
    "fpattn_device_error": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int32, _P(ctypes.c_int32)]),
    "fpattn_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "fpattn_version": (ctypes.c_char_p, []),
}

_lib = None


def load() -> ctypes.CDLL:
    """Load libfpattn.so (built in-tree). Raises if it is missing: there is no
    fallback implementation."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"fpattn CUDA library not built: {LIB_PATH} is missing "
                               "(run python -m precision_attention_nvfp4_b200.build)")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


class FpattnError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = load().fpattn_status_string(status).decode()
        super().__init__(f"{where}: {msg} (status {status})")
        self.status = status


def check(status: int, where: str) -> None:
    if status != OK:
        raise FpattnError(status, where)
