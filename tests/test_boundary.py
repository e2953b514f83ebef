"""C-ABI boundary checks that need no GPU.

* libfpattn.so loads and exports every function include/fpattn.h declares.
* Argument errors are returned synchronously, before any CUDA call.
* The host-only sliding-tile planner matches the oracle's block lists.
"""
import ctypes
import os
import re

import numpy as np
import pytest

import precision_attention_nvfp4_b200 as fp
from precision_attention_nvfp4_b200 import _lib
from oracle import sta

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    with open(os.path.join(ROOT, "include", "fpattn.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fpattn_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from precision_attention_nvfp4_b200 import build
    build.build()
    return fp.library()


def test_exports_every_declared_symbol(lib):
    names = _declared_functions()
    assert "fpattn_fwd" in names and "fpattn_quantize_nvfp4" in names and "fpattn_quantize_fp8" in names
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings_and_version(lib):
    assert lib.fpattn_status_string(_lib.OK) == b"ok"
    assert b"aligned" in lib.fpattn_status_string(_lib.ERR_ALIGNMENT)
    assert lib.fpattn_version().startswith(b"fpattn")


def test_sf_bytes(lib):
    assert lib.fpattn_nvfp4_sf_bytes(4, 32, 4096, 128) == 4 * 32 * 32 * 2 * 512
    assert lib.fpattn_nvfp4_sf_bytes(1, 1, 129, 64) == 2 * 512
    assert lib.fpattn_nvfp4_sf_bytes(1, 1, 0, 64) == 0


def _t(ptr, dtype, B=1, H=1, N=128, d=128):
    return _lib.Tensor(ptr, dtype, B, H, N, d)


def test_quantize_argument_errors(lib):
    buf = (ctypes.c_uint8 * 4096)()
    p = ctypes.addressof(buf)
    p16 = (p + 15) & ~15
    good = _t(p16, _lib.BF16)
    # null input / outputs
    assert lib.fpattn_quantize_fp8(None, 0, p16, p16, None, None) == _lib.ERR_INVALID_ARG
    assert lib.fpattn_quantize_fp8(ctypes.byref(good), 0, None, p16, None, None) == _lib.ERR_INVALID_ARG
    assert lib.fpattn_quantize_fp8(ctypes.byref(good), 7, p16, p16, None, None) == _lib.ERR_INVALID_ARG
    # wrong dtype, bad head size, bad shape, misalignment
    assert lib.fpattn_quantize_fp8(ctypes.byref(_t(p16, _lib.E4M3)), 0, p16, p16, None, None) == _lib.ERR_INVALID_ARG
    assert lib.fpattn_quantize_fp8(ctypes.byref(_t(p16, _lib.BF16, d=96)), 0, p16, p16, None, None) == _lib.ERR_UNSUPPORTED
    assert lib.fpattn_quantize_fp8(ctypes.byref(_t(p16, _lib.BF16, N=0)), 0, p16, p16, None, None) == _lib.ERR_INVALID_ARG
    assert lib.fpattn_quantize_fp8(ctypes.byref(_t(p16 + 2, _lib.BF16)), 0, p16, p16, None, None) == _lib.ERR_ALIGNMENT
    assert lib.fpattn_quantize_nvfp4(ctypes.byref(good), None, p16 + 8, p16, p16, None, None) == _lib.ERR_ALIGNMENT
    assert lib.fpattn_quantize_nvfp4(ctypes.byref(good), None, p16, None, p16, None, None) == _lib.ERR_INVALID_ARG


def test_fwd_argument_errors(lib):
    buf = (ctypes.c_uint8 * 4096)()
    p16 = (ctypes.addressof(buf) + 15) & ~15
    q = _t(p16, _lib.E4M3)
    v = _t(p16, _lib.E4M3)
    sc = _lib.Scales(p16, p16, p16, None, None, 1.0 / 448.0, 0.0)
    ok_args = (ctypes.byref(q), ctypes.byref(q), ctypes.byref(v), ctypes.byref(sc), None, 0, p16, None, None)
    bad_p = _lib.Scales(p16, p16, p16, None, None, 1.0 / 256.0, 0.0)
    assert lib.fpattn_fwd(ctypes.byref(q), ctypes.byref(q), ctypes.byref(v), ctypes.byref(bad_p), None, 0, p16,
                          None, None) == _lib.ERR_INVALID_ARG
    # NVFP4 q/k without block scales
    q4 = _t(p16, _lib.NVFP4)
    assert lib.fpattn_fwd(ctypes.byref(q4), ctypes.byref(q4), ctypes.byref(v), ctypes.byref(sc), None, 0, p16,
                          None, None) == _lib.ERR_INVALID_ARG
    # mismatched shapes, mixed q/k dtypes, bf16 v, bad d
    k2 = _t(p16, _lib.E4M3, N=256)
    assert lib.fpattn_fwd(ctypes.byref(q), ctypes.byref(k2), *ok_args[2:]) == _lib.ERR_INVALID_ARG
    assert lib.fpattn_fwd(ctypes.byref(q), ctypes.byref(q4), *ok_args[2:]) == _lib.ERR_INVALID_ARG
    vb = _t(p16, _lib.BF16)
    assert lib.fpattn_fwd(ctypes.byref(q), ctypes.byref(q), ctypes.byref(vb), *ok_args[3:]) == _lib.ERR_INVALID_ARG
    qbad = _t(p16, _lib.E4M3, d=32)
    assert lib.fpattn_fwd(ctypes.byref(qbad), ctypes.byref(qbad), ctypes.byref(qbad), *ok_args[3:]) == _lib.ERR_UNSUPPORTED
    qbf = _t(p16, _lib.BF16)
    assert lib.fpattn_fwd(ctypes.byref(qbf), ctypes.byref(qbf), *ok_args[2:]) == _lib.ERR_UNSUPPORTED
    # misaligned output, tile mask of the wrong size
    assert lib.fpattn_fwd(*ok_args[:6], p16 + 4, None, None) == _lib.ERR_ALIGNMENT
    tm = _lib.TileMask(5, 0, p16, p16, None)
    assert lib.fpattn_fwd(*ok_args[:4], ctypes.byref(tm), 0, p16, None, None) == _lib.ERR_INVALID_ARG


@pytest.mark.parametrize("grid,tile,window", [
    ((18, 48, 80), (6, 8, 8), (3, 3, 5)),
    ((12, 16, 24), (6, 8, 8), (3, 3, 5)),
    ((8, 16, 16), (4, 8, 8), (1, 3, 3)),
    ((6, 32, 32), (6, 16, 16), (3, 1, 1)),
])
def test_sta_planner_matches_oracle(lib, grid, tile, window):
    tg = tuple(g // t for g, t in zip(grid, tile))
    plan = fp.sta_plan(tg, tile, window)
    ref = sta.block_lists(grid, tile, window)
    assert plan.nblk == len(ref)
    for qb, kbs in enumerate(ref):
        assert list(plan.col_idx[plan.row_ptr[qb]:plan.row_ptr[qb + 1]]) == kbs
    lens = np.diff(plan.row_ptr)
    assert sorted(plan.row_order.tolist()) == list(range(plan.nblk))
    assert np.all(np.diff(lens[plan.row_order]) <= 0)


def test_sta_planner_rejects_unaligned_tiles(lib):
    nb, nz = ctypes.c_int32(0), ctypes.c_int32(0)
    st = lib.fpattn_sta_plan(3, 6, 10, 5, 8, 8, 3, 3, 5, None, None, None, 0, ctypes.byref(nb), ctypes.byref(nz))
    assert st == _lib.ERR_UNSUPPORTED
    st = lib.fpattn_sta_plan(3, 6, 10, 6, 8, 8, 0, 3, 5, None, None, None, 0, ctypes.byref(nb), ctypes.byref(nz))
    assert st == _lib.ERR_INVALID_ARG


def test_library_missing_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "nope.so"))
    with pytest.raises(RuntimeError, match="not built"):
        _lib.load()
