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
import torch

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
    for tau in (-0.5, 8.5, float("nan"), float("inf")):
        bad_tau = _lib.Scales(p16, p16, p16, None, None, 1.0 / 448.0, 0.0, tau)
        assert lib.fpattn_fwd(ctypes.byref(q), ctypes.byref(q), ctypes.byref(v), ctypes.byref(bad_tau), None, 0,
                              p16, None, None) == _lib.ERR_INVALID_ARG
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
    # rows of equal length keep their index order (a stable longest-first sort)
    order = plan.row_order.tolist()
    assert order == sorted(range(plan.nblk), key=lambda r: (-lens[r], r))


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


def _chunks_are_boxes(grid, tile):
    """Brute force on the oracle's permutation: every 32 consecutive
    tile-major tokens fill an axis-aligned box of the grid in raster order,
    and no 128-token block crosses a tile."""
    if (tile[0] * tile[1] * tile[2]) % 128:
        return False
    perm = sta.raster_index_of_tile_major(grid, tile)
    T, Hs, W = grid
    t, h, w = perm // (Hs * W), (perm // W) % Hs, perm % W
    for i0 in range(0, len(perm), 32):
        sl = slice(i0, i0 + 32)
        ext = [(a.max() - a.min() + 1) for a in (t[sl], h[sl], w[sl])]
        if ext[0] * ext[1] * ext[2] != 32:
            return False
        # the box in raster order is what a 3D box copy reads or writes
        tt, hh, ww = np.meshgrid(np.arange(t[sl].min(), t[sl].min() + ext[0]),
                                 np.arange(h[sl].min(), h[sl].min() + ext[1]),
                                 np.arange(w[sl].min(), w[sl].min() + ext[2]), indexing="ij")
        if not np.array_equal((tt * Hs + hh) * W + ww, perm[sl].reshape(ext)):
            return False
    return True


@pytest.mark.parametrize("tile", [(6, 8, 8), (4, 8, 8), (6, 16, 16), (2, 4, 16), (1, 4, 32), (2, 8, 8),
                                  (4, 4, 8), (8, 2, 8), (1, 2, 64), (2, 16, 4), (6, 12, 8), (3, 8, 8),
                                  (2, 2, 32), (4, 4, 4), (1, 1, 128), (2, 8, 16), (4, 8, 4), (2, 32, 2),
                                  (8, 3, 16), (16, 1, 24), (4, 2, 48), (2, 6, 32)])
def test_video_layout_rule_matches_bruteforce(lib, tile):
    grid = (tile[0] * 2, tile[1] * 2, tile[2] * 3)
    N = grid[0] * grid[1] * grid[2]
    lay = _lib.VideoLayout(*grid, *tile)
    st = lib.fpattn_video_layout_check(ctypes.byref(lay), N)
    assert st in (_lib.OK, _lib.ERR_UNSUPPORTED)
    assert (st == _lib.OK) == _chunks_are_boxes(grid, tile)


def test_video_argument_errors(lib):
    buf = (ctypes.c_uint8 * 4096)()
    p16 = (ctypes.addressof(buf) + 15) & ~15
    good = _lib.VideoLayout(1, 8, 16, 1, 8, 16)          # N = 128
    assert lib.fpattn_video_layout_check(ctypes.byref(good), 128) == _lib.OK
    assert lib.fpattn_video_layout_check(None, 128) == _lib.ERR_INVALID_ARG
    assert lib.fpattn_video_layout_check(ctypes.byref(good), 256) == _lib.ERR_INVALID_ARG
    assert lib.fpattn_video_layout_check(ctypes.byref(_lib.VideoLayout(1, 8, 16, 1, 0, 16)), 128) == _lib.ERR_INVALID_ARG
    ragged = _lib.VideoLayout(1, 8, 16, 1, 3, 16)         # Hs not a multiple of th
    assert lib.fpattn_video_layout_check(ctypes.byref(ragged), 128) == _lib.ERR_UNSUPPORTED
    x = _t(p16, _lib.BF16, N=128)
    for ok in [(1, 4, 32, 1, 4, 32),     # a chunk is one w-row of 32
               (1, 16, 8, 1, 16, 8),     # a chunk is 4 w-rows of 8
               (1, 1, 128, 1, 1, 128),   # a chunk is a quarter w-row
               (1, 2, 64, 1, 2, 64)]:    # a chunk is half a w-row
        assert lib.fpattn_video_layout_check(ctypes.byref(_lib.VideoLayout(*ok)), 128) == _lib.OK
    rej = _lib.VideoLayout(3, 8, 8, 3, 8, 8)              # tile volume 192: not a multiple of 128
    assert lib.fpattn_video_layout_check(ctypes.byref(rej), 192) == _lib.ERR_UNSUPPORTED
    # the entry points reject before any CUDA call
    assert lib.fpattn_quantize_fp8_video(ctypes.byref(x), None, 0, p16, p16, None, None) == _lib.ERR_INVALID_ARG
    assert lib.fpattn_quantize_fp8_video(ctypes.byref(x), ctypes.byref(ragged), 0, p16, p16, None,
                                         None) == _lib.ERR_UNSUPPORTED
    assert lib.fpattn_quantize_nvfp4_video(ctypes.byref(x), ctypes.byref(ragged), None, p16, p16, p16, None,
                                           None) == _lib.ERR_UNSUPPORTED
    assert lib.fpattn_quantize_nvfp4_video(ctypes.byref(x), None, None, p16, p16, p16, None,
                                           None) == _lib.ERR_INVALID_ARG
    q = _t(p16, _lib.E4M3, N=128)
    sc = _lib.Scales(p16, p16, p16, None, None, 1.0 / 448.0, 0.0)
    assert lib.fpattn_fwd_video(ctypes.byref(q), ctypes.byref(q), ctypes.byref(q), ctypes.byref(sc), None, 0,
                                None, p16, None, None) == _lib.ERR_INVALID_ARG
    assert lib.fpattn_fwd_video(ctypes.byref(q), ctypes.byref(q), ctypes.byref(q), ctypes.byref(sc), None, 0,
                                ctypes.byref(rej), p16, None, None) == _lib.ERR_INVALID_ARG
    assert lib.fpattn_fwd_video(ctypes.byref(q), ctypes.byref(q), ctypes.byref(q), ctypes.byref(sc), None, 0,
                                ctypes.byref(ragged), p16, None, None) == _lib.ERR_UNSUPPORTED


def test_step_phase_matches_oracle(lib):
    from oracle import schedule
    ph = ctypes.c_int32(-1)
    cases = [(t, D, a1, a2) for D in (1, 7, 10, 49, 50, 1000) for t in sorted({1, 2, D // 5, D // 5 + 1, D // 2,
                                                                               (7 * D) // 10, (7 * D) // 10 + 1,
                                                                               D - 1, D} - {0})
             for a1, a2 in ((0.2, 0.7), (0.0, 1.0), (0.5, 0.5), (0.1, 0.3), (1 / 3, 2 / 3))]
    for t, D, a1, a2 in cases:
        if not 1 <= t <= D:
            continue
        assert lib.fpattn_step_phase(t, D, a1, a2, ctypes.byref(ph)) == _lib.OK
        assert ph.value == schedule.step_phase(t, D, a1, a2), (t, D, a1, a2)
    for bad in ((0, 10, 0.2, 0.7), (11, 10, 0.2, 0.7), (1, 0, 0.2, 0.7), (1, 10, 0.8, 0.7),
                (1, 10, -0.1, 0.7), (1, 10, 0.2, 1.5), (1, 10, float("nan"), 0.7)):
        assert lib.fpattn_step_phase(*bad, ctypes.byref(ph)) == _lib.ERR_INVALID_ARG, bad
    assert lib.fpattn_step_phase(1, 10, 0.2, 0.7, None) == _lib.ERR_INVALID_ARG


def test_quantize_fp8_group_argument_errors(lib):
    buf = (ctypes.c_uint8 * 4096)()
    p16 = (ctypes.addressof(buf) + 15) & ~15
    x = _t(p16, _lib.BF16)
    assert lib.fpattn_quantize_fp8_group(ctypes.byref(x), None, 0, p16, p16, None, None) == _lib.ERR_INVALID_ARG
    assert lib.fpattn_quantize_fp8_group(ctypes.byref(x), None, 2, None, p16, None, None) == _lib.ERR_INVALID_ARG
    assert lib.fpattn_quantize_fp8_group(ctypes.byref(x), None, 2, p16 + 4, p16, None, None) == _lib.ERR_ALIGNMENT
    assert lib.fpattn_quantize_fp8_group(ctypes.byref(_t(p16, _lib.BF16, d=96)), None, 2, p16, p16, None,
                                         None) == _lib.ERR_UNSUPPORTED
    ragged = _lib.VideoLayout(1, 8, 16, 1, 3, 16)
    assert lib.fpattn_quantize_fp8_group(ctypes.byref(x), ctypes.byref(ragged), 2, p16, p16, None,
                                         None) == _lib.ERR_UNSUPPORTED


def test_nvfp4_v_sizes_and_argument_errors(lib):
    sf = ctypes.c_size_t(0)
    assert lib.fpattn_nvfp4_v_bytes(2, 3, 300, 128, ctypes.byref(sf)) == 2 * 3 * 128 * 3 * 64
    assert sf.value == 2 * 3 * 3 * 1024
    assert lib.fpattn_nvfp4_v_bytes(1, 1, 0, 64, ctypes.byref(sf)) == 0 and sf.value == 0
    buf = (ctypes.c_uint8 * 4096)()
    p16 = (ctypes.addressof(buf) + 15) & ~15
    x = _t(p16, _lib.BF16)
    assert lib.fpattn_quantize_nvfp4_v(ctypes.byref(x), None, None, None, p16, p16, None, None) == _lib.ERR_INVALID_ARG
    assert lib.fpattn_quantize_nvfp4_v(ctypes.byref(x), None, None, p16 + 8, p16, p16, None,
                                       None) == _lib.ERR_ALIGNMENT
    assert lib.fpattn_quantize_nvfp4_v(ctypes.byref(_t(p16, _lib.BF16, d=48)), None, None, p16, p16, p16, None,
                                       None) == _lib.ERR_UNSUPPORTED
    # an NVFP4 V needs its block scales
    q = _t(p16, _lib.E4M3)
    v4 = _t(p16, _lib.NVFP4)
    sc = _lib.Scales(p16, p16, p16, None, None, 1.0 / 448.0, 0.0, 0.0, None)
    assert lib.fpattn_fwd(ctypes.byref(q), ctypes.byref(q), ctypes.byref(v4), ctypes.byref(sc), None, 0, p16, None,
                          None) == _lib.ERR_INVALID_ARG
    sc_bad = _lib.Scales(p16, p16, p16, None, None, 1.0 / 448.0, 0.0, 0.0, p16 + 4)
    assert lib.fpattn_fwd(ctypes.byref(q), ctypes.byref(q), ctypes.byref(v4), ctypes.byref(sc_bad), None, 0, p16,
                          None, None) == _lib.ERR_ALIGNMENT


def _mask_status(lib, row_ptr, col_idx, row_order=None, nblk=None):
    rp = np.asarray(row_ptr, dtype=np.int32)
    ci = np.asarray(col_idx, dtype=np.int32)
    ro = None if row_order is None else np.asarray(row_order, dtype=np.int32)
    n = len(rp) - 1 if nblk is None else nblk
    return lib.fpattn_tile_mask_check(n, len(ci), rp.ctypes.data, ci.ctypes.data if len(ci) else None,
                                      None if ro is None else ro.ctypes.data)


def test_tile_mask_check_accepts_wellformed(lib):
    assert _mask_status(lib, [0, 2, 2, 3], [0, 2, 1], [0, 2, 1]) == _lib.OK
    assert _mask_status(lib, [0, 2, 2, 3], [0, 2, 1]) == _lib.OK        # row_order optional
    plan = fp.sta_plan((3, 6, 10), (6, 8, 8), (3, 3, 5))
    assert _mask_status(lib, plan.row_ptr, plan.col_idx, plan.row_order) == _lib.OK


@pytest.mark.parametrize("row_ptr,col_idx,row_order", [
    ([0, 2, 2, 3], [0, 3, 1], None),          # key block 3 >= nblk
    ([0, 2, 2, 3], [0, -1, 1], None),         # negative key block
    ([0, 2, 2, 3], [2, 0, 1], None),          # not ascending within a row
    ([0, 2, 2, 3], [1, 1, 1], None),          # repeated entry
    ([0, 2, 1, 3], [0, 2, 1], None),          # row_ptr decreasing
    ([1, 2, 2, 3], [0, 2, 1], None),          # row_ptr[0] != 0
    ([0, 2, 2, 4], [0, 2, 1], None),          # row_ptr[nblk] != nnz
    ([0, 2, 2, 3], [0, 2, 1], [0, 0, 1]),     # row_order not a permutation
    ([0, 2, 2, 3], [0, 2, 1], [0, 1, 3]),     # row_order out of range
])
def test_tile_mask_check_rejects_malformed(lib, row_ptr, col_idx, row_order):
    assert _mask_status(lib, row_ptr, col_idx, row_order) == _lib.ERR_INVALID_ARG
    # the Python mask refuses it before anything reaches a device
    with pytest.raises(fp.FpattnError):
        fp.StaPlan(np.asarray(row_ptr, np.int32), np.asarray(col_idx, np.int32),
                   None if row_order is None else np.asarray(row_order, np.int32)).to("cpu")


def test_attention_fwd_refuses_mismatched_operands():
    """Operands the kernel would read past are refused in Python, before any
    launch: shapes that differ, FP8 granularities swapped, q/k formats mixed,
    buffers too small for the shape."""
    import torch
    B, H, N, d = 1, 2, 256, 128

    def nv(n=N, h=H):
        return fp.Nvfp4Tensor(torch.zeros(B, h, n, d // 2, dtype=torch.uint8),
                              torch.zeros(B * h * ((n + 127) // 128) * 2 * 512, dtype=torch.uint8),
                              torch.zeros(1), (B, h, n, d))

    def f8(gran, n=N):
        sc = torch.zeros(B, H, (n + 127) // 128) if gran == "tile128" else torch.zeros(B, H, d)
        return fp.Fp8Tensor(torch.zeros(B, H, n, d, dtype=torch.uint8), sc, gran, (B, H, n, d))

    with pytest.raises(ValueError, match="shapes differ"):
        fp.attention_fwd(nv(), nv(n=128), f8("channel"))
    with pytest.raises(ValueError, match="shapes differ"):
        fp.attention_fwd(nv(h=1), nv(h=1), f8("channel"))
    with pytest.raises(ValueError, match="per-channel"):
        fp.attention_fwd(nv(), nv(), f8("tile128"))
    with pytest.raises(ValueError, match="per-tile"):
        fp.attention_fwd(f8("channel"), f8("channel"), f8("channel"))
    with pytest.raises(TypeError):
        fp.attention_fwd(nv(), f8("tile128"), f8("channel"))
    short = nv()
    short.block_sf = short.block_sf[:100]
    with pytest.raises(ValueError):
        fp.attention_fwd(short, nv(), f8("channel"))
    # CPU buffers never reach the library
    with pytest.raises(ValueError, match="contiguous tensor on"):
        fp.attention_fwd(nv(), nv(), f8("channel"))


def test_attention_refuses_bad_qk_amax():
    """A caller's Q/K amax is refused before any launch unless it is two CUDA
    float32 tensors and Q/K are NVFP4."""
    q = torch.zeros(1, 1, 128, 128, dtype=torch.bfloat16)
    amax = (torch.ones(1), torch.ones(1))
    with pytest.raises(ValueError):
        fp.attention(q, q, q, qk_format="fp8", qk_amax=amax)
    with pytest.raises(ValueError):
        fp.attention(q, q, q, qk_amax=amax)          # host tensors
    with pytest.raises(ValueError):
        fp.attention(q, q, q, qk_amax=(amax[0],))    # one tensor
