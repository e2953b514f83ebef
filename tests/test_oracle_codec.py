"""Pins for the oracle's element formats (CPU only).

The E4M3 decoder is checked against torch's float8_e4m3fn (an independent
library implementation) on all 256 codes; the encoder against hand-computed
codes (tests/golden/codec_hand.json) and against torch's round-to-nearest-even
cast on in-range values; E2M1 against its hand-computed table.
"""
import json
import os

import numpy as np
import pytest
import torch

from oracle import codec

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "codec_hand.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def test_e4m3_decode_all_codes_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = codec.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert nan.sum() == 2 and nan[0x7F] and nan[0xFF]
    assert np.array_equal(ours[~nan], ref[~nan])
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9


@pytest.mark.parametrize("case", _golden()["e4m3"], ids=lambda c: repr(c["x"]))
def test_e4m3_encode_hand(case):
    assert int(codec.e4m3_encode(np.float64(case["x"]))) == case["code"]


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(0)
    # random values over the whole range, plus every midpoint between grid points
    vals = rng.uniform(-448, 448, 20000)
    vals = np.concatenate([vals, rng.standard_normal(20000) * 2.0 ** rng.integers(-12, 8, 20000)])
    grid = codec.e4m3_decode(np.arange(0, 127))
    mids = (grid[1:] + grid[:-1]) / 2
    vals = np.concatenate([vals, mids, -mids, grid, -grid]).astype(np.float32)
    ours = codec.e4m3_encode(vals)
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_e4m3_encode_roundtrip_all_codes():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    assert np.array_equal(codec.e4m3_encode(codec.e4m3_decode(codes)), codes)


def test_e2m1_decode_table():
    expect = [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    got = codec.e2m1_decode(np.arange(16))
    assert list(got[:8]) == expect
    assert list(got[8:]) == [-v for v in expect]


@pytest.mark.parametrize("case", _golden()["e2m1"], ids=lambda c: repr(c["x"]))
def test_e2m1_encode_hand(case):
    assert int(codec.e2m1_encode(np.float64(case["x"]))) == case["code"]


def test_e2m1_roundtrip_and_monotone():
    codes = np.arange(16, dtype=np.uint8)
    back = codec.e2m1_encode(codec.e2m1_decode(codes))
    assert np.array_equal(back, codes)
    x = np.linspace(-7, 7, 4001)
    v = codec.e2m1_decode(codec.e2m1_encode(x))
    assert np.all(np.diff(v) >= 0)
    # nearest: never farther than half the local grid spacing (or saturation)
    clipped = np.clip(x, -6, 6)
    gap = np.where(np.abs(clipped) < 2, 0.5, np.where(np.abs(clipped) < 4, 1.0, 2.0))
    assert np.all(np.abs(v - clipped) <= gap / 2 + 1e-12)


def test_pack_nibble_order():
    packed = codec.pack_e2m1(np.array([1, 2, 0xF, 0x8], dtype=np.uint8))
    assert list(packed) == [0x21, 0x8F]
    codes = np.random.default_rng(1).integers(0, 16, (3, 64)).astype(np.uint8)
    assert np.array_equal(codec.unpack_e2m1(codec.pack_e2m1(codes)), codes)
