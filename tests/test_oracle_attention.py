"""Pins for the oracle's online-softmax attention and STA geometry (CPU only).

* With P unquantized, the tiled online algorithm equals torch's fp64
  scaled_dot_product_attention (a library routine), dense, causal and masked,
  over several tiles and a ragged tail.
* Rows of P/l sum to one (V = 1 gives output 1).
* Identical keys give exactly the mean of V (P = 1 is representable).
* Causal row 0 is v_0.
* Worked examples pin the E4M3 rounding of P against the running max and the
  rescale across tiles.
* The conditional rescale with threshold tau: unquantized, it equals the
  textbook softmax for any tau; worked examples pin the stale-max decision and
  the 448 * 2^-tau rounding scale on both sides of the threshold.
* The STA block lists agree with a brute-force token-level window test and
  with the pair counts of the (6,8,8)-tile, (3,3,5)-window video workload.
"""
import math

import numpy as np
import pytest
import torch

from oracle import attention as A
from oracle import sta


def _sdpa(q, k, v, causal=False, mask=None):
    tq, tk, tv = (torch.from_numpy(np.asarray(t, dtype=np.float64))[None, None] for t in (q, k, v))
    attn_mask = None if mask is None else torch.from_numpy(mask)[None, None]
    out = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=attn_mask,
                                                           is_causal=causal)
    return out[0, 0].numpy()


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,d", [(300, 64), (129, 128), (77, 32)])
def test_unquantized_matches_sdpa(N, d, causal):
    rng = np.random.default_rng(N + d)
    q, k, v = (rng.standard_normal((N, d)) * 2 for _ in range(3))
    out, lse = A.attention(q, k, v, causal=causal, quantize_p=False)
    ref = _sdpa(q, k, v, causal=causal)
    assert np.max(np.abs(out - ref)) < 1e-12
    S = (q @ k.T) / math.sqrt(d)
    if causal:
        S = np.where(np.tril(np.ones((N, N), bool)), S, -np.inf)
    mx = S.max(axis=1)
    ref_lse = mx + np.log(np.exp(S - mx[:, None]).sum(axis=1))
    assert np.max(np.abs(lse - ref_lse)) < 1e-12


def test_unquantized_block_mask_matches_sdpa():
    rng = np.random.default_rng(11)
    N, d = 512, 32
    q, k, v = (rng.standard_normal((N, d)) for _ in range(3))
    key_blocks = [[0, 2], [1], [0, 1, 2, 3], [3]]
    mask = np.zeros((N, N), bool)
    for qb, kbs in enumerate(key_blocks):
        for kb in kbs:
            mask[qb * 128:(qb + 1) * 128, kb * 128:(kb + 1) * 128] = True
    out, _ = A.attention(q, k, v, key_blocks=key_blocks, quantize_p=False)
    assert np.max(np.abs(out - _sdpa(q, k, v, mask=mask))) < 1e-12
    dense, _ = A.attention(q, k, v, quantize_p=True)
    allk, _ = A.attention(q, k, v, key_blocks=[[0, 1, 2, 3]] * 4, quantize_p=True)
    assert np.array_equal(dense, allk)


def test_rows_of_p_sum_to_one():
    rng = np.random.default_rng(12)
    N, d = 400, 64
    q, k = rng.standard_normal((N, d)) * 3, rng.standard_normal((N, d)) * 3
    out, _ = A.attention(q, k, np.ones((N, 8)), quantize_p=False)
    assert np.max(np.abs(out - 1.0)) < 1e-12
    out, _ = A.attention(q, k, np.ones((N, 8)), causal=True, quantize_p=False)
    assert np.max(np.abs(out - 1.0)) < 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_identical_keys_give_mean_of_v(causal):
    rng = np.random.default_rng(13)
    N, d = 300, 64
    q = rng.standard_normal((N, d))
    k = np.tile(rng.standard_normal((1, d)), (N, 1))
    v = rng.standard_normal((N, d))
    out, lse = A.attention(q, k, v, causal=causal, quantize_p=True)
    if causal:
        ref = np.cumsum(v, axis=0) / np.arange(1, N + 1)[:, None]
    else:
        ref = np.tile(v.mean(axis=0), (N, 1))
    assert np.max(np.abs(out - ref)) < 1e-12


def test_causal_row0_is_v0():
    rng = np.random.default_rng(14)
    q, k, v = (rng.standard_normal((200, 64)) for _ in range(3))
    out, lse = A.attention(q, k, v, causal=True)
    assert np.array_equal(out[0], v[0])
    assert lse[0] == pytest.approx(q[0] @ k[0] / 8.0, abs=1e-12)


def _two_key_setup(s0, s1):
    """q = e_0, keys with scores exactly s0, s1 under softmax_scale = 1."""
    q = np.zeros((1, 4)); q[0, 0] = 1.0
    k = np.zeros((2, 4)); k[0, 0] = s0; k[1, 0] = s1
    return q, k


def test_worked_example_p_rounding():
    # scores 0 and ln 0.3: P = [1, 0.3]; 448 * 0.3 = 134.4 -> E4M3 128
    q, k = _two_key_setup(0.0, math.log(0.3))
    v = np.array([[1.0, 0.0], [0.0, 1.0]])
    out, lse = A.attention_rows(q, k, v, np.array([0]), softmax_scale=1.0)
    l = 1.0 + 0.3
    assert out[0, 0] == pytest.approx(1.0 / l, abs=1e-15)
    assert out[0, 1] == pytest.approx((128.0 / 448.0) / l, abs=1e-15)
    assert lse[0] == pytest.approx(math.log(l), abs=1e-15)


def test_worked_example_rescale_across_tiles():
    # 128 keys with score 0 in tile 0, one key with score ln 3 in tile 1.
    # Tile 0 quantizes P = 1 against its own max (exact); tile 1 raises the
    # max, scaling the earlier sum by 1/3. Quantizing tile 0 against the final
    # max instead would give E4M3(448/3)/448 = 144/448 per key.
    N = 129
    q = np.zeros((1, 2)); q[0, 0] = 1.0
    k = np.zeros((N, 2)); k[128, 0] = math.log(3.0)
    v = np.zeros((N, 2)); v[:128, 0] = 1.0; v[128, 1] = 1.0
    out, lse = A.attention_rows(q, k, v, np.array([0]), softmax_scale=1.0)
    l = 128.0 / 3.0 + 1.0
    assert out[0, 0] == pytest.approx((128.0 / 3.0) / l, rel=1e-14)
    assert out[0, 1] == pytest.approx(1.0 / l, rel=1e-14)
    assert lse[0] == pytest.approx(math.log(3.0) + math.log(l), rel=1e-14)


def test_sta_counts_video_workload():
    grid, tile, window = (18, 48, 80), (6, 8, 8), (3, 3, 5)
    pairs = sta.tile_pairs(grid, tile, window)
    assert len(pairs) == 3 * 6 * 10
    assert sum(len(p) for p in pairs) == 4928
    blocks = sta.block_lists(grid, tile, window)
    assert len(blocks) == 18 * 48 * 80 // 128 == 540
    assert sum(len(b) for b in blocks) == 44352
    assert all(b == sorted(b) for b in blocks)
    # interior tile sees 3*3*5 tiles
    assert max(len(p) for p in pairs) == 45


def test_sta_block_lists_match_token_bruteforce():
    grid, tile, window = (12, 16, 24), (6, 8, 8), (3, 3, 5)
    blocks = sta.block_lists(grid, tile, window)
    N = 12 * 16 * 24
    rng = np.random.default_rng(15)
    qpos = np.unique(np.concatenate([rng.integers(0, N, 40), [0, N - 1, 383, 384]]))
    tok = sta.token_mask(grid, tile, window, qpos)
    for i, p in enumerate(qpos):
        from_blocks = np.zeros(N, bool)
        for kb in blocks[p // 128]:
            from_blocks[kb * 128:(kb + 1) * 128] = True
        assert np.array_equal(from_blocks, tok[i])


@pytest.mark.parametrize("tau", [1.0, 3.5, 8.0])
@pytest.mark.parametrize("causal", [False, True])
def test_threshold_rescale_unquantized_matches_sdpa(tau, causal):
    # A stale reference max cancels in O / l when P is not rounded, so any
    # threshold must reproduce the textbook softmax exactly.
    rng = np.random.default_rng(int(tau * 10) + causal)
    N, d = 300, 64
    q, k, v = (rng.standard_normal((N, d)) * 2 for _ in range(3))
    # raise the later keys' scores so the max keeps growing across tiles
    k[128:] *= 1.5
    out, lse = A.attention(q, k, v, causal=causal, quantize_p=False, rescale_threshold=tau)
    assert np.max(np.abs(out - _sdpa(q, k, v, causal=causal))) < 1e-12
    ref_out, ref_lse = A.attention(q, k, v, causal=causal, quantize_p=False)
    assert np.max(np.abs(lse - ref_lse)) < 1e-12


def _threshold_example(tau):
    # one query; key 0 (tile 0) scores 0; keys 128 and 129 (tile 1) score
    # 1.5 ln 2 and 1.5 ln 2 + ln 0.3; every other key -1000 (P = 0 exactly)
    N = 256
    q = np.ones((1, 1))
    k = np.full((N, 1), -1000.0)
    k[0, 0] = 0.0
    k[128, 0] = 1.5 * math.log(2.0)
    k[129, 0] = 1.5 * math.log(2.0) + math.log(0.3)
    v = np.zeros((N, 3))
    v[0, 0] = v[128, 1] = v[129, 2] = 1.0
    return A.attention_rows(q, k, v, np.array([0]), softmax_scale=1.0, rescale_threshold=tau)


def test_threshold_rescale_worked_example_keeps_stale_max():
    # tau = 3: the max grows by 1.5 (log2) <= 3, so m stays 0 and tile 1's P
    # reach 2^1.5. P is rounded at the scale 448 / 8 = 56:
    #   1 -> 56 (exact); 2^1.5 * 56 = 158.39 -> 160; 0.3 * 2^1.5 * 56 = 47.52 -> 48
    out, lse = _threshold_example(3.0)
    r = 2.0 ** 1.5
    l = 1.0 + r + 0.3 * r
    assert out[0].tolist() == pytest.approx([1.0 / l, (160.0 / 56.0) / l, (48.0 / 56.0) / l], rel=1e-14)
    assert lse[0] == pytest.approx(math.log(l), rel=1e-14)


def test_threshold_rescale_worked_example_moves_max():
    # tau = 1: 1.5 > 1, so m moves to 1.5 ln 2 and O, l scale by 2^-1.5. P is
    # rounded at 448 / 2 = 224: tile 0's 1 -> 224 (exact); tile 1: 1 -> 224,
    # 0.3 * 224 = 67.2 -> 64.
    out, lse = _threshold_example(1.0)
    a = 2.0 ** -1.5
    l = a + 1.0 + 0.3
    assert out[0].tolist() == pytest.approx([a / l, 1.0 / l, (64.0 / 224.0) / l], rel=1e-14)
    assert lse[0] == pytest.approx(1.5 * math.log(2.0) + math.log(l), rel=1e-14)
    # the same keys at tau = 0 round tile 1 at 448: 0.3 * 448 = 134.4 -> 128
    out0, _ = _threshold_example(0.0)
    assert out0[0, 2] == pytest.approx((128.0 / 448.0) / l, rel=1e-14)


def test_threshold_is_in_log2_units():
    # tau = 1.25 lies between the growth in log2 units (1.5) and in natural
    # units (1.04): the max must move. Rounding scale s = 448 * 2^-1.25 =
    # 188.36: 1 * s -> 192 (step 16 in [128, 256)); 0.3 * s = 56.51 -> 56
    # (step 4 in [32, 64)).
    out, _ = _threshold_example(1.25)
    s = 448.0 * 2.0 ** -1.25
    a = 2.0 ** -1.5
    l = a + 1.3
    assert out[0].tolist() == pytest.approx([a * (192.0 / s) / l, (192.0 / s) / l, (56.0 / s) / l], rel=1e-14)


def test_tile_major_raster_index_worked_example():
    # 2 x 2 x 4 grid in 1 x 2 x 2 tiles, worked out by hand: tiles in raster
    # order (0,0,0), (0,0,1), (1,0,0), (1,0,1); each lists its 2 x 2 tokens
    # (h, w) in raster order; raster row = t*8 + h*4 + w.
    perm = sta.raster_index_of_tile_major((2, 2, 4), (1, 2, 2))
    assert perm.tolist() == [0, 1, 4, 5, 2, 3, 6, 7, 8, 9, 12, 13, 10, 11, 14, 15]


def test_tile_major_raster_index_is_tile_contiguous_bijection():
    grid, tile = (12, 16, 24), (6, 8, 8)
    perm = sta.raster_index_of_tile_major(grid, tile)
    N = 12 * 16 * 24
    assert sorted(perm.tolist()) == list(range(N))
    vol = 6 * 8 * 8
    t, h, w = perm // (16 * 24), (perm // 24) % 16, perm % 24
    for i0 in range(0, N, vol):
        # one tile per vol consecutive positions, full extent on every axis
        sl = slice(i0, i0 + vol)
        assert len({(a // 6, b // 8, c // 8) for a, b, c in zip(t[sl], h[sl], w[sl])}) == 1
        # raster order inside the tile: (t, h, w) ascend lexicographically
        key = (t[sl] * 1000 + h[sl]) * 1000 + w[sl]
        assert np.all(np.diff(key) > 0)
    # tiles themselves in raster order over the 2 x 2 x 3 tile grid
    firsts = [(t[i] // 6, h[i] // 8, w[i] // 8) for i in range(0, N, vol)]
    assert firsts == [(a, b, c) for a in range(2) for b in range(2) for c in range(3)]


def test_nvfp4_p_worked_example():
    # One tile, keys 0 and 1 score 0 and ln 0.3, the rest -1000 (P = 0).
    # P's tensor amax is fixed at 1: s_t = 1/2688, and the first 16-key block
    # has A_b = 1 -> sb = E4M3(448) = 448, den = 448/2688 = 1/6.
    # Codes: 1 * 6 = 6 -> 6; 0.3 * 6 = 1.8 -> 2 (E2M1 grid 1.5, 2).
    # P_hat = [1, 2/6]; l uses the unquantized P.
    N = 128
    q = np.ones((1, 1))
    k = np.full((N, 1), -1000.0)
    k[0, 0] = 0.0
    k[1, 0] = math.log(0.3)
    v = np.zeros((N, 2))
    v[0, 0] = v[1, 1] = 1.0
    out, lse = A.attention_rows(q, k, v, np.array([0]), softmax_scale=1.0, p_format="nvfp4")
    assert out[0].tolist() == pytest.approx([1.0 / 1.3, (1.0 / 3.0) / 1.3], rel=1e-6)
    assert lse[0] == pytest.approx(math.log(1.3), rel=1e-12)


def test_nvfp4_p_small_block_scale():
    # Tile 0: key 0 at score 0 (P = 1). Keys 16 and 17 (the second 16-key
    # block) at ln 0.01 and ln 0.004: that block's A_b = 0.01, sb =
    # E4M3(4.48) = 4.5 (grid step 0.5 in [4, 8)), den = 4.5/2688.
    # Codes: 0.01 * 2688/4.5 = 5.973 -> 6; 0.004 * 2688/4.5 = 2.389 -> 2.
    N = 128
    q = np.ones((1, 1))
    k = np.full((N, 1), -1000.0)
    k[0, 0] = 0.0
    k[16, 0] = math.log(0.01)
    k[17, 0] = math.log(0.004)
    v = np.zeros((N, 3))
    v[0, 0] = v[16, 1] = v[17, 2] = 1.0
    out, _ = A.attention_rows(q, k, v, np.array([0]), softmax_scale=1.0, p_format="nvfp4")
    l = 1.0 + 0.01 + 0.004
    step = 4.5 / 2688.0
    assert out[0].tolist() == pytest.approx([1.0 / l, 6 * step / l, 2 * step / l], rel=1e-6)
