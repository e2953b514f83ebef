"""Sliding-tile attention (STA) geometry: TEST INFRASTRUCTURE ONLY.

FPSAttention page, section 2.2: the 3D video token space is cut into
non-overlapping tiles T_u; query tile u attends key tile v when the L-infinity
distance of their tile coordinates is within the window,
    W(u) = { v : ||c_u - c_v||_inf <= (window half-widths) }.
The printed bound is garbled; the reading used here takes the window size in
tiles (w_t, w_h, w_w) and the half-width per axis as floor(w / 2), clipped at
the grid edges (edge tiles see fewer tiles; the window is not shifted).

Tokens are in tile-major order: tiles in raster order over the tile grid, and
the tokens of a tile in raster order inside it. With a tile volume that is a
multiple of 128, every 128-token block lies inside one tile, so the tile mask
is exactly a list of allowed 128-key blocks per 128-query block.
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

import numpy as np


def tile_grid(grid: Sequence[int], tile: Sequence[int]) -> Tuple[int, int, int]:
    return tuple(g // t for g, t in zip(grid, tile))


def window_tiles(u: Sequence[int], ngrid: Sequence[int], window: Sequence[int]) -> List[Tuple[int, int, int]]:
    """All tile coordinates v with |u_a - v_a| <= window_a // 2 on every axis."""
    half = [w // 2 for w in window]
    ranges = [range(max(0, u[a] - half[a]), min(ngrid[a], u[a] + half[a] + 1)) for a in range(3)]
    return [(a, b, c) for a in ranges[0] for b in ranges[1] for c in ranges[2]]


def tile_index(c: Sequence[int], ngrid: Sequence[int]) -> int:
    return (c[0] * ngrid[1] + c[1]) * ngrid[2] + c[2]


def tile_pairs(grid, tile, window) -> List[List[int]]:
    """pairs[u] = sorted tile indices v in W(u), u in raster order."""
    ng = tile_grid(grid, tile)
    out = []
    for a in range(ng[0]):
        for b in range(ng[1]):
            for c in range(ng[2]):
                out.append(sorted(tile_index(v, ng) for v in window_tiles((a, b, c), ng, window)))
    return out


def block_lists(grid, tile, window, block: int = 128) -> List[List[int]]:
    """key_blocks[qb]: ascending 128-key blocks allowed for 128-query block qb."""
    vol = tile[0] * tile[1] * tile[2]
    assert vol % block == 0, "tile volume must be a multiple of the block size"
    per = vol // block
    pairs = tile_pairs(grid, tile, window)
    out = []
    for u, vs in enumerate(pairs):
        blocks = [v * per + i for v in vs for i in range(per)]
        for _ in range(per):
            out.append(blocks)
    return out


def token_coords_tile_major(grid, tile) -> np.ndarray:
    """(t, h, w) coordinates of each token position in tile-major order."""
    ng = tile_grid(grid, tile)
    coords = []
    for a in range(ng[0]):
        for b in range(ng[1]):
            for c in range(ng[2]):
                for i in range(tile[0]):
                    for j in range(tile[1]):
                        for k in range(tile[2]):
                            coords.append((a * tile[0] + i, b * tile[1] + j, c * tile[2] + k))
    return np.array(coords, dtype=np.int64)


def raster_index_of_tile_major(grid, tile) -> np.ndarray:
    """perm[i] = raster (time-major) row of the token at tile-major position i.

    Raster order numbers token (t, h, w) of a T x Hs x W grid as
    (t * Hs + h) * W + w. FPSAttention page, section 3.3, item 1 (contiguous
    memory through a tile transpose): x_tile_major = x_raster[perm].
    """
    coords = token_coords_tile_major(grid, tile)
    return (coords[:, 0] * grid[1] + coords[:, 1]) * grid[2] + coords[:, 2]


def token_mask(grid, tile, window, query_pos: np.ndarray) -> np.ndarray:
    """Brute-force token-level mask: rows = query positions, cols = all keys.

    Allowed when every axis satisfies |floor(tq/T) - floor(tk/T)| <= window//2.
    """
    coords = token_coords_tile_major(grid, tile)
    tq = coords[query_pos] // np.array(tile)
    tk = coords // np.array(tile)
    half = np.array([w // 2 for w in window])
    diff = np.abs(tq[:, None, :] - tk[None, :, :])
    return np.all(diff <= half, axis=-1)
