// Video token order: tile-major position -> raster (time-major) position.
//
// The sliding-tile pattern (FPSAttention page, section 2.2) works on 3D
// tiles of a T x Hs x W token grid, and the kernel keeps each tile's tokens
// contiguous (section 3.3, item 1: contiguous memory access through a tile
// transpose). Tile-major order lists the tiles in raster order over the tile
// grid and, inside a tile, its tokens in raster order. The quantizers read
// raster-order activations through this map and write tile-major codes; the
// attention epilogue writes its rows back to raster positions.
#pragma once

#include <cstdint>

namespace fpattn {

// Division by a run-time invariant divisor through one multiply and one shift
// (Granlund and Montgomery, "Division by Invariant Integers using
// Multiplication", 1994, theorem 4.2 with a 31-bit numerator): with
// l = ceil(log2 d) and m = floor(2^(31+l) / d) + 1, floor(n / d) equals
// floor(n * m / 2^(31+l)) for every 0 <= n < 2^31.
struct FastDiv {
  unsigned long long m;
  uint32_t shift;
  uint32_t d;
};

inline FastDiv make_fastdiv(uint32_t d) {
  uint32_t l = 0;
  while ((1ull << l) < d) ++l;
  return {((1ull << (31 + l)) / d) + 1ull, 31u + l, d};
}

__device__ __forceinline__ uint32_t fdiv_u(uint32_t n, const FastDiv& f) {
  return static_cast<uint32_t>((static_cast<unsigned long long>(n) * f.m) >> f.shift);
}

struct TokenMap {
  int on;              // 0: identity (tokens already in the order the kernels use)
  int tt, th, tw;      // tile, in tokens
  int Hs, W;           // grid extents that set the raster strides
  FastDiv vol;         // tt * th * tw
  FastDiv plane;       // th * tw
  FastDiv row;         // tw
  FastDiv ngw;         // W / tw
  FastDiv ngh;         // Hs / th
};

inline TokenMap make_token_map(int T, int Hs, int W, int tt, int th, int tw) {
  (void)T;
  TokenMap m;
  m.on = 1;
  m.tt = tt;
  m.th = th;
  m.tw = tw;
  m.Hs = Hs;
  m.W = W;
  m.vol = make_fastdiv(static_cast<uint32_t>(tt * th * tw));
  m.plane = make_fastdiv(static_cast<uint32_t>(th * tw));
  m.row = make_fastdiv(static_cast<uint32_t>(tw));
  m.ngw = make_fastdiv(static_cast<uint32_t>(W / tw));
  m.ngh = make_fastdiv(static_cast<uint32_t>(Hs / th));
  return m;
}

// Grid coordinates (t, h, w) of tile-major position n (0 <= n < T*Hs*W).
__device__ __forceinline__ void tile_major_coords(const TokenMap& m, uint32_t n, int& t, int& h, int& w) {
  const uint32_t tile = fdiv_u(n, m.vol);
  const uint32_t i = n - tile * m.vol.d;
  const uint32_t it = fdiv_u(i, m.plane);
  const uint32_t r = i - it * m.plane.d;
  const uint32_t ih = fdiv_u(r, m.row);
  const uint32_t iw = r - ih * m.row.d;
  const uint32_t tr = fdiv_u(tile, m.ngw);  // tile row index over (t, h) of the tile grid
  const uint32_t c = tile - tr * m.ngw.d;
  const uint32_t a = fdiv_u(tr, m.ngh);
  const uint32_t b = tr - a * m.ngh.d;
  t = static_cast<int>(a) * m.tt + static_cast<int>(it);
  h = static_cast<int>(b) * m.th + static_cast<int>(ih);
  w = static_cast<int>(c) * m.tw + static_cast<int>(iw);
}

// Raster position of tile-major position n; n itself when the map is off.
__device__ __forceinline__ int to_raster(const TokenMap& m, int n) {
  if (!m.on) return n;
  int t, h, w;
  tile_major_coords(m, static_cast<uint32_t>(n), t, h, w);
  return (t * m.Hs + h) * m.W + w;
}

}  // namespace fpattn
