// Tile-major token order (Token Radius Attention summary, §2 "TRA pipeline",
// tile-major layout).  Tiles of tt x ty x tx tokens are taken in
// (frame-tile, tile-row, tile-col) order; inside a tile the tokens are in
// (t, y, x) row-major order; tiles at the far edges of the grid are truncated.
//
// Position p of the tile-major sequence is decoded in closed form: every
// frame-tile but the last holds tt*H*W tokens, every tile-row of a frame-tile
// but the last holds ft*ty*W tokens, every tile of a tile-row but the last
// holds ft*hy*tx tokens (ft, hy = frames / rows of that frame-tile / tile-row).
#pragma once
#include <cstdint>

namespace tra {

struct TileLayout {
  int F, H, W;     // grid
  int tt, ty, tx;  // tile
};

struct Coord {
  int t, y, x;
};

__host__ __device__ __forceinline__ int imin(int a, int b) { return a < b ? a : b; }

// (t, y, x) of the token at tile-major position p (0 <= p < F*H*W).
__host__ __device__ __forceinline__ Coord tile_major_coord(const TileLayout& L, int p) {
  const int frame_tile = L.tt * L.H * L.W;
  const int Tt = p / frame_tile;
  int rem = p - Tt * frame_tile;
  const int ft = imin(L.tt, L.F - Tt * L.tt);
  const int row_tile = ft * L.ty * L.W;
  const int Ty = rem / row_tile;
  rem -= Ty * row_tile;
  const int hy = imin(L.ty, L.H - Ty * L.ty);
  const int tile = ft * hy * L.tx;
  const int Tx = rem / tile;
  rem -= Tx * tile;
  const int wx = imin(L.tx, L.W - Tx * L.tx);
  const int plane = hy * wx;
  const int tl = rem / plane;
  rem -= tl * plane;
  const int yl = rem / wx;
  const int xl = rem - yl * wx;
  return Coord{Tt * L.tt + tl, Ty * L.ty + yl, Tx * L.tx + xl};
}

// Original index (t*H + y)*W + x of the token at tile-major position p.
__host__ __device__ __forceinline__ int tile_major_source(const TileLayout& L, int p) {
  const Coord c = tile_major_coord(L, p);
  return (c.t * L.H + c.y) * L.W + c.x;
}

}  // namespace tra
