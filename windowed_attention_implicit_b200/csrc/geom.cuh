// geom.cuh -- window / tile geometry shared by the attention and copy kernels.
//
// A window of M x M tokens (M % 16 == 0) is cut into tiles of 8 rows x 16
// columns = 128 tokens.  Each tile is fetched as two TMA boxes of 8 x 8
// pixels (columns j0..j0+7 and j0+8..j0+15), so the 128 rows of a tile in
// shared memory are ordered  row = c*64 + ii*8 + jj  with c the box, ii the
// row inside the tile and jj the column inside the box.  Window-local token
// (i, j) lives at map pixel ((wy*M + i + s) mod H, (wx*M + j + s) mod W):
// the cyclic roll by -s is folded into the TMA box coordinates.  With
// s % 8 == 0 and H, W multiples of 8 a box never straddles the wrap.
#pragma once

namespace rib {

struct UnitCoord {
  int b, w, head, wy, wx;
};

__device__ __forceinline__ UnitCoord decode_unit(int unit, int heads, int nW, int nWx) {
  UnitCoord u;
  u.head = unit % heads;
  const int bw = unit / heads;
  u.w = bw % nW;
  u.b = bw / nW;
  u.wy = u.w / nWx;
  u.wx = u.w % nWx;
  return u;
}

// Top-left window-local (i0, j0) of 128-token tile t; tiles_x = M / 16.
__device__ __forceinline__ void tile_origin(int t, int tiles_x, int& i0, int& j0) {
  i0 = (t / tiles_x) * 8;
  j0 = (t % tiles_x) * 16;
}

// Shifted-window region mask (optional; the pages describe none): on the map
// rolled by -s, row band of rolled row y is 0 below H - M, 1 below H - s,
// else 2 (columns alike with W).  A query attends only to keys of its own
// (row band, column band).  Band boundaries fall on multiples of 8 (M % 16
// and s % 8 are 0), so every 8 x 8 token block of a tile lies in one band
// pair.  Only windows of the last window row or column hold more than one.
__device__ __forceinline__ int region_band(int pos, int size, int M, int s) {
  return pos < size - M ? 0 : (pos < size - s ? 1 : 2);
}

// v in [0, 2n) -> v mod n.
__device__ __forceinline__ int wrap_once(int v, int n) { return v >= n ? v - n : v; }

// Row r (0..127) of tile (i0, j0) -> window-local (i, j).
__device__ __forceinline__ void tile_row_local(int r, int i0, int j0, int& i, int& j) {
  i = i0 + ((r >> 3) & 7);
  j = j0 + ((r >> 6) << 3) + (r & 7);
}

}  // namespace rib
