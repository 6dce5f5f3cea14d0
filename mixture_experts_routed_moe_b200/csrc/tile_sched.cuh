// Device-side tile scheduler of the grouped GEMMs. The tile list exists only on
// the device: expert e owns the 128-row blocks mt_base[e] .. mt_base[e+1]-1 of
// the permuted rows, and every row block is crossed with n_tiles column blocks.
// Tiles are numbered expert by expert; inside an expert the column block is the
// outer index and the row block the inner one, so CTAs running at the same time
// share weight tiles (and activation rows) through L2.
#pragma once

#include "moe_internal.h"

namespace moe {

struct TileCoord {
  int e, m, n, row0, valid;  // expert, row block in expert, column block, first row, rows holding assignments
};

// Largest e in [0, E) with s_mt[e] <= mtile (the expert owning that row block).
__device__ __forceinline__ int find_expert(const int* s_mt, int E, int mtile) {
  int lo = 0, hi = E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_mt[mid] <= mtile)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ TileCoord tile_coord(int tile, const int* s_mt, const int* s_cnt, int E, int NT) {
  TileCoord c;
  c.e = find_expert(s_mt, E, tile / NT);
  const int base = s_mt[c.e];
  const int nm = s_mt[c.e + 1] - base;
  const int local = tile - base * NT;
  c.n = local / nm;
  c.m = local - c.n * nm;
  c.row0 = (base + c.m) * kTileM;
  c.valid = min(kTileM, s_cnt[c.e] - c.m * kTileM);
  return c;
}

}  // namespace moe
