// Device-side tile scheduler of the grouped GEMMs. The tile list exists only on
// the device: expert e owns the 128-row blocks mt_base[e] .. mt_base[e+1]-1 of
// the permuted rows, and every row block is crossed with n_tiles column blocks.
// Tiles are numbered expert by expert; inside an expert the column block is the
// outer index and the row block the inner one, so CTAs running at the same time
// share weight tiles (and activation rows) through L2.
#pragma once

#include "moe_common.cuh"
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

namespace moe {

// Dynamic hand-out of the tiles of a persistent GEMM. The producer thread
// takes the next tile number from a global counter (zeroed before the launch)
// and publishes it through a small ring in shared memory; every other role
// (MMA issuer, epilogue warps) reads the tiles from the ring in the same order.
// Tiles are handed out in increasing order as CTAs become free, so the tiles
// in flight at any moment are a window of consecutive numbers: the row blocks
// of one (expert, column block) run at the same time and share its weight
// tile through L2, and CTAs that finish early take more tiles. A number past
// the last tile, or a bounded wait that gave up, ends every role's loop (-1).
constexpr int kTileRing = 4;

struct TileRing {
  int* ids;         // [kTileRing] shared memory
  uint64_t* full;   // [kTileRing] 1 arrival: the producer published the slot
  uint64_t* empty;  // [kTileRing] `consumers` arrivals: every reader is done with it
};

// Producer: the tile of sequence number i (or -1 when there are no more).
__device__ __forceinline__ int tiles_publish(const TileRing& r, int i, int* counter, int total,
                                             volatile int* abort_flag, int* dev_status, uint64_t limit_ns) {
  const int slot = i % kTileRing;
  const uint32_t par = static_cast<uint32_t>(i / kTileRing) & 1u;
  if (!mbar_wait_bounded(&r.empty[slot], par ^ 1u, abort_flag, dev_status, limit_ns)) return -1;
  int t = atomicAdd(counter, 1);
  if (t >= total) t = -1;
  r.ids[slot] = t;
  mbar_arrive(&r.full[slot]);
  return t;
}

// One consumer thread (the MMA issuer): the tile of sequence number i.
__device__ __forceinline__ int tiles_take(const TileRing& r, int i, volatile int* abort_flag, int* dev_status,
                                          uint64_t limit_ns) {
  const int slot = i % kTileRing;
  const uint32_t par = static_cast<uint32_t>(i / kTileRing) & 1u;
  if (!mbar_wait_bounded(&r.full[slot], par, abort_flag, dev_status, limit_ns)) return -1;
  const int t = r.ids[slot];
  mbar_arrive(&r.empty[slot]);
  return t;
}

// A consumer warp (one arrival per warp): the tile of sequence number i.
__device__ __forceinline__ int tiles_take_warp(const TileRing& r, int i, int lane, volatile int* abort_flag,
                                               int* dev_status, uint64_t limit_ns) {
  const int slot = i % kTileRing;
  const uint32_t par = static_cast<uint32_t>(i / kTileRing) & 1u;
  const bool got = mbar_wait_bounded(&r.full[slot], par, abort_flag, dev_status, limit_ns);
  int t = got ? r.ids[slot] : -1;
  if (!__all_sync(0xffffffffu, got)) t = -1;
  __syncwarp();
  if (lane == 0) mbar_arrive(&r.empty[slot]);
  return t;
}

}  // namespace moe
