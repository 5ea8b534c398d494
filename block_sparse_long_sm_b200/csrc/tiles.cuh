// tiles.cuh -- the key tiles of one 128-row query block, in the order the
// one-head kernels walk them: sink tiles (contiguous), selected tiles (the
// plan's kept candidates, gathered) and local tiles (contiguous, the last one
// the causally masked diagonal).  In dense mode the local range starts at
// key 0.  Used by the FP8 attention and the key-mass kernels.
#pragma once

#include "common.cuh"

namespace spa {

// Geometry and plan pointers shared by the kernels that walk a block's tiles.
struct TileGeom {
  int Hq, Hkv, L, nqb, group;
  int sink, local, mode;
  const int* counts;          // kept candidates per block (keys, or key blocks in SALE mode)
  const int* lists;           // index lists at closed-form offsets
  long long list_per_head;    // list elements per (b, h)
  long long cap_a;            // local + sink
  int list_unit;              // 1 (keys) or block_k (SALE: key-block ids)
};

struct BlockTiles {
  int b, h, kvh, qb, row0, le, ls, sink_end;
  int n_sink_t, n_sel_t, n_loc_t, n_sel, loc_start;
  long long list_off;
};

// CTA x -> (b, kv head, q head, block), the longest blocks of each kv head first.
__device__ __forceinline__ BlockTiles block_tiles(const TileGeom& g, int x) {
  BlockTiles it;
  const int per_kv = g.nqb * g.group;
  const int bkv = x / per_kv;
  const int rem = x - bkv * per_kv;
  it.qb = g.nqb - 1 - rem / g.group;
  it.b = bkv / g.Hkv;
  it.kvh = bkv - it.b * g.Hkv;
  it.h = it.kvh * g.group + rem % g.group;
  it.row0 = it.qb * 128;
  it.le = min(it.row0 + 128, g.L);
  it.ls = max(0, it.row0 + 128 - g.local);
  it.sink_end = min(g.sink, it.ls);
  if (g.mode == kModeDense) {
    it.n_sink_t = 0;
    it.n_sel = 0;
    it.loc_start = 0;
    it.list_off = 0;
  } else {
    it.n_sink_t = (it.sink_end + 127) / 128;
    const int bh = it.b * g.Hq + it.h;
    it.n_sel = g.counts[(long long)bh * g.nqb + it.qb] * g.list_unit;
    it.loc_start = it.ls;
    it.list_off = (long long)bh * g.list_per_head + cap_prefix(it.qb, 128, g.cap_a) / g.list_unit;
  }
  it.n_sel_t = (it.n_sel + 127) / 128;
  it.n_loc_t = (it.le - it.loc_start + 127) / 128;
  return it;
}

struct Tile {
  int gather;   // 1 -> selected (gathered) tile
  int key0;     // first key of a contiguous tile / first selected ordinal of a gathered tile
  int valid;    // valid columns
  int causal;   // diagonal tile
};

__device__ __forceinline__ Tile tile_of(const BlockTiles& it, int t) {
  Tile d;
  if (t < it.n_sink_t) {
    d = {0, t * 128, min(128, it.sink_end - t * 128), 0};
  } else if (t < it.n_sink_t + it.n_sel_t) {
    const int k0 = (t - it.n_sink_t) * 128;
    d = {1, k0, min(128, it.n_sel - k0), 0};
  } else {
    const int k0 = it.loc_start + (t - it.n_sink_t - it.n_sel_t) * 128;
    d = {0, k0, min(128, it.le - k0), k0 == it.row0 ? 1 : 0};
  }
  return d;
}

// Key of selected ordinal n of the block's list.
__device__ __forceinline__ int selected_key(const TileGeom& g, const BlockTiles& it, int n) {
  if (g.list_unit == 1) return g.lists[it.list_off + n];
  return g.lists[it.list_off + n / g.list_unit] * g.list_unit + n % g.list_unit;
}

}  // namespace spa
