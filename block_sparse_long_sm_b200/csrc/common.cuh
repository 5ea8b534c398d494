// common.cuh -- constants and closed forms shared by the selection and the
// attention kernels (and their host launchers).
#pragma once

#include <cstdint>

namespace spa {

constexpr uint32_t kTileBytes = 128u * 128u * 2u;       // one 128x128 bf16 tile
constexpr uint32_t kHalfBytes = kTileBytes / 2u;        // 128 rows x 64 columns
constexpr int kKmeanChunks = 64;                        // K-mean partial sums per (b, kv head)

enum : int { kModeAnchor = 0, kModeSale = 1, kModeDense = 2 };

// sum_{q < n} max(0, (q+1)*bq - A): closed-form prefix of the per-block
// candidate capacity max(0, ls_q - sink) with A = local + sink.
__host__ __device__ __forceinline__ long long cap_prefix(long long n, long long bq, long long A) {
  long long q0 = A / bq;
  if (n <= q0) return 0;
  long long cnt = n - q0;
  return bq * ((n * (n + 1) - q0 * (q0 + 1)) / 2) - cnt * A;
}

// Candidate key tiles.  The candidates of query block q, [sink, ls_q) with
// ls_q = (q + 1) * 128 - local a multiple of 128, lie in the 128-key tiles
// kt0 <= kt < ls_q / 128, kt0 = sink / 128: tmask_tiles(q, c) of them with
// c = tmask_c(sink, local).  The plan writes one 128-bit mask per such tile
// (bit k of word w <=> key 128 kt + 32 w + k kept); the masks of block q start
// at tile tmask_prefix(q, c) of its head's region.
__host__ __device__ __forceinline__ int tmask_c(int sink, int local) {
  return 1 - local / 128 - sink / 128;
}
__host__ __device__ __forceinline__ int tmask_tiles(int q, int c) { return q + c > 0 ? q + c : 0; }
__host__ __device__ __forceinline__ long long tmask_prefix(long long n, int c) {
  const long long m = n + c;
  return m > 0 ? m * (m - 1) / 2 : 0;
}

// Tile bitmaps.  Beside the masks the plan writes, per (b, h, query block),
// three bitmaps over the block's candidate tiles (bit t of word t / 32 <=>
// candidate tile kt0 + t), each tmask_bit_words(nqb, c) words long:
// non-empty (some key kept), dense (at least tile_dense_min(unit) keys kept)
// and full (all 128 keys kept).  The paired attention kernel walks its tiles
// from them: a tile a head pair keeps densely is loaded whole, the keys of
// the others are gathered.  Keys selected one by one (unit 1) gather row by
// row, so a tile half kept is cheaper loaded whole; key blocks of 16 or more
// keys (SALE) gather as whole boxes, so only a full tile is loaded whole.
__host__ __device__ __forceinline__ int tile_dense_min(int unit) { return unit > 1 ? 128 : 64; }
__host__ __device__ __forceinline__ int tmask_bit_words(int nqb, int c) {
  return (tmask_tiles(nqb - 1, c) + 31) / 32;
}

}  // namespace spa
