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

}  // namespace spa
