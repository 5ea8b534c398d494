// key_mass.cuh -- attention mass each key receives from the prefill rows,
// reusing the prefill's log-sum-exp (KVpop, Sec. 3: the future attention mass
// of a token, recovered by a transposed attention pass that reuses the sparse
// LSE normalisers and aggregates over the query heads sharing a kv head):
//
//   mass[b, g, j] = sum_{h in kv head g} sum_{i : j in K_i, i - j >= window}
//                   exp(s_ij - LSE[b, h, i]),
//
// K_i the kept set of row i in the plan (sink + selected + local, causal).
//
// One CTA = one 128-row query block of one q head, walking the block's key
// tiles as the attention does.  Per tile: S = Q K^T on the tensor cores
// (bf16, fp32 in TMEM); the softmax warps write P = 2^(s log2e scale -
// LSE_i log2e) as bf16 into shared memory as the MN-major B operand of a
// second MMA, ones(128 x 128) . P, whose every row is the tile's column sums;
// a seventh warp reads those 128 sums from TMEM and adds them to mass[] with
// global atomics (selected tiles through the block's list).  The window
// test needs each key's index: on sink and local tiles it is key0 + column;
// selected keys lie below ls = row0 + 128 - local, so every one of them
// passes when window <= local - 128, which the API requires.
//
// Roles (224 threads):
//   warp 0     TMA producer: Q once, K tiles into a 2-stage ring;
//   warp 1     TMEM allocation; one thread issues S_t = Q K_t^T and
//              C_{t-1} = ones . P_{t-1};
//   warps 2-5  thread = query row: P_t into shared memory;
//   warp 6     column sums C_t -> atomics.
// TMEM columns: S0 [0,128)  S1 [128,256)  C0 [256,384)  C1 [384,512).
#pragma once

#include "common.cuh"
#include "ptx.cuh"
#include "tiles.cuh"

namespace spa {

constexpr int kMassThreads = 224;
constexpr int kMassStages = 2;
constexpr uint32_t kMassBarBytes = 256u;
// Q, K ring, two P buffers, the ones tile, barriers
constexpr uint32_t kMassSmemBytes =
    1024u + kTileBytes + kMassStages * kTileBytes + 2u * kTileBytes + kTileBytes + kMassBarBytes;
static_assert(kMassSmemBytes <= 232448u, "more shared memory than a CTA may use");

struct MassArgs {
  TileGeom g;
  float sl2;                  // softmax scale * log2(e)
  int window;                 // rows i contribute to key j only when i - j >= window
  const float* lse;           // [B*Hq][L], natural log
  float* mass;                // [B*Hkv][L]
  uint32_t* err;
  uint64_t wait_ns;
};

__global__ void __launch_bounds__(kMassThreads, 1)
key_mass_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_kg, const MassArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t s_base = smem_u32(smem);
  const uint32_t s_q = s_base;
  auto s_k = [&](int st) { return s_base + kTileBytes * (1u + st); };
  auto s_p = [&](int b) { return s_base + kTileBytes * (1u + kMassStages + b); };
  const uint32_t s_ones = s_base + kTileBytes * (3u + kMassStages);
  uint8_t* bar_area = smem + kTileBytes * (4u + kMassStages);
  const uint32_t b0 = smem_u32(bar_area);
  const uint32_t bar_q = b0;
  auto bar_kfull = [&](int s) { return b0 + 8u * (1 + s); };
  auto bar_kempty = [&](int s) { return b0 + 8u * (1 + kMassStages + s); };
  const uint32_t bar_sfull0 = b0 + 8u * (1 + 2 * kMassStages);
  const uint32_t bar_sfree0 = bar_sfull0 + 16u;
  const uint32_t bar_pfull0 = bar_sfull0 + 32u;
  const uint32_t bar_pfree0 = bar_sfull0 + 48u;
  const uint32_t bar_cfull0 = bar_sfull0 + 64u;
  const uint32_t bar_cfree0 = bar_sfull0 + 80u;
  const uint32_t bar_drain = bar_sfull0 + 96u;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bar_area + 8 * (1 + 2 * kMassStages) + 104);
  volatile uint32_t* abort_flag = tmem_holder + 1;
  static_assert(8 * (1 + 2 * kMassStages) + 104 + 8 <= kMassBarBytes, "barrier area");

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < kMassStages; ++s) {
      mbar_init(bar_kfull(s), 1);
      mbar_init(bar_kempty(s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_sfull0 + 8u * i, 1);
      mbar_init(bar_sfree0 + 8u * i, 128);
      mbar_init(bar_pfull0 + 8u * i, 128);
      mbar_init(bar_pfree0 + 8u * i, 1);
      mbar_init(bar_cfull0 + 8u * i, 1);
      mbar_init(bar_cfree0 + 8u * i, 32);
    }
    mbar_init(bar_drain, 1);
    *abort_flag = 0u;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), 512);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_kg);
  }
  // the constant A operand: 128 x 128 bf16 ones (every swizzle of it is itself)
  {
    uint4* ones = reinterpret_cast<uint4*>(smem + kTileBytes * (3u + kMassStages));
    const uint4 w = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
    for (int i = threadIdx.x; i < (int)(kTileBytes / 16); i += kMassThreads) ones[i] = w;
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitCtx wc{abort_flag, a.err, a.wait_ns};

  const BlockTiles it = block_tiles(a.g, blockIdx.x);
  const int T = it.n_sink_t + it.n_sel_t + it.n_loc_t;
  const int kv_row0 = (it.b * a.g.Hkv + it.kvh) * a.g.L;

  if (warp == 0) {
    // ------------------------------------------------------------- producer
    int issued = 0;
    if (lane == 0) {
      mbar_arrive_expect_tx(bar_q, kTileBytes);
      const int qrow = (it.b * a.g.Hq + it.h) * a.g.L + it.row0;
      tma_load_2d(s_q, &tm_q, bar_q, 0, qrow);
      tma_load_2d(s_q + kHalfBytes, &tm_q, bar_q, 64, qrow);
    }
    for (int t = 0; t < T; ++t) {
      const int st = t % kMassStages;
      if (t >= kMassStages) {
        if (!warp_wait(bar_kempty(st), ((t / kMassStages) - 1) & 1, wc)) break;
      }
      const Tile td = tile_of(it, t);
      const uint32_t kf = bar_kfull(st);
      if (!td.gather) {
        if (lane == 0) {
          mbar_arrive_expect_tx(kf, kTileBytes);
          tma_load_2d(s_k(st), &tm_k, kf, 0, kv_row0 + td.key0);
          tma_load_2d(s_k(st) + kHalfBytes, &tm_k, kf, 64, kv_row0 + td.key0);
        }
      } else {
        int j[4];
        const int first = selected_key(a.g, it, td.key0);
        bool bad = false;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int row = lane * 4 + r;
          j[r] = row < td.valid ? selected_key(a.g, it, td.key0 + row) : first;
          if (j[r] < 0 || j[r] >= a.g.L) {
            bad = true;
            j[r] = 0;
          }
        }
        if (bad) atomicOr(a.err, kErrBadIndex);
        // 128 consecutive keys (a near-dense selection): two tiled copies
        const int last = __shfl_sync(0xffffffffu, j[3], 31);
        // (every lane's four keys exactly the next ones: a list entry out of
        // order or repeated keeps the gather path)
        const bool contiguous = td.valid == 128 && last - first == 127 && first >= 0 &&
                                last < a.g.L &&
                                __all_sync(0xffffffffu, j[0] == first + 4 * lane &&
                                                            j[1] == first + 4 * lane + 1 &&
                                                            j[2] == first + 4 * lane + 2 &&
                                                            j[3] == first + 4 * lane + 3);
        if (lane == 0) mbar_arrive_expect_tx(kf, kTileBytes);
        __syncwarp();
        if (contiguous) {
          if (lane == 0) {
            tma_load_2d(s_k(st), &tm_k, kf, 0, kv_row0 + first);
            tma_load_2d(s_k(st) + kHalfBytes, &tm_k, kf, 64, kv_row0 + first);
          }
        } else {
          const uint32_t roff = lane * 4u * 128u;
          tma_gather4(s_k(st) + roff, &tm_kg, kf, 0, kv_row0 + j[0], kv_row0 + j[1],
                      kv_row0 + j[2], kv_row0 + j[3]);
          tma_gather4(s_k(st) + kHalfBytes + roff, &tm_kg, kf, 64, kv_row0 + j[0],
                      kv_row0 + j[1], kv_row0 + j[2], kv_row0 + j[3]);
        }
      }
      issued = t + 1;
    }
    if (lane == 0) {
      mbar_drain(bar_q, 0, a.wait_ns);
      for (int t = max(0, issued - kMassStages); t < issued; ++t)
        mbar_drain(bar_kfull(t % kMassStages), (t / kMassStages) & 1, a.wait_ns);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(bar_q, 0, wc);
      auto issue_cs = [&](int u) -> bool {
        const int bu = u & 1;
        if (!mbar_wait(bar_pfull0 + 8u * bu, (u >> 1) & 1, wc)) return false;
        if (u >= 2 && !mbar_wait(bar_cfree0 + 8u * bu, ((u - 2) >> 1) & 1, wc)) return false;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          // K = 16 query rows per MMA: A = ones (K-major), B = P (MN-major, two
          // 64-key chunks 16 KiB apart)
          const uint32_t aoff = (ks >> 2) * kHalfBytes + (ks & 3) * 32u;
          mma_bf16_ss(tmem + 256u + 128u * bu, smem_desc_sw128(s_ones + aoff, 16),
                      smem_desc_sw128(s_p(bu) + ks * 2048u, kHalfBytes), kIdescPV,
                      ks > 0 ? 1u : 0u);
        }
        mma_commit(bar_cfull0 + 8u * bu);
        mma_commit(bar_pfree0 + 8u * bu);
        return true;
      };
      for (int t = 0; ok && t < T; ++t) {
        const int st = t % kMassStages, b = t & 1;
        if (!(ok = mbar_wait(bar_kfull(st), (t / kMassStages) & 1, wc))) break;
        if (t >= 2 && !(ok = mbar_wait(bar_sfree0 + 8u * b, ((t - 2) >> 1) & 1, wc))) break;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t off = (ks >> 2) * kHalfBytes + (ks & 3) * 32u;
          mma_bf16_ss(tmem + 128u * b, smem_desc_sw128(s_q + off, 16),
                      smem_desc_sw128(s_k(st) + off, 16), kIdescQK, ks > 0 ? 1u : 0u);
        }
        mma_commit(bar_sfull0 + 8u * b);
        mma_commit(bar_kempty(st));
        if (t >= 1) ok = issue_cs(t - 1);
      }
      if (ok && T > 0) issue_cs(T - 1);
      mma_commit(bar_drain);
      mbar_drain(bar_drain, 0, a.wait_ns);
    }
    __syncwarp();
  } else if (warp < 6) {
    // ------------------------------------------------------ P = 2^(s - LSE)
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int row = it.row0 + r;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const long long bh = (long long)it.b * a.g.Hq + it.h;
    const float lse2 = row < a.g.L ? a.lse[bh * a.g.L + row] * 1.4426950408889634f : INFINITY;
    const float sl2 = a.sl2;
    for (int t = 0; t < T; ++t) {
      const int b = t & 1;
      if (!warp_wait(bar_sfull0 + 8u * b, (t >> 1) & 1, wc)) break;
      tc_fence_after();
      uint32_t sr[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tmem + lane_off + 128u * b + 32u * c, sr[c]);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(bar_sfree0 + 8u * b);

      const Tile td = tile_of(it, t);
      // columns [0, limit) count; on contiguous tiles also key <= row - window
      int limit = td.valid;
      if (!td.gather) limit = min(limit, row - a.window - td.key0 + 1);
      if (row >= a.g.L) limit = 0;
      if (limit < 0) limit = 0;
      if (t >= 2 && !warp_wait(bar_pfree0 + 8u * b, ((t - 2) >> 1) & 1, wc)) break;
      uint8_t* prow = smem + (s_p(b) - s_base);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          uint32_t w[4];
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) {
            const int col = c * 32 + m * 8 + e2 * 2;
            const float p0 = col < limit
                                 ? fast_exp2(fmaf(__uint_as_float(sr[c][m * 8 + e2 * 2]), sl2, -lse2))
                                 : 0.f;
            const float p1 = col + 1 < limit
                                 ? fast_exp2(fmaf(__uint_as_float(sr[c][m * 8 + e2 * 2 + 1]), sl2, -lse2))
                                 : 0.f;
            w[e2] = pack_bf16x2(p0, p1);
          }
          // keys c*32 + m*8 .. +7: chunk (c >> 1), byte (c & 1) * 64 + m * 16 of row r
          *reinterpret_cast<uint4*>(prow + (c >> 1) * kHalfBytes +
                                    sw128_offset(r, (c & 1) * 64 + m * 16)) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(bar_pfull0 + 8u * b);
    }
  } else {
    // ------------------------------------------------- column sums -> mass
    // warp 6 reads TMEM lanes 64..95; every row of C holds the same sums
    const uint32_t lane_off = 64u << 16;
    float* mass = a.mass + (long long)(it.b * a.g.Hkv + it.kvh) * a.g.L;
    for (int t = 0; t < T; ++t) {
      const int b = t & 1;
      if (!warp_wait(bar_cfull0 + 8u * b, (t >> 1) & 1, wc)) break;
      tc_fence_after();
      float v[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t cr[32];
        tmem_ld32(tmem + lane_off + 256u + 128u * b + 32u * c, cr);
        tmem_ld_wait();
        float x = 0.f;
#pragma unroll
        for (int e = 0; e < 32; ++e) x = (e == lane) ? __uint_as_float(cr[e]) : x;
        v[c] = x;
      }
      tc_fence_before();
      mbar_arrive(bar_cfree0 + 8u * b);
      const Tile td = tile_of(it, t);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int col = c * 32 + lane;
        if (col >= td.valid || v[c] == 0.f) continue;
        int key = td.gather ? selected_key(a.g, it, td.key0 + col) : td.key0 + col;
        if (key < 0 || key >= a.g.L) {
          atomicOr(a.err, kErrBadIndex);
          continue;
        }
        atomicAdd(mass + key, v[c]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace spa
