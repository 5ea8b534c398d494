// select.cuh -- anchor-mode key selection (AnchorAttention: Difference-Aware
// Sparse Attention with Stripe Granularity, Eq. (1)-(3)) and the generic
// bitmask -> ascending-index-list compaction shared with SALE mode.
//
//   anchor_pool_kernel   per query block: S = Q [K_sink; K_local]^T on the
//                        tensor cores, row max over the causal sink-local
//                        keys (Eq. (1), the row-max buffer M), its mean over
//                        the block (avgpool(x_a)), and the pooled query
//                        avgpool(Q) * scale split into bf16 hi + lo parts.
//   stripe_scan_kernel   per (128 query blocks) x (16 key tiles): the pooled
//                        scores avgpool(Q) K^T * scale as one tcgen05 GEMM
//                        (hi and lo products accumulated in fp32), the
//                        difference-aware test of Eq. (2) and the candidate
//                        range check, written as a key bitmask per block.
//   stripe_select_kernel the scan fused with the compaction (no bitmask):
//                        per M tile of query blocks, kept keys appended to
//                        each block's list in key order; used when the
//                        selection groups fit in a warp (step <= 32, power
//                        of two).
//   compact_kernel       per query block: the bitmask's set bits in
//                        ascending order, written with coalesced warp stores
//                        into the block's list (Eq. (3): discrete key
//                        coordinates), plus the count.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace spa {

// ---------------------------------------------------------------------------
// anchor + pooling
// ---------------------------------------------------------------------------
// One CTA streams kPoolQbs consecutive query blocks of one q head: warp 0
// loads each block's Q tile (2-stage ring) and its sink and local K tiles
// (3-stage ring); warp 1 issues S = Q K^T per key tile into three TMEM
// accumulators and, per block, the column sums of Q as one more MMA,
// ones(128 x 128) * Q, into a fourth (every row of it holds the sums);
// warps 2-9 (two per TMEM lane quadrant, 64 columns each) take the causal
// row max of every tile.  Per block the two halves are combined through
// shared memory behind a bounded mbarrier wait: x_a = max * scale, its mean
// over the block's rows, and avgpool(Q) * scale split into bf16 hi + lo.  A
// last block shorter than 128 rows sums its valid Q rows on the CUDA cores
// instead (the tile's other rows belong to the next head).
constexpr int kPoolQbs = 8;
constexpr int kPoolThreads = 320;
constexpr int kPoolQStages = 2;
constexpr int kPoolKStages = 3;
constexpr int kPoolBufs = 3;                  // S accumulators; TMEM columns [384, 512) hold the sums
constexpr uint32_t kPoolBarBytes = 8192u;
constexpr uint32_t kPoolSmemBytes =
    1024u + (kPoolQStages + kPoolKStages + 1) * kTileBytes + kPoolBarBytes;   // + the ones tile
static_assert(kPoolSmemBytes <= 232448u, "more shared memory than a CTA may use");

struct PoolArgs {
  int B, Hq, Hkv, L, nqb, group;
  int sink, local;
  float scale;                  // softmax scale
  float* xbar;                  // [B*Hq*nqb]
  __nv_bfloat16* qbar;          // [2][B*Hq][nqb][128]: hi then lo
  uint32_t* err;
  uint64_t wait_ns;
  int groups;                   // ceil(nqb / kPoolQbs)
};

__global__ void __launch_bounds__(kPoolThreads, 1)
anchor_pool_kernel(const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_k, const PoolArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t s_base = smem_u32(smem);
  auto s_q = [&](int st) { return s_base + st * kTileBytes; };
  auto s_k = [&](int st) { return s_base + (kPoolQStages + st) * kTileBytes; };
  const uint32_t s_ones = s_base + (kPoolQStages + kPoolKStages) * kTileBytes;
  uint8_t* bar_area = smem + (kPoolQStages + kPoolKStages + 1) * kTileBytes;
  const uint32_t b0 = smem_u32(bar_area);
  auto bar_qfull = [&](int s) { return b0 + 8u * s; };
  auto bar_qempty = [&](int s) { return b0 + 8u * (2 + s); };
  auto bar_kfull = [&](int s) { return b0 + 8u * (4 + s); };
  auto bar_kempty = [&](int s) { return b0 + 8u * (7 + s); };
  auto bar_sfull = [&](int s) { return b0 + 8u * (10 + s); };
  auto bar_sfree = [&](int s) { return b0 + 8u * (14 + s); };
  auto bar_x = [&](int s) { return b0 + 8u * (18 + s); };       // halves combined
  auto bar_r = [&](int s) { return b0 + 8u * (20 + s); };       // row sums per quadrant
  const uint32_t bar_drain = b0 + 8u * 22;
  const uint32_t bar_pfull = b0 + 8u * 23;                      // column sums in TMEM
  const uint32_t bar_pfree = b0 + 8u * 24;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bar_area + 256);
  volatile uint32_t* abort_flag = tmem_holder + 1;
  float* x_max = reinterpret_cast<float*>(bar_area + 512);      // [2][2 halves][128]
  float* x_red = reinterpret_cast<float*>(bar_area + 4608);     // [2][4 quadrants]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = static_cast<int>(blockIdx.x) / a.groups;
  const int grp = static_cast<int>(blockIdx.x) - bh * a.groups;
  const int qb0 = grp * kPoolQbs;
  const int nq = min(kPoolQbs, a.nqb - qb0);
  const int b = bh / a.Hq, h = bh - b * a.Hq;
  const int kv_row0 = (b * a.Hkv + h / a.group) * a.L;
  // tiles of block qb: sink tiles [0, sink_end), then local tiles [ls, le)
  auto geom = [&](int qb, int& ls, int& le, int& sink_end, int& n_sink_t, int& T) {
    const int row0 = qb * 128;
    le = min(row0 + 128, a.L);
    ls = max(0, row0 + 128 - a.local);
    sink_end = min(a.sink, ls);
    n_sink_t = (sink_end + 127) / 128;
    T = n_sink_t + (le - ls + 127) / 128;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPoolQStages; ++s) {
      mbar_init(bar_qfull(s), 1);
      mbar_init(bar_qempty(s), 1 + 128);            // the MMAs' commit + the q-bar threads
    }
    mbar_init(bar_pfull, 1);
    mbar_init(bar_pfree, 128);
    for (int s = 0; s < kPoolKStages; ++s) {
      mbar_init(bar_kfull(s), 1);
      mbar_init(bar_kempty(s), 1);
    }
    for (int s = 0; s < kPoolBufs; ++s) {
      mbar_init(bar_sfull(s), 1);
      mbar_init(bar_sfree(s), 256);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar_x(s), 256);
      mbar_init(bar_r(s), 128);
    }
    mbar_init(bar_drain, 1);
    *abort_flag = 0u;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), 512);
    tmem_relinquish();
  }
  {  // the all-ones A operand of the column-sum MMA (1.0 in bf16; any swizzle)
    uint4* ones = reinterpret_cast<uint4*>(smem + (s_ones - s_base));
    for (int i = threadIdx.x; i < static_cast<int>(kTileBytes / 16); i += blockDim.x)
      ones[i] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
  }
  fence_proxy_async_smem();                         // generic-proxy writes -> tensor-core reads
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitCtx wc{abort_flag, a.err, a.wait_ns};

  if (warp == 0) {
    if (lane == 0) {
      int gk = 0, issued_q = 0;
      bool ok = true;
      for (int i = 0; ok && i < nq; ++i) {
        const int qb = qb0 + i, qs = i % kPoolQStages;
        int ls, le, sink_end, n_sink_t, T;
        geom(qb, ls, le, sink_end, n_sink_t, T);
        if (i >= kPoolQStages &&
            !(ok = mbar_wait(bar_qempty(qs), ((i / kPoolQStages) - 1) & 1, wc)))
          break;
        mbar_arrive_expect_tx(bar_qfull(qs), kTileBytes);
        const int qrow = bh * a.L + qb * 128;
        tma_load_2d(s_q(qs), &tm_q, bar_qfull(qs), 0, qrow);
        tma_load_2d(s_q(qs) + kHalfBytes, &tm_q, bar_qfull(qs), 64, qrow);
        issued_q = i + 1;
        for (int t = 0; t < T; ++t, ++gk) {
          const int ks = gk % kPoolKStages;
          if (gk >= kPoolKStages &&
              !(ok = mbar_wait(bar_kempty(ks), ((gk / kPoolKStages) - 1) & 1, wc)))
            break;
          const int key0 = t < n_sink_t ? t * 128 : ls + (t - n_sink_t) * 128;
          mbar_arrive_expect_tx(bar_kfull(ks), kTileBytes);
          tma_load_2d(s_k(ks), &tm_k, bar_kfull(ks), 0, kv_row0 + key0);
          tma_load_2d(s_k(ks) + kHalfBytes, &tm_k, bar_kfull(ks), 64, kv_row0 + key0);
        }
      }
      // no copy may still be in flight when the CTA exits
      for (int i = max(0, issued_q - kPoolQStages); i < issued_q; ++i)
        mbar_drain(bar_qfull(i % kPoolQStages), (i / kPoolQStages) & 1, a.wait_ns);
      for (int g = max(0, gk - kPoolKStages); g < gk; ++g)
        mbar_drain(bar_kfull(g % kPoolKStages), (g / kPoolKStages) & 1, a.wait_ns);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      int gk = 0;
      bool ok = true;
      for (int i = 0; ok && i < nq; ++i) {
        const int qb = qb0 + i, qs = i % kPoolQStages;
        int ls, le, sink_end, n_sink_t, T;
        geom(qb, ls, le, sink_end, n_sink_t, T);
        if (!(ok = mbar_wait(bar_qfull(qs), (i / kPoolQStages) & 1, wc))) break;
        for (int t = 0; t < T; ++t, ++gk) {
          const int ks = gk % kPoolKStages, bb = gk % kPoolBufs;
          if (!(ok = mbar_wait(bar_kfull(ks), (gk / kPoolKStages) & 1, wc))) break;
          if (gk >= kPoolBufs && !(ok = mbar_wait(bar_sfree(bb), ((gk / kPoolBufs) - 1) & 1, wc)))
            break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32u;
            mma_bf16_ss(tmem + 128u * bb, smem_desc_sw128(s_q(qs) + off, 16),
                        smem_desc_sw128(s_k(ks) + off, 16), kIdescQK, kk > 0 ? 1u : 0u);
          }
          mma_commit(bar_sfull(bb));
          mma_commit(bar_kempty(ks));
        }
        if (!ok) break;
        // column sums of Q: ones(128 x 128) * Q, Q read as a (rows x d) MN-major operand
        if (i > 0 && !(ok = mbar_wait(bar_pfree, (i - 1) & 1, wc))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32u;
          mma_bf16_ss(tmem + 384u, smem_desc_sw128(s_ones + off, 16),
                      smem_desc_sw128(s_q(qs) + kk * 2048u, kHalfBytes), kIdescPV,
                      kk > 0 ? 1u : 0u);
        }
        mma_commit(bar_pfull);
        mma_commit(bar_qempty(qs));                    // Q no longer read by the MMAs
      }
      mma_commit(bar_drain);
      mbar_drain(bar_drain, 0, a.wait_ns);
    }
    __syncwarp();
  } else {
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;              // columns [64 half, 64 half + 64), rows likewise
    const int r = quad * 32 + lane;                // TMEM lane = query row; also the Q column summed
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t dhalf = (r >> 6) * kHalfBytes;  // Q column r: 64-column half and byte offset
    const uint32_t dbyte = (r & 63) * 2;
    int gb = 0;
    for (int i = 0; i < nq; ++i) {
      const int qb = qb0 + i, qs = i % kPoolQStages, xs = i & 1;
      int ls, le, sink_end, n_sink_t, T;
      geom(qb, ls, le, sink_end, n_sink_t, T);
      const int row0 = qb * 128;
      const int nrows = le - row0;
      if (!warp_wait(bar_qfull(qs), (i / kPoolQStages) & 1, wc)) break;
      // a short last block: its valid rows' column sums on the CUDA cores
      float col_short = 0.f;
      if (half == 1) {
        if (nrows < 128) {
          const uint8_t* qt = smem + (s_q(qs) - s_base);
          float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;   // four independent chains
          int rr = 0;
          for (; rr + 4 <= nrows; rr += 4) {
            p0 += __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(qt + dhalf + sw128_offset(rr, dbyte)));
            p1 += __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(qt + dhalf + sw128_offset(rr + 1, dbyte)));
            p2 += __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(qt + dhalf + sw128_offset(rr + 2, dbyte)));
            p3 += __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(qt + dhalf + sw128_offset(rr + 3, dbyte)));
          }
          for (; rr < nrows; ++rr)
            p0 += __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(qt + dhalf + sw128_offset(rr, dbyte)));
          col_short = (p0 + p1) + (p2 + p3);
        }
        mbar_arrive(bar_qempty(qs));
      }
      // causal row max over this half's columns of the block's key tiles
      float mx = -INFINITY;
      bool ok = true;
      for (int t = 0; t < T; ++t, ++gb) {
        const int bb = gb % kPoolBufs;
        if (!(ok = warp_wait(bar_sfull(bb), (gb / kPoolBufs) & 1, wc))) break;
        tc_fence_after();
        uint32_t sr[2][32];
#pragma unroll
        for (int c = 0; c < 2; ++c)
          tmem_ld32(tmem + lane_off + 128u * bb + 64u * half + 32u * c, sr[c]);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(bar_sfree(bb));
        const int key0 = (t < n_sink_t ? t * 128 : ls + (t - n_sink_t) * 128) + 64 * half;
        // valid keys: sink tiles below sink_end; local tiles causal (j <= i) and below L
        int limit = (t < n_sink_t) ? (sink_end - key0) : min(le - key0, row0 + r - key0 + 1);
        limit = max(0, min(limit, 64));
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        if (limit == 64) {                             // whole half tile valid
#pragma unroll
          for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int e = 0; e < 32; ++e) m4[e & 3] = fmaxf(m4[e & 3], __uint_as_float(sr[c][e]));
        } else {
#pragma unroll
          for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (c * 32 + e < limit) m4[e & 3] = fmaxf(m4[e & 3], __uint_as_float(sr[c][e]));
        }
        mx = fmaxf(mx, fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])));
      }
      if (!ok) break;
      // combine the two halves
      x_max[(xs * 2 + half) * 128 + r] = mx;
      mbar_arrive(bar_x(xs));
      if (!warp_wait(bar_x(xs), (i >> 1) & 1, wc)) break;
      if (half == 0) {
        const float m = fmaxf(x_max[(xs * 2) * 128 + r], x_max[(xs * 2 + 1) * 128 + r]);
        float s = r < nrows ? m * a.scale : 0.f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) x_red[xs * 4 + quad] = s;
        mbar_arrive(bar_r(xs));
        if (!warp_wait(bar_r(xs), (i >> 1) & 1, wc)) break;
        if (r == 0)
          a.xbar[(long long)bh * a.nqb + qb] =
              (x_red[xs * 4 + 0] + x_red[xs * 4 + 1] + x_red[xs * 4 + 2] + x_red[xs * 4 + 3]) /
              static_cast<float>(nrows);
      } else {
        // pooled query, column d = r: every TMEM row of the column-sum MMA holds
        // the sums, so this thread takes column r from its own row
        if (!warp_wait(bar_pfull, i & 1, wc)) break;
        tc_fence_after();
        uint32_t cs[32];
        tmem_ld32(tmem + lane_off + 384u + 32u * quad, cs);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(bar_pfree);
        float sum = 0.f;
#pragma unroll
        for (int e = 0; e < 32; ++e) sum = e == lane ? __uint_as_float(cs[e]) : sum;
        if (nrows < 128) sum = col_short;
        const float qbar = (sum / static_cast<float>(nrows)) * a.scale;
        const __nv_bfloat16 hi = __float2bfloat16_rn(qbar);
        const __nv_bfloat16 lo = __float2bfloat16_rn(qbar - __bfloat162float(hi));
        const long long base = ((long long)bh * a.nqb + qb) * 128 + r;
        const long long lo_off = (long long)a.B * a.Hq * a.nqb * 128;
        a.qbar[base] = hi;
        a.qbar[lo_off + base] = lo;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------------------
// pooled-score scan: bitmask[bh][qb][word] over keys
// ---------------------------------------------------------------------------
// One CTA: 128 query blocks (rows of the pooled-Q tile) x up to 16 key tiles.
// Four TMEM accumulators of 128 columns let the MMA run three tiles ahead of
// the epilogue; warps 2-9 each own one TMEM lane quadrant and 64 columns.
constexpr int kScanThreads = 320;
constexpr int kScanStages = 3;
constexpr int kScanBufs = 4;
constexpr int kScanTilesPerChunk = 16;
constexpr uint32_t kScanSmemBytes = 1024u + 2u * kTileBytes + kScanStages * kTileBytes + 512u;
static_assert(kScanSmemBytes <= 232448u, "more shared memory than a CTA may use");

struct ScanArgs {
  int B, Hq, Hkv, L, nqb, group;
  int sink, local;
  float theta;
  const float* xbar;
  uint32_t* mask;        // [B*Hq*nqb][nwords]
  int nwords;            // words per block row (multiple of 4)
  uint32_t* err;
  uint64_t wait_ns;
};

__global__ void __launch_bounds__(kScanThreads, 1)
stripe_scan_kernel(const __grid_constant__ CUtensorMap tm_qbar,
                   const __grid_constant__ CUtensorMap tm_k, const ScanArgs a) {
  const int bh = blockIdx.z;
  const int mt = blockIdx.y;
  const int chunk = blockIdx.x;
  const int qb_lo = mt * 128;
  const int qb_hi = min(qb_lo + 128, a.nqb);
  const int key_end = max(0, qb_hi * 128 - a.local);      // ls of the last block
  if (key_end <= a.sink) return;
  const int kt0 = a.sink / 128;
  const int kt_end = (key_end + 127) / 128;
  const int t_lo = kt0 + chunk * kScanTilesPerChunk;
  const int t_hi = min(t_lo + kScanTilesPerChunk, kt_end);
  if (t_lo >= t_hi) return;
  const int T = t_hi - t_lo;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t s_base = smem_u32(smem);
  const uint32_t s_a = s_base;                            // hi tile, then lo tile
  auto s_k = [&](int st) { return s_base + 2u * kTileBytes + st * kTileBytes; };
  uint8_t* bar_area = smem + 2 * kTileBytes + kScanStages * kTileBytes;
  const uint32_t b0 = smem_u32(bar_area);
  const uint32_t bar_a = b0;
  auto bar_full = [&](int st) { return b0 + 8u * (1 + st); };
  auto bar_empty = [&](int st) { return b0 + 8u * (1 + kScanStages + st); };
  auto bar_sfull = [&](int bb) { return b0 + 8u * (1 + 2 * kScanStages + bb); };
  auto bar_sfree = [&](int bb) { return b0 + 8u * (1 + 2 * kScanStages + kScanBufs + bb); };
  const uint32_t bar_drain = b0 + 8u * (1 + 2 * kScanStages + 2 * kScanBufs);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bar_area + 256);
  volatile uint32_t* abort_flag = tmem_holder + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(bar_a, 1);
    for (int st = 0; st < kScanStages; ++st) {
      mbar_init(bar_full(st), 1);
      mbar_init(bar_empty(st), 1);
    }
    for (int i = 0; i < kScanBufs; ++i) {
      mbar_init(bar_sfull(i), 1);
      mbar_init(bar_sfree(i), 256);
    }
    mbar_init(bar_drain, 1);
    *abort_flag = 0u;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitCtx wc{abort_flag, a.err, a.wait_ns};
  const int b = bh / a.Hq, h = bh - b * a.Hq;
  const int kv_row0 = (b * a.Hkv + h / a.group) * a.L;
  const int BH = a.B * a.Hq;

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(bar_a, 2 * kTileBytes);
      tma_load_3d(s_a, &tm_qbar, bar_a, 0, qb_lo, bh);
      tma_load_3d(s_a + kHalfBytes, &tm_qbar, bar_a, 64, qb_lo, bh);
      tma_load_3d(s_a + kTileBytes, &tm_qbar, bar_a, 0, qb_lo, BH + bh);
      tma_load_3d(s_a + kTileBytes + kHalfBytes, &tm_qbar, bar_a, 64, qb_lo, BH + bh);
      int issued = 0;
      for (int t = 0; t < T; ++t) {
        const int st = t % kScanStages;
        if (t >= kScanStages && !mbar_wait(bar_empty(st), ((t / kScanStages) - 1) & 1, wc)) break;
        const int key0 = (t_lo + t) * 128;
        mbar_arrive_expect_tx(bar_full(st), kTileBytes);
        tma_load_2d(s_k(st), &tm_k, bar_full(st), 0, kv_row0 + key0);
        tma_load_2d(s_k(st) + kHalfBytes, &tm_k, bar_full(st), 64, kv_row0 + key0);
        issued = t + 1;
      }
      {  // no copy may still be in flight when the CTA exits
        mbar_drain(bar_a, 0, a.wait_ns);
        for (int t = max(0, issued - kScanStages); t < issued; ++t)
          mbar_drain(bar_full(t % kScanStages), (t / kScanStages) & 1, a.wait_ns);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = mbar_wait(bar_a, 0, wc);
      for (int t = 0; ok && t < T; ++t) {
        const int st = t % kScanStages, bb = t % kScanBufs;
        if (!(ok = mbar_wait(bar_full(st), (t / kScanStages) & 1, wc))) break;
        if (t >= kScanBufs &&
            !(ok = mbar_wait(bar_sfree(bb), ((t / kScanBufs) - 1) & 1, wc)))
          break;
        tc_fence_after();
#pragma unroll
        for (int part = 0; part < 2; ++part) {       // hi, then lo
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32u;
            mma_bf16_ss(tmem + 128u * bb, smem_desc_sw128(s_a + part * kTileBytes + off, 16),
                        smem_desc_sw128(s_k(st) + off, 16), kIdescQK,
                        (part > 0 || kk > 0) ? 1u : 0u);
          }
        }
        mma_commit(bar_sfull(bb));
        mma_commit(bar_empty(st));
      }
      mma_commit(bar_drain);
      mbar_drain(bar_drain, 0, a.wait_ns);
    }
    __syncwarp();
  } else {
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;            // key columns [64*half, 64*half + 64)
    const int r = quad * 32 + lane;
    const int qb = qb_lo + r;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const bool row_valid = qb < a.nqb;
    const float xb = row_valid ? a.xbar[(long long)bh * a.nqb + qb] : 0.f;
    const int cand_hi = row_valid ? max(0, (qb + 1) * 128 - a.local) : 0;   // ls of this block
    uint32_t* mrow = a.mask + ((long long)bh * a.nqb + (row_valid ? qb : 0)) * a.nwords;
    for (int t = 0; t < T; ++t) {
      const int bb = t % kScanBufs;
      if (!warp_wait(bar_sfull(bb), (t / kScanBufs) & 1, wc)) break;
      tc_fence_after();
      uint32_t sr[2][32];
#pragma unroll
      for (int c = 0; c < 2; ++c) tmem_ld32(tmem + lane_off + 128u * bb + 64u * half + 32u * c, sr[c]);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(bar_sfree(bb));
      const int key0 = (t_lo + t) * 128 + 64 * half;
      // candidate keys of this row inside these 64 columns: [lo, hi)
      const int lo = max(a.sink - key0, 0);
      const int hi = min(cand_hi - key0, 64);
      uint2 wv;
      uint32_t* w = &wv.x;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t bits = 0;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float s = __uint_as_float(sr[c][e]);
          bits |= ((xb - s) <= a.theta ? 1u : 0u) << e;
        }
        const int wlo = c * 32, whi = c * 32 + 32;
        const int l0 = max(lo, wlo) - wlo, l1 = min(hi, whi) - wlo;
        uint32_t range = 0;
        if (l1 > l0) range = (l1 - l0 >= 32 ? 0xffffffffu : ((1u << (l1 - l0)) - 1u)) << l0;
        w[c] = bits & range;
      }
      if (row_valid && key0 < cand_hi) {
        *reinterpret_cast<uint2*>(mrow + key0 / 32) = wv;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------------------
// pooled-score scan fused with compaction: kept-key lists without a bitmask
// ---------------------------------------------------------------------------
// One CTA = one M tile of 128 TMEM lanes = 128 query blocks of one q head,
// or 64 query blocks of each head of a pair (2p, 2p+1) when the attention
// kernel pairs heads (rows 0-63 head 2p, rows 64-127 head 2p+1: both heads
// share the kv head, so each K tile feeds both).  The CTA walks every key tile
// of its candidate range in ascending order and appends each query block's
// kept keys to the block's list at a running offset, so the lists come out
// ascending with no intermediate mask.  It also writes, for every candidate
// tile of every block, the block's 128 keep bits of that tile (the tile masks
// the paired attention kernel cuts its tiles from).  Selection groups
// (step > 1) must lie inside one warp: step a power of two <= 32.
//
// Warp 0 loads the pooled-Q tile once and the K tiles (4-stage ring); warp 1
// issues the hi and lo MMAs into four TMEM accumulators; warps 2-17 each own
// a TMEM lane quadrant and 32 of the 128 columns (one 32-key word per row).
// Per key tile the sixteen warps exchange their words through shared memory
// behind a bounded mbarrier wait, so that every thread knows its row's kept
// count before its word, and the first four warps store each row's four
// words as its tile mask.  Stores, by density of the warp's 32 words: all
// keys kept -- one shuffle and one coalesced store of the same 32 values per
// row; few keys in every word -- each thread stores its own row's keys;
// otherwise row by row over the rows with keys, the row's word and list
// position shuffled to the warp, one coalesced store of its kept keys.  CTAs
// are numbered heaviest first (last M tile first), so the block scheduler
// fills the GPU longest-job-first.
constexpr int kSelEpiWarps = 16;
constexpr int kSelThreads = 32 * (2 + kSelEpiWarps);
constexpr int kSelStages = 4;
constexpr int kSelBufs = 4;
constexpr uint32_t kSelBarBytes = 8192u;    // barriers, TMEM slot, word exchange
constexpr uint32_t kSelSmemBytes = 1024u + 2u * kTileBytes + kSelStages * kTileBytes + kSelBarBytes;
static_assert(kSelSmemBytes <= 232448u, "more shared memory than a CTA may use");

struct SelectArgs {
  int B, Hq, Hkv, L, nqb, group;
  int sink, local, step;
  float theta;
  int heads_per_item;       // 1, or 2 for a head pair
  int rows_per_head;        // 128 / heads_per_item
  int n_mt;                 // M tiles per head
  int n_items_per_mt;       // B * Hq / heads_per_item
  const float* xbar;        // [B*Hq*nqb]
  int* lists;
  long long list_per_head;
  long long cap_a;
  int* counts;              // [B*Hq*nqb]
  uint4* tmask;             // [B*Hq][tmask_per_head] candidate-tile masks
  long long tmask_per_head;
  int tc;                   // tmask_c(sink, local)
  uint32_t* tbits;          // [B*Hq*nqb][3][tbit_words]: non-empty, dense, full tiles
  int tbit_words;
  uint32_t* err;
  uint64_t wait_ns;
};

__global__ void __launch_bounds__(kSelThreads, 1)
stripe_select_kernel(const __grid_constant__ CUtensorMap tm_qbar,
                     const __grid_constant__ CUtensorMap tm_k, const SelectArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t s_base = smem_u32(smem);
  const uint32_t s_a = s_base;                            // hi tile, then lo tile
  auto s_k = [&](int st) { return s_base + 2u * kTileBytes + st * kTileBytes; };
  uint8_t* bar_area = smem + 2 * kTileBytes + kSelStages * kTileBytes;
  const uint32_t b0 = smem_u32(bar_area);
  const uint32_t bar_a = b0;
  auto bar_full = [&](int st) { return b0 + 8u * (1 + st); };
  auto bar_empty = [&](int st) { return b0 + 8u * (1 + kSelStages + st); };
  auto bar_sfull = [&](int bb) { return b0 + 8u * (1 + 2 * kSelStages + bb); };
  auto bar_sfree = [&](int bb) { return b0 + 8u * (1 + 2 * kSelStages + kSelBufs + bb); };
  auto bar_x = [&](int i) { return b0 + 8u * (1 + 2 * kSelStages + 2 * kSelBufs + i); };
  const uint32_t bar_drain = b0 + 8u * (3 + 2 * kSelStages + 2 * kSelBufs);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bar_area + 256);
  volatile uint32_t* abort_flag = tmem_holder + 1;
  uint4* x_words = reinterpret_cast<uint4*>(bar_area + 1024);     // [2][128 rows]: 4 words

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // item: heaviest M tile first
  const int mt = a.n_mt - 1 - static_cast<int>(blockIdx.x) / a.n_items_per_mt;
  const int gi = static_cast<int>(blockIdx.x) % a.n_items_per_mt;
  const int bh0 = gi * a.heads_per_item;                  // b * Hq + first head
  const int R = a.rows_per_head;
  const int qb0 = mt * R;
  const int qb_last = min(qb0 + R, a.nqb) - 1;
  const int key_end = max(0, (qb_last + 1) * 128 - a.local);  // ls of the last block
  const int kt0 = a.sink / 128;
  const int T = key_end > a.sink ? (key_end + 127) / 128 - kt0 : 0;
  const int b = bh0 / a.Hq;
  const int kv_row0 = (b * a.Hkv + (bh0 - b * a.Hq) / a.group) * a.L;
  const int BH = a.B * a.Hq;
  // epilogue row of this thread (warps 2-17): TMEM lane r, key word qtr
  const int quad = warp & 3;
  const int qtr = (warp - 2) >> 2;               // key columns [32*qtr, 32*qtr + 32)
  const int r = quad * 32 + lane;
  const int hs = r / R;                          // head of the pair (0 when unpaired)
  const int qb = qb0 + (r - hs * R);
  const int bh = bh0 + hs;
  const bool row_valid = warp >= 2 && qb < a.nqb;
  int off = 0;                                   // kept keys written so far (this row)

  if (threadIdx.x == 0) {
    mbar_init(bar_a, 1);
    for (int st = 0; st < kSelStages; ++st) {
      mbar_init(bar_full(st), 1);
      mbar_init(bar_empty(st), 1);
    }
    for (int i = 0; i < kSelBufs; ++i) {
      mbar_init(bar_sfull(i), 1);
      mbar_init(bar_sfree(i), kSelEpiWarps);       // one arrival per epilogue warp
    }
    mbar_init(bar_x(0), kSelEpiWarps);
    mbar_init(bar_x(1), kSelEpiWarps);
    mbar_init(bar_drain, 1);
    *abort_flag = 0u;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitCtx wc{abort_flag, a.err, a.wait_ns};

  if (warp == 0) {
    if (lane == 0 && T > 0) {
      mbar_arrive_expect_tx(bar_a, 2 * kTileBytes);
      for (int part = 0; part < 2; ++part)            // hi, then lo
        for (int h2 = 0; h2 < a.heads_per_item; ++h2) {
          const uint32_t dst = s_a + part * kTileBytes + h2 * R * 128u;
          const int plane = part * BH + bh0 + h2;
          tma_load_3d(dst, &tm_qbar, bar_a, 0, qb0, plane);
          tma_load_3d(dst + kHalfBytes, &tm_qbar, bar_a, 64, qb0, plane);
        }
      int issued = 0;
      for (int t = 0; t < T; ++t) {
        const int st = t % kSelStages;
        if (t >= kSelStages && !mbar_wait(bar_empty(st), ((t / kSelStages) - 1) & 1, wc)) break;
        const int key0 = (kt0 + t) * 128;
        mbar_arrive_expect_tx(bar_full(st), kTileBytes);
        tma_load_2d(s_k(st), &tm_k, bar_full(st), 0, kv_row0 + key0);
        tma_load_2d(s_k(st) + kHalfBytes, &tm_k, bar_full(st), 64, kv_row0 + key0);
        issued = t + 1;
      }
      {  // no copy may still be in flight when the CTA exits
        mbar_drain(bar_a, 0, a.wait_ns);
        for (int t = max(0, issued - kSelStages); t < issued; ++t)
          mbar_drain(bar_full(t % kSelStages), (t / kSelStages) & 1, a.wait_ns);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && T > 0) {
      bool ok = mbar_wait(bar_a, 0, wc);
      for (int t = 0; ok && t < T; ++t) {
        const int st = t % kSelStages, bb = t % kSelBufs;
        if (!(ok = mbar_wait(bar_full(st), (t / kSelStages) & 1, wc))) break;
        if (t >= kSelBufs && !(ok = mbar_wait(bar_sfree(bb), ((t / kSelBufs) - 1) & 1, wc)))
          break;
        tc_fence_after();
#pragma unroll
        for (int part = 0; part < 2; ++part) {       // hi, then lo
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off8 = (kk >> 2) * kHalfBytes + (kk & 3) * 32u;
            mma_bf16_ss(tmem + 128u * bb, smem_desc_sw128(s_a + part * kTileBytes + off8, 16),
                        smem_desc_sw128(s_k(st) + off8, 16), kIdescQK,
                        (part > 0 || kk > 0) ? 1u : 0u);
          }
        }
        mma_commit(bar_sfull(bb));
        mma_commit(bar_empty(st));
      }
      mma_commit(bar_drain);
      mbar_drain(bar_drain, 0, a.wait_ns);
    }
    __syncwarp();
  } else {
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    // keep key j  <=>  anchor mean - pooled score <= theta  <=>  score >= xbar - theta
    const float thr = row_valid ? a.xbar[(long long)bh * a.nqb + qb] - a.theta : INFINITY;
    const int cand_hi = row_valid ? max(0, (qb + 1) * 128 - a.local) : 0;   // ls of this block
    // element offset of this row's list inside its head's list region
    const int row_elem = row_valid ? static_cast<int>(cap_prefix(qb, 128, a.cap_a)) : 0;
    int* head_lists = a.lists + (long long)bh * a.list_per_head;    // the same for the warp
    // this row's candidate-tile masks (written by the warps of the first key word)
    const int n_ct = row_valid ? tmask_tiles(qb, a.tc) : 0;
    uint4* row_tmask = a.tmask + (long long)bh * a.tmask_per_head + tmask_prefix(qb, a.tc);
    uint32_t* row_bits = a.tbits + ((long long)bh * a.nqb + qb) * 3 * a.tbit_words;
    uint32_t occ_acc = 0u, den_acc = 0u, full_acc = 0u;   // this row's tile bits, 32 tiles at a time
    const uint32_t lt = (1u << lane) - 1u;
    const uint32_t below_q = (1u << qtr) - 1u;  // words of this row before this warp's
    for (int t = 0; t < T; ++t) {
      const int bb = t % kSelBufs, xs = t & 1;
      if (!warp_wait(bar_sfull(bb), (t / kSelBufs) & 1, wc)) break;
      tc_fence_after();
      uint32_t sr[32];
      tmem_ld32(tmem + lane_off + 128u * bb + 32u * qtr, sr);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_sfree(bb));
      const int key0 = (kt0 + t) * 128 + 32 * qtr;
      // candidate keys of this row inside these 32 columns: [lo, hi)
      const int lo = max(a.sink - key0, 0);
      const int hi = min(cand_hi - key0, 32);
      uint32_t part[4] = {0u, 0u, 0u, 0u};             // four independent chains
#pragma unroll
      for (int e = 0; e < 32; ++e)
        if (__uint_as_float(sr[e]) >= thr) part[e & 3] |= 1u << e;
      const uint32_t bits = (part[0] | part[1]) | (part[2] | part[3]);
      uint32_t range = 0;
      if (hi > lo) range = (hi - lo >= 32 ? 0xffffffffu : ((1u << (hi - lo)) - 1u)) << lo;
      uint32_t w = bits & range;
      // selection group: OR over the group's rows (neighbouring lanes), each
      // row cut to its own candidates before and after
      for (int o = 1; o < a.step; o <<= 1) w |= __shfl_xor_sync(0xffffffffu, w, o);
      if (a.step > 1) w &= range;
      reinterpret_cast<uint32_t*>(x_words + xs * 128 + r)[qtr] = w;
      __syncwarp();                                   // the warp's words, then its one arrival
      if (lane == 0) mbar_arrive(bar_x(xs));
      if (!warp_wait(bar_x(xs), (t >> 1) & 1, wc)) break;
      const uint4 mine = x_words[xs * 128 + r];            // this row's four words
      const uint32_t* mw = &mine.x;
      int before = 0, total = 0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int c = __popc(mw[q]);
        before += ((below_q >> q) & 1u) ? c : 0;
        total += c;
      }
      if (qtr == 0 && t < n_ct) {
        row_tmask[t] = mine;
        const uint32_t bit = 1u << (t & 31);
        if (total > 0) occ_acc |= bit;
        if (total >= tile_dense_min(1)) den_acc |= bit;
        if (total == 128) full_acc |= bit;
        if ((t & 31) == 31 || t == n_ct - 1) {
          row_bits[t >> 5] = occ_acc;
          row_bits[a.tbit_words + (t >> 5)] = den_acc;
          row_bits[2 * a.tbit_words + (t >> 5)] = full_acc;
          occ_acc = den_acc = full_acc = 0u;
        }
      }
      // append.  When every row of the warp keeps all 32 keys of its word (the
      // dense case), every row stores the same 32 values: one shuffle and one
      // coalesced store per row.
      const int key = key0 + lane;
      const int pos = row_elem + off + before;
      const bool dense = __all_sync(0xffffffffu, w == 0xffffffffu);
      if (dense) {
        int* hl = head_lists + lane;
#pragma unroll 8
        for (int j = 0; j < 32; ++j) hl[__shfl_sync(0xffffffffu, pos, j)] = key;
      }
      // Otherwise either each thread stores its own row's keys, one per step
      // (as many steps as the fullest row has keys, each store scattered over
      // the rows), when no row has more than 8 keys, or no more than 16 and
      // at most half as many as there are rows with keys; or row by row, the
      // row's word and list position shuffled to the warp and its kept keys
      // stored coalesced (as many steps as rows with keys, two in flight).
      const int most = dense ? 0 : __reduce_max_sync(0xffffffffu, __popc(w));
      const uint32_t need = __ballot_sync(0xffffffffu, w != 0u);
      if (most > 0 && (most <= 8 || (most <= 16 && 2 * most <= __popc(need)))) {
        uint32_t rem = w;
        int k = 0;
        while (__any_sync(0xffffffffu, rem != 0u)) {
          if (rem) {
            head_lists[pos + k++] = key0 + __ffs(rem) - 1;
            rem &= rem - 1u;
          }
        }
      } else if (most > 0 && need == 0xffffffffu) {
#pragma unroll 8
        for (int j = 0; j < 32; ++j) {
          const uint32_t wj = __shfl_sync(0xffffffffu, w, j);
          const int pj = __shfl_sync(0xffffffffu, pos, j);
          if ((wj >> lane) & 1u) head_lists[pj + __popc(wj & lt)] = key;
        }
      } else if (most > 0) {
        for (uint32_t rest = need; rest;) {
          const int j0 = __ffs(rest) - 1;
          rest &= rest - 1u;
          const int j1 = rest ? __ffs(rest) - 1 : -1;
          rest &= rest - 1u;
          const uint32_t w0 = __shfl_sync(0xffffffffu, w, j0);
          const int p0 = __shfl_sync(0xffffffffu, pos, j0);
          const uint32_t w1 = __shfl_sync(0xffffffffu, w, j1 & 31);
          const int p1 = __shfl_sync(0xffffffffu, pos, j1 & 31);
          if ((w0 >> lane) & 1u) head_lists[p0 + __popc(w0 & lt)] = key;
          if (j1 >= 0 && ((w1 >> lane) & 1u)) head_lists[p1 + __popc(w1 & lt)] = key;
        }
      }
      off += total;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // written even after an abort: a count never exceeds its block's capacity
  if (warp >= 2 && qtr == 0 && row_valid) a.counts[(long long)bh * a.nqb + qb] = off;
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------------------
// bitmask -> ascending index list
// ---------------------------------------------------------------------------
constexpr int kCompactThreads = 256;

struct CompactArgs {
  int nrows_total;          // B*Hq*nqb
  int nqb;
  int L;
  int sink, local;
  int unit;                 // 1: bits are keys; bk: bits are key blocks
  int step;                 // query blocks per selection group (>= 1)
  const uint32_t* mask;     // [rows][nwords]
  int nwords;
  int* lists;
  long long list_per_head;  // list elements per (b, h)
  long long cap_a;          // local + sink
  int* counts;
};

__global__ void __launch_bounds__(kCompactThreads)
compact_kernel(const CompactArgs a) {
  const int row = blockIdx.x;
  const int bh = row / a.nqb, qb = row - (row / a.nqb) * a.nqb;
  const int ls = max(0, (qb + 1) * 128 - a.local);
  const int bit_lo = a.sink / a.unit;
  const int bit_hi = max(a.sink, ls) / a.unit;
  const int w_lo = bit_lo / 32;
  const int w_hi = bit_hi > bit_lo ? (bit_hi + 31) / 32 : w_lo;
  const int n = w_hi - w_lo;
  int* out = a.lists + (long long)bh * a.list_per_head + cap_prefix(qb, 128, a.cap_a) / a.unit;
  // Selection groups (step > 1): a word is the OR of the group's rows, each
  // read only inside its own candidate range (the rest of a row is never
  // written) -- the result is then cut to this block's range by [w_lo, w_hi).
  const int g0 = (qb / a.step) * a.step;
  const int g1 = min(g0 + a.step, a.nqb);
  const uint32_t* mrow0 = a.mask + ((long long)row - qb) * a.nwords;   // block 0 of this head
  auto word_at = [&](int w) -> uint32_t {
    if (a.step == 1) return mrow0[(long long)qb * a.nwords + w];
    uint32_t v = 0;
    for (int b2 = g0; b2 < g1; ++b2) {
      const int ls2 = max(0, (b2 + 1) * 128 - a.local);
      const int hi2 = max(a.sink, ls2) / a.unit;
      if (w < (hi2 + 31) / 32) v |= mrow0[(long long)b2 * a.nwords + w];
    }
    return v;
  };

  __shared__ int warp_cnt[kCompactThreads / 32];
  __shared__ int warp_base[kCompactThreads / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nw = kCompactThreads / 32;
  const int seg = (((n + nw - 1) / nw) + 31) & ~31;      // words per warp, multiple of 32
  const int s_lo = w_lo + warp * seg;
  const int s_hi = min(s_lo + seg, w_hi);
  int cnt = 0;
  for (int w = s_lo + lane; w < s_hi; w += 32) cnt += __popc(word_at(w));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if (lane == 0) warp_cnt[warp] = cnt;
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int i = 0; i < nw; ++i) {
      warp_base[i] = run;
      run += warp_cnt[i];
    }
    a.counts[row] = run;
  }
  __syncthreads();
  int base = warp_base[warp];
  const uint32_t lt = (1u << lane) - 1u;
  for (int w0 = s_lo; w0 < s_hi; w0 += 32) {
    const uint32_t word = (w0 + lane < s_hi) ? word_at(w0 + lane) : 0u;
    const int pc = __popc(word);
    int incl = pc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const int excl = incl - pc;
    for (int j = 0; j < 32; ++j) {
      const uint32_t wj = __shfl_sync(0xffffffffu, word, j);
      if (wj == 0u) continue;                         // warp-uniform
      const int oj = __shfl_sync(0xffffffffu, excl, j);
      if ((wj >> lane) & 1u) out[base + oj + __popc(wj & lt)] = 32 * (w0 + j) + lane;
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
}

// ---------------------------------------------------------------------------
// bitmask -> candidate-tile masks
// ---------------------------------------------------------------------------
// The bitmask paths (SALE, and ANCHOR when step is not a power of two <= 32)
// write the tile masks the paired attention kernel reads: for query block qb
// and candidate tile kt (kt0 <= kt < ls / 128), bit k of word w is set when
// key 128 kt + 32 w + k lies in [sink, ls) and its unit (the key, or its key
// block in SALE mode) is kept by some block of the selection group, exactly
// the keys compact_kernel lists; and the block's three tile bitmaps.  One
// CTA per block row, one thread per tile.
struct TileMaskArgs {
  int nqb, sink, local, unit, step, tc;
  const uint32_t* mask;     // [B*Hq*nqb][nwords] over units
  int nwords;
  uint4* tmask;             // [B*Hq][tmask_per_head]
  long long tmask_per_head;
  uint32_t* tbits;          // [B*Hq*nqb][3][tbit_words]
  int tbit_words;
};

__global__ void __launch_bounds__(128) tile_mask_kernel(const TileMaskArgs a) {
  const int row = blockIdx.x;
  const int bh = row / a.nqb, qb = row - bh * a.nqb;
  const int ls = max(0, (qb + 1) * 128 - a.local);
  const int n_ct = tmask_tiles(qb, a.tc);
  const int kt0 = a.sink / 128;
  const int g0 = (qb / a.step) * a.step;
  const int g1 = min(g0 + a.step, a.nqb);
  const int lane = threadIdx.x & 31;
  const uint32_t* mrow0 = a.mask + ((long long)row - qb) * a.nwords;   // block 0 of this head
  // bit u of the group's selection (each row read only inside its own range)
  auto unit_kept = [&](int u) -> uint32_t {
    uint32_t v = 0;
    for (int b2 = g0; b2 < g1; ++b2) {
      const int ls2 = max(0, (b2 + 1) * 128 - a.local);
      const int hi2 = max(a.sink, ls2) / a.unit;
      if (u >= a.sink / a.unit && u < hi2) v |= mrow0[(long long)b2 * a.nwords + u / 32] >> (u % 32);
    }
    return v & 1u;
  };
  uint4* out = a.tmask + (long long)bh * a.tmask_per_head + tmask_prefix(qb, a.tc);
  uint32_t* bits = a.tbits + (long long)row * 3 * a.tbit_words;
  // one tile per thread; a warp covers 32 consecutive tiles (one bitmap word)
  for (int t0 = threadIdx.x & ~31; t0 < n_ct; t0 += blockDim.x) {
    const int t = t0 + lane;
    uint32_t w4[4] = {0u, 0u, 0u, 0u};
    if (t < n_ct) {
      for (int wi = 0; wi < 4; ++wi) {
        const int key0 = 128 * (kt0 + t) + 32 * wi;
        uint32_t word = 0;
        if (a.unit == 1) {
          // the 32 keys are one bitmask word; a row's words inside its range
          // are written whole (compact_kernel reads them the same way)
          for (int b2 = g0; b2 < g1; ++b2) {
            const int ls2 = max(0, (b2 + 1) * 128 - a.local);
            if (key0 / 32 < (max(a.sink, ls2) + 31) / 32)
              word |= mrow0[(long long)b2 * a.nwords + key0 / 32];
          }
        } else {
          for (int k = 0; k < 32; k += min(a.unit, 32)) {
            const uint32_t run = a.unit >= 32 ? 0xffffffffu : ((1u << a.unit) - 1u);
            if (unit_kept((key0 + k) / a.unit)) word |= run << k;
          }
        }
        // the block's candidates [sink, ls)
        const int lo = max(a.sink - key0, 0), hi = min(ls - key0, 32);
        uint32_t range = 0;
        if (hi > lo) range = (hi - lo >= 32 ? 0xffffffffu : ((1u << (hi - lo)) - 1u)) << lo;
        w4[wi] = word & range;
      }
      out[t] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
    }
    const int c = __popc(w4[0]) + __popc(w4[1]) + __popc(w4[2]) + __popc(w4[3]);
    const uint32_t occ = __ballot_sync(0xffffffffu, c > 0);
    const uint32_t den = __ballot_sync(0xffffffffu, c >= tile_dense_min(a.unit));
    const uint32_t full = __ballot_sync(0xffffffffu, c == 128);
    if (lane == 0) {
      bits[t0 >> 5] = occ;
      bits[a.tbit_words + (t0 >> 5)] = den;
      bits[2 * a.tbit_words + (t0 >> 5)] = full;
    }
  }
}

// ---------------------------------------------------------------------------
// stats: totals over all query blocks into the workspace header
// ---------------------------------------------------------------------------
struct StatsArgs {
  int nrows_total, nqb, L, sink, local, mode, unit;
  const int* counts;
  unsigned long long* acc;   // [5]: blocks, candidates, kept, kept_pairs, dense_pairs
};

__global__ void stats_kernel(const StatsArgs a) {
  const int row = blockIdx.x * blockDim.x + threadIdx.x;
  unsigned long long v[5] = {0, 0, 0, 0, 0};
  if (row < a.nrows_total) {
    const int qb = row % a.nqb;
    const long long row0 = (long long)qb * 128;
    const long long le = min(row0 + 128, (long long)a.L);
    const long long n = le - row0;
    const long long ls = max(0LL, row0 + 128 - a.local);
    const long long sink_end = min((long long)a.sink, ls);
    const long long cand = max(0LL, ls - a.sink);
    const long long kept = (a.mode == kModeDense) ? 0 : (long long)a.counts[row] * a.unit;
    // sum_{i=row0}^{le-1} (i + 1 - ls) and sum (i + 1)
    const long long sum_i1 = (le * (le + 1) - row0 * (row0 + 1)) / 2;
    v[0] = 1;
    v[1] = (a.mode == kModeDense) ? 0 : cand;
    v[2] = kept;
    v[3] = (a.mode == kModeDense) ? sum_i1 : n * (sink_end + kept) + sum_i1 - n * ls;
    v[4] = sum_i1;
  }
#pragma unroll
  for (int k = 0; k < 5; ++k) {
    unsigned long long x = v[k];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    if ((threadIdx.x & 31) == 0 && x) atomicAdd(a.acc + k, x);
  }
}

}  // namespace spa
