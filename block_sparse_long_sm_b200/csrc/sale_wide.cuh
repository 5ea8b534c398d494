// sale_wide.cuh -- the SALE block scan of sale.cuh with sixteen epilogue
// warps (selected with SPA_DEBUG_SALE_WIDE).
//
// sale_scan_kernel's eight epilogue warps each read two heads' 64-column dot
// tiles from TMEM one after the other (load, wait, reduce, load, wait,
// reduce); its profile is latency-bound, with the int8 tensor pipe 24 % busy
// at ten warps per SM.  Here each of sixteen epilogue warps owns one head's
// TMEM lane quadrant, so a tile costs every warp one load latency, twice as
// many warps hide it, and the accumulator buffer is released with one
// barrier arrival per warp instead of one per thread.  The MMA and TMA roles
// and the result are sale_scan_kernel's.
#pragma once

#include "sale.cuh"

namespace spa {

constexpr int kSaleWideThreads = 576;        // warp 0 TMA, warp 1 MMA, warps 2-17 epilogue

__global__ void __launch_bounds__(kSaleWideThreads, 1)
sale_scan_wide_kernel(const __grid_constant__ CUtensorMap tm_q8,
                 const __grid_constant__ CUtensorMap tm_k8, const SaleArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t s_base = smem_u32(smem);
  const uint32_t s_q = s_base;                                   // [head][128 x 128 int8]
  auto s_k = [&](int st) { return s_base + kSaleHeads * kQ8Bytes + st * kK8Bytes; };
  uint8_t* bar_area = smem + kSaleHeads * kQ8Bytes + kSaleStages * kK8Bytes;
  const uint32_t b0 = smem_u32(bar_area);
  const uint32_t bar_q = b0;
  auto bar_full = [&](int st) { return b0 + 8u * (1 + st); };
  auto bar_empty = [&](int st) { return b0 + 8u * (1 + kSaleStages + st); };
  auto bar_afull = [&](int bb) { return b0 + 8u * (1 + 2 * kSaleStages + bb); };
  auto bar_afree = [&](int bb) { return b0 + 8u * (3 + 2 * kSaleStages + bb); };
  const uint32_t bar_drain = b0 + 8u * (5 + 2 * kSaleStages);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bar_area + 512);
  volatile uint32_t* abort_flag = tmem_holder + 1;
  uint32_t* gflags = reinterpret_cast<uint32_t*>(bar_area + 1024);       // [head][words]
  float* kscale = reinterpret_cast<float*>(gflags + kSaleHeads * kMaxGroupWords);  // sk*scale

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int x = blockIdx.x;
  const int chunk = x % a.chunks;
  x /= a.chunks;
  const int qb = x % a.nqb;
  const int bkv = x / a.nqb;                      // b * Hkv + kv head
  const int b = bkv / a.Hkv, kvh = bkv - b * a.Hkv;
  const int h0 = kvh * a.group + chunk * kSaleHeads;
  const int nh = min(kSaleHeads, a.group - chunk * kSaleHeads);
  const int row0 = qb * 128;
  const int le = min(row0 + 128, a.L);
  const int ls = max(0, row0 + 128 - a.local);
  const int sink_end = min(a.sink, ls);
  const int n_sink_t = (sink_end + kSaleKeys - 1) / kSaleKeys;
  const int n_loc_t = (le - ls + kSaleKeys - 1) / kSaleKeys;
  const int cand_lo = a.sink, cand_hi = max(a.sink, ls);
  const int n_cand_t = (cand_hi - cand_lo + kSaleKeys - 1) / kSaleKeys;
  const int n_stat_t = n_sink_t + n_loc_t;
  const int T = n_stat_t + n_cand_t;
  auto tile_key0 = [&](int t) {
    if (t < n_sink_t) return t * kSaleKeys;
    if (t < n_stat_t) return ls + (t - n_sink_t) * kSaleKeys;
    return cand_lo + (t - n_stat_t) * kSaleKeys;
  };

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int st = 0; st < kSaleStages; ++st) {
      mbar_init(bar_full(st), 1);
      mbar_init(bar_empty(st), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_afull(i), 1);
      mbar_init(bar_afree(i), 16);              // one arrival per epilogue warp
    }
    mbar_init(bar_drain, 1);
    *abort_flag = 0u;
    fence_barrier_init();
  }
  for (int i = threadIdx.x; i < kSaleHeads * kMaxGroupWords; i += blockDim.x) gflags[i] = 0u;
  {
    const int nkb_used = min(a.nkb, (le + a.bk - 1) / a.bk);
    const float* skp = a.sk + (long long)bkv * a.nkb;
    for (int i = threadIdx.x; i < nkb_used; i += blockDim.x) kscale[i] = skp[i] * a.scale;
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
    if (lane == 0) {
      mbar_arrive_expect_tx(bar_q, nh * kQ8Bytes);
      for (int j = 0; j < nh; ++j)
        tma_load_2d(s_q + j * kQ8Bytes, &tm_q8, bar_q, 0, (b * a.Hq + h0 + j) * a.L + row0);
      int issued = 0;
      for (int t = 0; t < T; ++t) {
        const int st = t % kSaleStages;
        if (t >= kSaleStages && !mbar_wait(bar_empty(st), ((t / kSaleStages) - 1) & 1, wc)) break;
        mbar_arrive_expect_tx(bar_full(st), kK8Bytes);
        tma_load_2d(s_k(st), &tm_k8, bar_full(st), 0, bkv * a.L + tile_key0(t));
        issued = t + 1;
      }
      {  // no copy may still be in flight when the CTA exits
        mbar_drain(bar_q, 0, a.wait_ns);
        for (int t = max(0, issued - kSaleStages); t < issued; ++t)
          mbar_drain(bar_full(t % kSaleStages), (t / kSaleStages) & 1, a.wait_ns);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = mbar_wait(bar_q, 0, wc);
      for (int t = 0; ok && t < T; ++t) {
        const int st = t % kSaleStages, bb = t & 1;
        if (!(ok = mbar_wait(bar_full(st), (t / kSaleStages) & 1, wc))) break;
        if (t >= 2 && !(ok = mbar_wait(bar_afree(bb), ((t >> 1) - 1) & 1, wc))) break;
        tc_fence_after();
        for (int j = 0; j < nh; ++j) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            mma_i8_ss(tmem + 64u * (bb * kSaleHeads + j),
                      smem_desc_sw128(s_q + j * kQ8Bytes + kk * 32u, 16),
                      smem_desc_sw128(s_k(st) + kk * 32u, 16), kIdescI8N64, kk > 0 ? 1u : 0u);
          }
        }
        mma_commit(bar_afull(bb));
        mma_commit(bar_empty(st));
      }
      mma_commit(bar_drain);
      mbar_drain(bar_drain, 0, a.wait_ns);
    }
    __syncwarp();
  } else {
    // warps 2-17: warp w reads TMEM lanes 32 (w % 4) .. + 31 of head (w - 2) / 4
    const int quad = warp & 3;
    const int j = (warp - 2) >> 2;
    const int r = quad * 32 + lane;
    const int row = row0 + r;
    const bool row_valid = row < a.L;
    const bool active = j < nh;                // warp-uniform
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const float cq = active ? a.sq[((long long)b * a.Hq + h0 + j) * a.nqb + qb] : 0.f;
    float m = -INFINITY, l = 0.f, thr = INFINITY;
    for (int t = 0; t < T; ++t) {
      const int bb = t & 1;
      if (!warp_wait(bar_afull(bb), (t >> 1) & 1, wc)) break;
      tc_fence_after();
      const int key0 = tile_key0(t);
      if (active) {
        const uint32_t taddr = tmem + lane_off + 64u * (bb * kSaleHeads + j);
        if (t < n_stat_t) {
          uint32_t sr[2][32];
          tmem_ld32(taddr, sr[0]);
          tmem_ld32(taddr + 32u, sr[1]);
          tmem_ld_wait();
          // S~ over the causal sink-local keys of this row
          int limit = (t < n_sink_t) ? sink_end - key0 : min(le - key0, row - key0 + 1);
          limit = max(0, min(limit, kSaleKeys));
          float tm = -INFINITY;
#pragma unroll
          for (int c = 0; c < 2; ++c) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int col = c * 32 + e;
              const float v = col < limit
                                  ? static_cast<float>(static_cast<int>(sr[c][e])) *
                                        (cq * kscale[min(key0 + col, a.L - 1) >> a.bk_log2])
                                  : -INFINITY;
              sr[c][e] = __float_as_uint(v);
              tm = fmaxf(tm, v);
            }
          }
          if (tm > -INFINITY) {
            const float mn = fmaxf(m, tm);
            float acc = 0.f;
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
              for (int e = 0; e < 32; ++e) acc += __expf(__uint_as_float(sr[c][e]) - mn);
            l = l * __expf(m - mn) + acc;
            m = mn;
          }
          if (t == n_stat_t - 1)
            thr = row_valid ? m + logf(a.tau_h[h0 + j] * l) : INFINITY;   // t_i = em + ln(tau el)
        } else {
          uint32_t pk[32];
          tmem_ld32_pack16(taddr, pk);
          tmem_ld_wait();
          uint32_t gbits = 0;                          // bit g: group g of this tile
#pragma unroll
          for (int g = 0; g < 4; ++g) {               // 16 keys = 8 packed registers
            const uint32_t* q = pk + 8 * g;
            const uint32_t m01 = max_s16x2(max_s16x2(q[0], q[1]), max_s16x2(q[2], q[3]));
            const uint32_t m23 = max_s16x2(max_s16x2(q[4], q[5]), max_s16x2(q[6], q[7]));
            const uint32_t mm = max_s16x2(m01, m23);
            const int mx = max(static_cast<int>(static_cast<int16_t>(mm & 0xffffu)),
                               static_cast<int>(mm) >> 16);
            const int key = key0 + 16 * g;
            if (key < cand_hi && static_cast<float>(mx) * (cq * kscale[key >> a.bk_log2]) >= thr)
              gbits |= 1u << g;
          }
          gbits = __reduce_or_sync(0xffffffffu, gbits);
          if (lane == 0 && gbits) {
            const int g0 = (key0 - cand_lo) / 16;    // multiple of 4: one word holds 4 bits
            atomicOr(&gflags[j * kMaxGroupWords + (g0 >> 5)], gbits << (g0 & 31));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_afree(bb));
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // key-block flags -> global bitmask rows (every word of every row is written)
  if (!*abort_flag) {
    const int gpb = a.bk / 16;                     // groups per key block
    const int kb_lo = cand_lo / a.bk;
    for (int idx = threadIdx.x; idx < nh * a.nwords; idx += blockDim.x) {
      const int j = idx / a.nwords, w = idx - j * a.nwords;
      uint32_t* mrow = a.mask + (((long long)b * a.Hq + h0 + j) * a.nqb + qb) * a.nwords;
      const uint32_t* gf = gflags + j * kMaxGroupWords;
      uint32_t word = 0;
      for (int bit = 0; bit < 32; ++bit) {
        const int kb = w * 32 + bit;
        if (kb < kb_lo || kb * a.bk >= cand_hi) continue;
        const int g0 = (kb - kb_lo) * gpb;
        bool any = false;
        for (int g = g0; g < g0 + gpb; ++g) any |= (gf[g >> 5] >> (g & 31)) & 1u;
        word |= (any ? 1u : 0u) << bit;
      }
      mrow[w] = word;
    }
  }
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace spa
