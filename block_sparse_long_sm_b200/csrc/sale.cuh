// sale.cuh -- SALE-mode key-block selection (SALE: Low-bit Estimation for
// Efficient Sparse Attention in Long-context LLM Prefilling, Sec. 3.2-3.4).
//
//   kmean_partial_kernel / kmean_final_kernel
//       per (b, kv head): mean of K over the sequence, summed in fp64 over
//       fixed chunks and rounded once to fp32 (smoothing, as SageAttention2).
//   quant_kernel
//       symmetric per-block 4-bit codes held in int8: scale = absmax / 7 and
//       code = round-half-even(x / scale) in IEEE fp32, clamped to [-7, 7];
//       K is smoothed first; an all-zero block gets scale 1.
//   sale_scan_kernel
//       per query block on the int8 tensor cores (tcgen05 kind::i8, M = 128,
//       N = 128): first the sink-local tiles give em_i, el_i and the row
//       threshold t_i = em_i + ln(tau * el_i) (Eq. (4) as corrected); then
//       every candidate tile: a key block is kept when some valid row's
//       largest estimated score in it reaches t_i.  The integer dot products
//       are compared through max(dot) * (s_q * s_k * scale) >= t_i, exact in
//       the integer part.  Output: one bit per key block.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace spa {

struct KmeanArgs {
  const __nv_bfloat16* k;   // [B*Hkv][L][128]
  int L;
  double* partial;          // [B*Hkv][chunks][128]
  float* mean;              // [B*Hkv][128]
};

__global__ void kmean_partial_kernel(const KmeanArgs a) {
  const int bkv = blockIdx.y, chunk = blockIdx.x, d = threadIdx.x;
  const int per = (a.L + kKmeanChunks - 1) / kKmeanChunks;
  const int r0 = chunk * per, r1 = min(r0 + per, a.L);
  const __nv_bfloat16* kp = a.k + (long long)bkv * a.L * 128 + d;
  double s = 0.0;
  for (int r = r0; r < r1; ++r) s += static_cast<double>(__bfloat162float(kp[(long long)r * 128]));
  a.partial[((long long)bkv * kKmeanChunks + chunk) * 128 + d] = s;
}

__global__ void kmean_final_kernel(const KmeanArgs a) {
  const int bkv = blockIdx.x, d = threadIdx.x;
  double s = 0.0;
  for (int c = 0; c < kKmeanChunks; ++c) s += a.partial[((long long)bkv * kKmeanChunks + c) * 128 + d];
  a.mean[(long long)bkv * 128 + d] = static_cast<float>(s / static_cast<double>(a.L));
}

struct QuantArgs {
  const __nv_bfloat16* x;   // [heads][L][128]
  const float* mean;        // [heads][128] or null (no smoothing)
  int L, rows;              // rows per quantisation block
  int nblk;                 // blocks per head
  int8_t* codes;            // [heads][L][128]
  float* scales;            // [heads][nblk]
};

// grid (nblk, heads), 128 threads: thread d owns column d of the block.
__global__ void __launch_bounds__(128) quant_kernel(const QuantArgs a) {
  const int head = blockIdx.y, blk = blockIdx.x, d = threadIdx.x;
  const int r0 = blk * a.rows, r1 = min(r0 + a.rows, a.L);
  const __nv_bfloat16* xp = a.x + (long long)head * a.L * 128 + d;
  const float mu = a.mean ? a.mean[(long long)head * 128 + d] : 0.f;
  float amax = 0.f;
  for (int r = r0; r < r1; ++r) {
    const float v = __fsub_rn(__bfloat162float(xp[(long long)r * 128]), mu);
    amax = fmaxf(amax, fabsf(v));
  }
  __shared__ float red[4];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((d & 31) == 0) red[d >> 5] = amax;
  __syncthreads();
  amax = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  const float sc = amax > 0.f ? __fdiv_rn(amax, 7.0f) : 1.0f;
  int8_t* cp = a.codes + (long long)head * a.L * 128 + d;
  for (int r = r0; r < r1; ++r) {
    const float v = __fsub_rn(__bfloat162float(xp[(long long)r * 128]), mu);
    float c = rintf(__fdiv_rn(v, sc));
    c = fminf(fmaxf(c, -7.f), 7.f);
    cp[(long long)r * 128] = static_cast<int8_t>(c);
  }
  if (d == 0) a.scales[(long long)head * a.nblk + blk] = sc;
}

// ---------------------------------------------------------------------------
// fused sink-local statistics + block scan
// ---------------------------------------------------------------------------
// One CTA = (b, kv head, query block, up to two q heads of that kv head's
// group): the q heads share every int8 K tile, so each 128-key tile fetched
// from L2 feeds two MMAs (M = 128 rows, N = 128 keys, K = 128 in four K = 32
// steps; few, large MMAs, since the issue of an int8 MMA of N = 64 costs
// about what it computes).  TMEM: two accumulator sets x two heads x 128
// columns.  The epilogue (warps 2-9) gives each thread one row of one head,
// all 128 columns of every tile, so the sink-local statistics need no
// cross-thread merge.  Candidate tiles are read from TMEM as packed 16-bit
// pairs (the dots fit: |dot| <= 7*7*128) and reduced with max.s16x2; the
// accumulator set is released as soon as it is in registers.
constexpr int kSaleThreads = 320;            // warp 0 TMA, warp 1 MMA, warps 2-9 epilogue
constexpr int kSaleStages = 6;
constexpr int kSaleKeys = 128;               // keys per K tile
constexpr int kSaleHeads = 2;                // q heads per CTA
constexpr int kSaleBufs = 2;                 // accumulator sets in TMEM
static_assert(kSaleBufs * kSaleHeads * kSaleKeys <= 512, "more TMEM columns than a CTA has");
constexpr uint32_t kQ8Bytes = 128u * 128u;   // 128 rows x 128 int8
constexpr uint32_t kK8Bytes = kSaleKeys * 128u;
constexpr int kMaxGroupWords = 512;          // candidate 16-key groups / 32 (L <= 262144)
constexpr int kMaxScales = 16384;            // key blocks per head (L / bk <= 16384)
constexpr uint32_t kSaleSmemBytes = 1024u + kSaleHeads * kQ8Bytes + kSaleStages * kK8Bytes +
                                    1024u + kSaleHeads * kMaxGroupWords * 4u + kMaxScales * 4u;
static_assert(kSaleSmemBytes <= 232448u, "more shared memory than a CTA may use");
constexpr uint32_t kIdescI8N128 = make_idesc(2, 1, 128, 128, 0, 0);

struct SaleArgs {
  int B, Hq, Hkv, L, nqb, group;
  int sink, local, bk, nkb;
  int bk_log2;              // bk is a power of two
  int chunks;               // ceil(group / kSaleHeads)
  float scale, tau;
  const float* sq;          // [B*Hq][nqb]
  const float* sk;          // [B*Hkv][nkb]
  uint32_t* mask;           // [B*Hq*nqb][nwords] over key blocks
  int nwords;
  uint32_t* err;
  uint64_t wait_ns;
  float tau_h[128];         // threshold of each q head (index h), SPA_MAX_TAU_HEADS
};

__global__ void __launch_bounds__(kSaleThreads, 1)
sale_scan_kernel(const __grid_constant__ CUtensorMap tm_q8,
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
  auto bar_afree = [&](int bb) { return b0 + 8u * (1 + 2 * kSaleStages + kSaleBufs + bb); };
  const uint32_t bar_drain = b0 + 8u * (1 + 2 * kSaleStages + 2 * kSaleBufs);
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
    for (int i = 0; i < kSaleBufs; ++i) {
      mbar_init(bar_afull(i), 1);
      mbar_init(bar_afree(i), 8);                  // the eight epilogue warps
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
        const int st = t % kSaleStages, bb = t % kSaleBufs;
        if (!(ok = mbar_wait(bar_full(st), (t / kSaleStages) & 1, wc))) break;
        if (t >= kSaleBufs && !(ok = mbar_wait(bar_afree(bb), ((t / kSaleBufs) - 1) & 1, wc))) break;
        tc_fence_after();
        for (int j = 0; j < nh; ++j) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            mma_i8_ss(tmem + static_cast<uint32_t>(kSaleKeys) * (bb * kSaleHeads + j),
                      smem_desc_sw128(s_q + j * kQ8Bytes + kk * 32u, 16),
                      smem_desc_sw128(s_k(st) + kk * 32u, 16), kIdescI8N128, kk > 0 ? 1u : 0u);
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
    const int quad = warp & 3;               // TMEM lane quadrant
    const int hsel = (warp - 2) >> 2;        // head h0 + hsel
    const bool head_valid = hsel < nh;       // warp-uniform
    const int r = quad * 32 + lane;
    const int row = row0 + r;
    const bool row_valid = row < a.L;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const float cq = head_valid ? a.sq[((long long)b * a.Hq + h0 + hsel) * a.nqb + qb] : 0.f;
    float m = -INFINITY, l = 0.f, thr = INFINITY;
    for (int t = 0; t < T; ++t) {
      const int bb = t % kSaleBufs;
      if (!warp_wait(bar_afull(bb), (t / kSaleBufs) & 1, wc)) break;
      tc_fence_after();
      const int key0 = tile_key0(t);
      const uint32_t taddr = tmem + lane_off + static_cast<uint32_t>(kSaleKeys) * (bb * kSaleHeads + hsel);
      bool released = false;
      if (head_valid && t < n_stat_t) {
        // S~ over the causal sink-local keys of this row, 64 columns at a time
        int limit = (t < n_sink_t) ? sink_end - key0 : min(le - key0, row - key0 + 1);
        limit = max(0, min(limit, kSaleKeys));
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          uint32_t sr[2][32];
          tmem_ld32(taddr + 64u * half, sr[0]);
          tmem_ld32(taddr + 64u * half + 32u, sr[1]);
          tmem_ld_wait();
          float tm = -INFINITY;
#pragma unroll
          for (int c = 0; c < 2; ++c) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int col = 64 * half + c * 32 + e;
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
        }
        if (t == n_stat_t - 1)
          thr = row_valid ? m + logf(a.tau_h[h0 + hsel] * l) : INFINITY;   // t_i = em + ln(tau el)
      } else if (head_valid) {
        // the 128 columns as packed 16-bit pairs, one wait for the two loads;
        // the eight 16-key groups' K scales are read meanwhile
        uint32_t pk[2][32];
        tmem_ld32_pack16(taddr, pk[0]);
        tmem_ld32_pack16(taddr + 64u, pk[1]);
        float ksg[8];
#pragma unroll
        for (int g = 0; g < 8; ++g) ksg[g] = kscale[min(key0 + 16 * g, cand_hi - 1) >> a.bk_log2];
        tmem_ld_wait();
        // the dots are in registers: the set is free for tile t + kSaleBufs
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_afree(bb));
        released = true;
        uint32_t gbits = 0;                            // bit g: 16-key group g of the tile
#pragma unroll
        for (int g = 0; g < 8; ++g) {                  // 16 keys = 8 packed registers
          const uint32_t* q = pk[g >> 2] + 8 * (g & 3);
          const uint32_t m01 = max_s16x2(max_s16x2(q[0], q[1]), max_s16x2(q[2], q[3]));
          const uint32_t m23 = max_s16x2(max_s16x2(q[4], q[5]), max_s16x2(q[6], q[7]));
          const uint32_t mm = max_s16x2(m01, m23);
          const int mx = max(static_cast<int>(static_cast<int16_t>(mm & 0xffffu)),
                             static_cast<int>(mm) >> 16);
          if (key0 + 16 * g < cand_hi && static_cast<float>(mx) * (cq * ksg[g]) >= thr)
            gbits |= 1u << g;
        }
        // one warp reduction and at most one shared atomic per tile
        gbits = __reduce_or_sync(0xffffffffu, gbits);
        if (lane == 0 && gbits) {
          const int g0 = (key0 - cand_lo) / 16;        // multiple of 8: one word holds the 8 bits
          atomicOr(&gflags[hsel * kMaxGroupWords + (g0 >> 5)], gbits << (g0 & 31));
        }
      }
      if (!released) {
        // the set is free once every epilogue warp has read it: one arrival per warp
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_afree(bb));
      }
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
