// attn.cuh -- sparse causal attention forward over the kept keys of every
// query block, on the 5th-generation tensor cores.
//
// Follows AnchorAttention (Sec. 3.4, "fine-grained sparse computation": load
// the kept key/value rows by their discrete coordinates instead of contiguous
// blocks) and SALE's Computation Pass (attention over the kept key blocks),
// with the online-softmax recurrence of FlashAttention.
//
// One CTA computes one 128-row query block of one q head.  Its key sequence
// is a list of 128-key tiles:
//   sink tiles      keys [0, sink_end), contiguous TMA loads;
//   selected tiles  the plan's kept keys, gathered row by row (TMA gather4)
//                   -- or with two tiled loads when the 128 indices happen to
//                   be consecutive -- the last one padded and masked;
//   local tiles     keys [ls, min(row0 + 128, L)), contiguous; the last one is
//                   the diagonal tile and is causally masked.
// In dense mode the local range simply starts at key 0.
//
// Roles (192 threads):
//   warp 0     TMA producer: Q once, then K and V of each tile into a
//              3-stage ring of shared-memory buffers;
//   warp 1     TMEM allocation, then one thread issues tcgen05.mma:
//              S_t = Q K_t^T into one of two TMEM S buffers, and
//              O += P_{t-1} V_{t-1} with P read straight from TMEM;
//   warps 2-5  softmax: thread = query row (TMEM lane).  Reads S_t, masks,
//              updates the running max (rescaling O in TMEM only when the max
//              grows by more than 2^8), writes P_t (bf16) to TMEM, and at the
//              end normalises O and stores O and the LSE.
//
// TMEM columns: S0 [0,128)  S1 [128,256)  O [256,384)  P0 [384,448)  P1 [448,512).
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace spa {

constexpr int kAttnStages = 3;
constexpr int kAttnThreads = 192;
constexpr uint32_t kAttnSmemBytes =
    1024u + kTileBytes + kAttnStages * 2u * kTileBytes + 256u;
static_assert(kAttnSmemBytes <= 232448u, "more shared memory than a CTA may use");

struct AttnArgs {
  int B, Hq, Hkv, L, nqb, group;
  int sink, local;
  int mode, bk;
  float sl2;                  // softmax scale * log2(e)
  const int* counts;          // kept candidates per block (keys, or key blocks in SALE mode)
  const int* lists;           // index lists at closed-form offsets
  long long list_per_head;    // list elements per (b, h)
  long long cap_a;            // local + sink (capacity prefix constant), in keys
  int list_unit;              // 1 (keys) or bk (SALE: list holds key-block ids)
  const uint4* tmask;         // paired kernel: candidate-tile masks [B*Hq][tmask_per_head]
  long long tmask_per_head;
  int tc;                     // tmask_c(sink, local)
  const uint32_t* tbits;      // paired kernel: tile bitmaps [B*Hq*nqb][3][tbit_words]
  int tbit_words;
  const __nv_bfloat16* k;     // paired kernel: K and V rows for the gathered tiles
  const __nv_bfloat16* v;
  __nv_bfloat16* o;
  float* lse;
  uint32_t* err;
  uint64_t wait_ns;
  uint32_t debug;
};

struct AttnItem {
  int b, h, kvh, qb, row0, le, ls, sink_end;
  int n_sink_t, n_sel_t, n_loc_t, n_sel;  // n_sel in keys
  int loc_start;
  long long list_off;                     // element offset of this block's list
};

__device__ __forceinline__ AttnItem attn_item(const AttnArgs& a, int x) {
  AttnItem it;
  const int per_kv = a.nqb * a.group;
  const int bkv = x / per_kv;
  const int rem = x - bkv * per_kv;
  it.qb = a.nqb - 1 - rem / a.group;
  const int hh = rem % a.group;
  it.b = bkv / a.Hkv;
  it.kvh = bkv - it.b * a.Hkv;
  it.h = it.kvh * a.group + hh;
  it.row0 = it.qb * 128;
  it.le = min(it.row0 + 128, a.L);
  it.ls = max(0, it.row0 + 128 - a.local);
  it.sink_end = min(a.sink, it.ls);
  if (a.mode == kModeDense) {
    it.n_sink_t = 0;
    it.n_sel = 0;
    it.loc_start = 0;
    it.list_off = 0;
  } else {
    it.n_sink_t = (it.sink_end + 127) / 128;
    const int bh = it.b * a.Hq + it.h;
    const int cnt = a.counts[(long long)bh * a.nqb + it.qb];
    it.n_sel = cnt * a.list_unit;
    it.loc_start = it.ls;
    it.list_off = (long long)bh * a.list_per_head +
                  cap_prefix(it.qb, 128, a.cap_a) / a.list_unit;
  }
  it.n_sel_t = (it.n_sel + 127) / 128;
  it.n_loc_t = (it.le - it.loc_start + 127) / 128;
  return it;
}

struct TileDesc {
  int gather;   // 1 -> selected (gathered) tile
  int key0;     // first key of a contiguous tile / first selected ordinal of a gathered tile
  int valid;    // valid columns
  int causal;   // diagonal tile
};

__device__ __forceinline__ TileDesc tile_desc(const AttnItem& it, int t) {
  TileDesc d;
  if (t < it.n_sink_t) {
    d.gather = 0;
    d.key0 = t * 128;
    d.valid = min(128, it.sink_end - d.key0);
    d.causal = 0;
  } else if (t < it.n_sink_t + it.n_sel_t) {
    d.gather = 1;
    d.key0 = (t - it.n_sink_t) * 128;
    d.valid = min(128, it.n_sel - d.key0);
    d.causal = 0;
  } else {
    d.gather = 0;
    d.key0 = it.loc_start + (t - it.n_sink_t - it.n_sel_t) * 128;
    d.valid = min(128, it.le - d.key0);
    d.causal = (d.key0 == it.row0);
  }
  return d;
}

// Key index of selected ordinal `n` of the block's list.
__device__ __forceinline__ int sel_key(const AttnArgs& a, const AttnItem& it, int n) {
  if (a.list_unit == 1) return a.lists[it.list_off + n];
  const int blk = a.lists[it.list_off + n / a.list_unit];
  return blk * a.list_unit + n % a.list_unit;
}

__global__ void __launch_bounds__(kAttnThreads, 1)
sparse_attn_kernel(const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_kg,
                   const __grid_constant__ CUtensorMap tm_v,
                   const __grid_constant__ CUtensorMap tm_vg, const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t s_base = smem_u32(smem);
  const uint32_t s_q = s_base;
  auto s_k = [&](int st) { return s_base + kTileBytes + st * 2u * kTileBytes; };
  auto s_v = [&](int st) { return s_base + kTileBytes + st * 2u * kTileBytes + kTileBytes; };
  uint8_t* bar_area = smem + kTileBytes + kAttnStages * 2 * kTileBytes;
  const uint32_t b0 = smem_u32(bar_area);
  // barrier addresses (8 bytes each)
  const uint32_t bar_q = b0;
  auto bar_kfull = [&](int s) { return b0 + 8u * (1 + s); };
  auto bar_vfull = [&](int s) { return b0 + 8u * (1 + kAttnStages + s); };
  auto bar_empty = [&](int s) { return b0 + 8u * (1 + 2 * kAttnStages + s); };
  const uint32_t bar_sfull0 = b0 + 8u * (1 + 3 * kAttnStages);
  const uint32_t bar_sfree0 = bar_sfull0 + 16u;
  const uint32_t bar_pfull0 = bar_sfull0 + 32u;
  const uint32_t bar_pvdone0 = bar_sfull0 + 48u;
  const uint32_t bar_drain = bar_sfull0 + 64u;
  const uint32_t bar_stall = bar_sfull0 + 72u;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bar_area + 8 * (1 + 3 * kAttnStages) + 80);
  volatile uint32_t* abort_flag = tmem_holder + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < kAttnStages; ++s) {
      mbar_init(bar_kfull(s), 1);
      mbar_init(bar_vfull(s), 1);
      mbar_init(bar_empty(s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_sfull0 + 8u * i, 1);
      mbar_init(bar_sfree0 + 8u * i, 128);
      mbar_init(bar_pfull0 + 8u * i, 128);
      mbar_init(bar_pvdone0 + 8u * i, 1);
    }
    mbar_init(bar_drain, 1);
    mbar_init(bar_stall, 1);
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
    prefetch_tensormap(&tm_v);
    prefetch_tensormap(&tm_vg);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitCtx wc{abort_flag, a.err, a.wait_ns};

  const AttnItem it = attn_item(a, blockIdx.x);
  const int T = it.n_sink_t + it.n_sel_t + it.n_loc_t;
  const int kv_row0 = (it.b * a.Hkv + it.kvh) * a.L;

  if (warp == 0) {
    // ------------------------------------------------------------- producer
    int issued = 0;  // tiles whose loads were issued
    if (lane == 0) {
      mbar_arrive_expect_tx(bar_q, kTileBytes);
      const int qrow = (it.b * a.Hq + it.h) * a.L + it.row0;
      tma_load_2d(s_q, &tm_q, bar_q, 0, qrow);
      tma_load_2d(s_q + kHalfBytes, &tm_q, bar_q, 64, qrow);
    }
    // Indices of a gathered tile: this lane's four rows (padding rows repeat
    // the tile's first key).  They are fetched one tile ahead so that the
    // global-load latency overlaps the wait for a free stage.
    auto fetch = [&](int t, int (&j)[4], int& first) {
      const TileDesc td = tile_desc(it, t);
      if (!td.gather) return;
      first = sel_key(a, it, td.key0);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int row = lane * 4 + r;
        j[r] = row < td.valid ? sel_key(a, it, td.key0 + row) : first;
      }
    };
    int nj[4] = {0, 0, 0, 0}, nfirst = 0;
    if (T > 0) fetch(0, nj, nfirst);
    for (int t = 0; t < T; ++t) {
      int j[4] = {nj[0], nj[1], nj[2], nj[3]};
      const int first = nfirst;
      if (t + 1 < T) fetch(t + 1, nj, nfirst);
      const int st = t % kAttnStages;
      if (t >= kAttnStages) {
        if (!warp_wait(bar_empty(st), ((t / kAttnStages) - 1) & 1, wc)) break;
      }
      const TileDesc td = tile_desc(it, t);
      const uint32_t kf = bar_kfull(st), vf = bar_vfull(st);
      if (!td.gather) {
        if (lane == 0) {
          mbar_arrive_expect_tx(kf, kTileBytes);
          tma_load_2d(s_k(st), &tm_k, kf, 0, kv_row0 + td.key0);
          tma_load_2d(s_k(st) + kHalfBytes, &tm_k, kf, 64, kv_row0 + td.key0);
          mbar_arrive_expect_tx(vf, kTileBytes);
          tma_load_2d(s_v(st), &tm_v, vf, 0, kv_row0 + td.key0);
          tma_load_2d(s_v(st) + kHalfBytes, &tm_v, vf, 64, kv_row0 + td.key0);
        }
      } else {
        bool bad = false;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          if (j[r] < 0 || j[r] >= a.L) {
            bad = true;
            j[r] = 0;
          }
        }
        if (bad) atomicOr(a.err, kErrBadIndex);
        const int last = __shfl_sync(0xffffffffu, j[3], 31);
        // 128 consecutive keys: every lane's four keys are exactly the next
        // ones (a list entry out of order or repeated keeps the gather path)
        const bool contiguous = (td.valid == 128) && (last - first == 127) && first >= 0 &&
                                first < a.L && last < a.L &&
                                __all_sync(0xffffffffu, j[0] == first + 4 * lane &&
                                                            j[1] == first + 4 * lane + 1 &&
                                                            j[2] == first + 4 * lane + 2 &&
                                                            j[3] == first + 4 * lane + 3);
        if (lane == 0) {
          mbar_arrive_expect_tx(kf, kTileBytes);
          mbar_arrive_expect_tx(vf, kTileBytes);
        }
        __syncwarp();
        if (contiguous) {
          if (lane == 0) {
            tma_load_2d(s_k(st), &tm_k, kf, 0, kv_row0 + first);
            tma_load_2d(s_k(st) + kHalfBytes, &tm_k, kf, 64, kv_row0 + first);
            tma_load_2d(s_v(st), &tm_v, vf, 0, kv_row0 + first);
            tma_load_2d(s_v(st) + kHalfBytes, &tm_v, vf, 64, kv_row0 + first);
          }
        } else {
          const uint32_t roff = lane * 4u * 128u;
          tma_gather4(s_k(st) + roff, &tm_kg, kf, 0, kv_row0 + j[0], kv_row0 + j[1],
                      kv_row0 + j[2], kv_row0 + j[3]);
          tma_gather4(s_k(st) + kHalfBytes + roff, &tm_kg, kf, 64, kv_row0 + j[0],
                      kv_row0 + j[1], kv_row0 + j[2], kv_row0 + j[3]);
          tma_gather4(s_v(st) + roff, &tm_vg, vf, 0, kv_row0 + j[0], kv_row0 + j[1],
                      kv_row0 + j[2], kv_row0 + j[3]);
          tma_gather4(s_v(st) + kHalfBytes + roff, &tm_vg, vf, 64, kv_row0 + j[0],
                      kv_row0 + j[1], kv_row0 + j[2], kv_row0 + j[3]);
        }
      }
      issued = t + 1;
    }
    // Make sure no copy is still in flight before the CTA releases its shared
    // memory (immediate in normal operation, bounded after an abort).
    if (lane == 0) {
      mbar_drain(bar_q, 0, a.wait_ns);
      for (int t = max(0, issued - kAttnStages); t < issued; ++t) {
        mbar_drain(bar_kfull(t % kAttnStages), (t / kAttnStages) & 1, a.wait_ns);
        mbar_drain(bar_vfull(t % kAttnStages), (t / kAttnStages) & 1, a.wait_ns);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = true;
      if (a.debug & 1u) ok = mbar_wait(bar_stall, 0, wc);   // never signalled: test hook
      if (ok) ok = mbar_wait(bar_q, 0, wc);
      auto issue_pv = [&](int u) -> bool {
        const int bu = u & 1, st = u % kAttnStages;
        if (!mbar_wait(bar_pfull0 + 8u * bu, (u >> 1) & 1, wc)) return false;
        if (!mbar_wait(bar_vfull(st), (u / kAttnStages) & 1, wc)) return false;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint64_t bd = smem_desc_sw128(s_v(st) + ks * 2048u, kHalfBytes);
          mma_bf16_ts(tmem + 256u, tmem + 384u + 64u * bu + 8u * ks, bd, kIdescPV,
                      (u > 0 || ks > 0) ? 1u : 0u);
        }
        mma_commit(bar_pvdone0 + 8u * bu);
        mma_commit(bar_empty(st));
        return true;
      };
      for (int t = 0; ok && t < T; ++t) {
        const int st = t % kAttnStages, b = t & 1;
        if (!(ok = mbar_wait(bar_kfull(st), (t / kAttnStages) & 1, wc))) break;
        if (t >= 2 && !(ok = mbar_wait(bar_sfree0 + 8u * b, ((t - 2) >> 1) & 1, wc))) break;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t off = (ks >> 2) * kHalfBytes + (ks & 3) * 32u;
          mma_bf16_ss(tmem + 128u * b, smem_desc_sw128(s_q + off, 16),
                      smem_desc_sw128(s_k(st) + off, 16), kIdescQK, ks > 0 ? 1u : 0u);
        }
        mma_commit(bar_sfull0 + 8u * b);
        if (t >= 1) ok = issue_pv(t - 1);
      }
      if (ok && T > 0) issue_pv(T - 1);
      // every MMA issued by this thread has completed once this arrives
      mma_commit(bar_drain);
      mbar_drain(bar_drain, 0, a.wait_ns);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------- softmax
    const int quad = warp & 3;
    const int r = quad * 32 + lane;            // row within the block
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const float sl2 = a.sl2;
    float m_used = -INFINITY;
    float lsum = 0.f;
    bool ok = true;
    for (int t = 0; t < T; ++t) {
      const int b = t & 1;
      if (!(ok = warp_wait(bar_sfull0 + 8u * b, (t >> 1) & 1, wc))) break;
      tc_fence_after();
      uint32_t sr[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tmem + lane_off + 128u * b + 32u * c, sr[c]);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(bar_sfree0 + 8u * b);

      const TileDesc td = tile_desc(it, t);
      const int limit = td.causal ? min(td.valid, r + 1) : td.valid;
      // row max with eight independent accumulators (no serial chain)
      float mxv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) mxv[u] = -INFINITY;
      if (limit < 128) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            if (c * 32 + e >= limit) sr[c][e] = __float_as_uint(-INFINITY);
          }
        }
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) {
#pragma unroll
        for (int e = 0; e < 32; ++e) mxv[e & 7] = fmaxf(mxv[e & 7], __uint_as_float(sr[c][e]));
      }
      const float mx = fmaxf(fmaxf(fmaxf(mxv[0], mxv[1]), fmaxf(mxv[2], mxv[3])),
                             fmaxf(fmaxf(mxv[4], mxv[5]), fmaxf(mxv[6], mxv[7])));
      const float mx2 = mx * sl2;
      const bool grow = mx2 > m_used + 8.0f;
      if (t == 0) {
        m_used = mx2;
      } else if (__any_sync(0xffffffffu, grow)) {
        // O must hold every PV up to tile t-1 before it is rescaled.
        const int u = t - 1;
        if (!(ok = warp_wait(bar_pvdone0 + 8u * (u & 1), (u >> 1) & 1, wc))) break;
        tc_fence_after();
        const float f = grow ? fast_exp2(m_used - mx2) : 1.0f;
        if (grow) {
          lsum *= f;
          m_used = mx2;
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t ov[32];
          tmem_ld32(tmem + lane_off + 256u + 32u * c, ov);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * f);
          tmem_st32(tmem + lane_off + 256u + 32u * c, ov);
        }
        tmem_st_wait();
      }
      // p = 2^(s * scale * log2 e - m); masked entries give 0
      const float neg_m = -m_used;
      uint32_t pk[2][32];
      float ps[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) ps[u] = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const float p0 = fast_exp2(fmaf(__uint_as_float(sr[c][e]), sl2, neg_m));
          const float p1 = fast_exp2(fmaf(__uint_as_float(sr[c][e + 1]), sl2, neg_m));
          ps[(e >> 1) & 7] += p0 + p1;
          pk[c >> 1][(c & 1) * 16 + (e >> 1)] = pack_bf16x2(p0, p1);
        }
      }
      lsum += ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
      // P_b is free once the PV of tile t-2 has completed
      if (t >= 2 && !(ok = warp_wait(bar_pvdone0 + 8u * b, ((t - 2) >> 1) & 1, wc))) break;
      tc_fence_after();
      tmem_st32(tmem + lane_off + 384u + 64u * b, pk[0]);
      tmem_st32(tmem + lane_off + 384u + 64u * b + 32u, pk[1]);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_pfull0 + 8u * b);
    }
    if (ok && T > 0) {
      const int u = T - 1;
      ok = warp_wait(bar_pvdone0 + 8u * (u & 1), (u >> 1) & 1, wc);
      if (ok) {
        tc_fence_after();
        const int row = it.row0 + r;
        const float inv = 1.0f / lsum;
        __nv_bfloat16* orow =
            a.o + (((long long)(it.b * a.Hq + it.h) * a.L) + row) * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t ov[32];
          tmem_ld32(tmem + lane_off + 256u + 32u * c, ov);
          tmem_ld_wait();
          if (row < a.L) {
            uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) {
              uint4 w;
              w.x = pack_bf16x2(__uint_as_float(ov[8 * v4 + 0]) * inv, __uint_as_float(ov[8 * v4 + 1]) * inv);
              w.y = pack_bf16x2(__uint_as_float(ov[8 * v4 + 2]) * inv, __uint_as_float(ov[8 * v4 + 3]) * inv);
              w.z = pack_bf16x2(__uint_as_float(ov[8 * v4 + 4]) * inv, __uint_as_float(ov[8 * v4 + 5]) * inv);
              w.w = pack_bf16x2(__uint_as_float(ov[8 * v4 + 6]) * inv, __uint_as_float(ov[8 * v4 + 7]) * inv);
              dst[v4] = w;
            }
          }
        }
        if (row < a.L && a.lse != nullptr) {
          a.lse[(long long)(it.b * a.Hq + it.h) * a.L + row] =
              m_used * 0.69314718055994531f + logf(lsum);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace spa
