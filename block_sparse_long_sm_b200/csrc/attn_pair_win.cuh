// attn_pair_win.cuh -- the paired attention of attn_pair.cuh with window
// tiles for the selected keys (selected with SPA_DEBUG_WINDOW_TILES).
//
// The paired kernel cuts the pair's union list into tiles of 128 consecutive
// entries and gathers each one row by row (TMA gather4) unless its 128 keys
// happen to be consecutive.  When a few keys are missing everywhere (a
// near-dense selection) no tile is consecutive, and gather4 issue, not the
// tensor cores, sets the pace.  Here a selected tile starts at the next
// union key k0: when at least kWinMin of the union's keys lie in
// [k0, k0 + 128), the tile is that key window, loaded with two tiled TMA
// copies per operand, and the keys not in the union are masked column by
// column through the per-head membership masks the producer already
// publishes; otherwise the next 128 union keys are gathered as before.
// When both heads keep every candidate of the block (the near-dense case: at
// theta = 5 on the 128K layer every block), the selected keys are simply
// [sink, ls) and go as plain contiguous tiles without reading the list at
// all.  Attention over a key set does not depend on the order of its tiles,
// so the result is the paired kernel's up to rounding.
//
// The number of selected tiles now depends on the keys.  Rather than count
// them up front (a chain of dependent list reads), the producer publishes for
// every tile, through the tag barrier of its V slot, a descriptor (valid
// columns, causal, masked, last) beside the head masks; the MMA warp and the
// softmax warps stop after the tile marked last.  Everything else (roles,
// barriers, TMEM layout, softmax) is the paired kernel's.
#pragma once

#include "attn_pair.cuh"

namespace spa {

constexpr int kWinMin = 96;    // keys in the window for a contiguous tile

__global__ void __launch_bounds__(kPairThreads, 1)
sparse_attn_pair_win_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_kg,
                        const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_vg, const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t s_base = smem_u32(smem);
  const uint32_t s_q = s_base;                                      // Q_A, then Q_B
  auto s_k = [&](int st) { return s_base + kTileBytes * (2 + st); };
  auto s_v = [&](int st) { return s_base + kTileBytes * (2 + kPairKStages + st); };
  uint8_t* bar_area = smem + kTileBytes * (2 + kPairKStages + kPairVStages);
  const uint32_t b0 = smem_u32(bar_area);
  const uint32_t bar_q = b0;
  auto bar_kfull = [&](int st) { return b0 + 8u * (1 + st); };
  auto bar_kempty = [&](int st) { return b0 + 8u * (1 + kPairKStages + st); };
  auto bar_vfull = [&](int st) { return b0 + 8u * (1 + 2 * kPairKStages + st); };
  auto bar_vempty = [&](int st) { return b0 + 8u * (1 + 2 * kPairKStages + kPairVStages + st); };
  const uint32_t bar_sfull0 = b0 + 8u * (1 + 2 * kPairKStages + 2 * kPairVStages);   // [2 heads]
  const uint32_t bar_pfull0 = bar_sfull0 + 16u;                                       // [2 heads]
  const uint32_t bar_odone = bar_sfull0 + 32u;
  const uint32_t bar_drain = bar_sfull0 + 40u;
  const uint32_t bar_stall = bar_sfull0 + 48u;
  const uint32_t bar_tag0 = bar_sfull0 + 56u;                                         // [vstages]
  uint32_t* tags = reinterpret_cast<uint32_t*>(bar_area + 256);   // [vstage][head][4 words]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bar_area + 512);
  volatile uint32_t* abort_flag = tmem_holder + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int st = 0; st < kPairKStages; ++st) {
      mbar_init(bar_kfull(st), 1);
      mbar_init(bar_kempty(st), 1);
    }
    for (int st = 0; st < kPairVStages; ++st) {
      mbar_init(bar_vfull(st), 1);
      mbar_init(bar_vempty(st), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_sfull0 + 8u * i, 1);
      mbar_init(bar_pfull0 + 8u * i, 128);
    }
    for (int st = 0; st < kPairVStages; ++st) mbar_init(bar_tag0 + 8u * st, 1);
    mbar_init(bar_odone, 1);
    mbar_init(bar_drain, 1);
    mbar_init(bar_stall, 1);
    *abort_flag = 0u;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_holder), 512);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
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

  const PairItem pi = pair_item(a, blockIdx.x);
  const AttnItem& it = pi.it;
  const int kv_row0 = (it.b * a.Hkv + it.kvh) * a.L;
  const int n_total = it.n_sel;              // union keys of the block

  // Union keys n + 4 lane + r (r < 4) and their head tags; past the end the
  // first key repeats with an empty tag.
  auto fetch_at = [&](int n, int (&j)[4], uint32_t (&tg)[4]) {
    int first;
    uint32_t ftag;
    pair_sel(a, pi, n, first, ftag);
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int o = n + lane * 4 + r;
      if (o < n_total) {
        pair_sel(a, pi, o, j[r], tg[r]);
      } else {
        j[r] = first;
        tg[r] = 0u;
      }
    }
  };
  // Tiling of the union from ordinal n: the keys within [k0, k0 + 128) of the
  // first one form a contiguous tile when there are at least kWinMin of them;
  // otherwise the next 128 keys are gathered.  Returns the keys consumed.
  auto decide = [&](int n, const int (&j)[4], bool& window, int& k0) -> int {
    k0 = __shfl_sync(0xffffffffu, j[0], 0);
    int cnt = 0;
#pragma unroll
    for (int r = 0; r < 4; ++r) cnt += (n + lane * 4 + r < n_total && j[r] < k0 + 128) ? 1 : 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    window = cnt >= kWinMin;
    return window ? cnt : min(128, n_total - n);
  };
  // Per V slot, the descriptor of the tile in it: valid columns (bits 0-8),
  // causal diagonal (9), masked through the head masks (10), last tile (11).
  // Written by the producer before it arrives on the slot's tag barrier.
  uint32_t* tdesc = reinterpret_cast<uint32_t*>(bar_area + 528);

  // Register split: the load/MMA warpgroup needs few registers, the softmax
  // warpgroups hold a full 128-column S row each.  Launched with 168 per
  // thread (384 threads): 128 x (168 - 40) = 256 x (232 - 168).
  if (warp >= 8) {
  // Register split: the load/MMA warpgroup (warps 8-11, executing this one
  // instruction together) needs few registers, the softmax warpgroups hold a
  // full 128-column S row each.  Launched with 168 per thread (384 threads):
  // 128 x 80 + 256 x 208 <= 384 x 168.
  asm volatile("setmaxnreg.dec.sync.aligned.u32 80;" ::: "memory");
  if (warp == 8) {
    // ------------------------------------------------------------- producer
    int issued = 0;
    if (lane == 0) {
      mbar_arrive_expect_tx(bar_q, 2 * kTileBytes);
      const int qrow = (it.b * a.Hq + it.h) * a.L + it.row0;
      tma_load_2d(s_q, &tm_q, bar_q, 0, qrow);
      tma_load_2d(s_q + kHalfBytes, &tm_q, bar_q, 64, qrow);
      tma_load_2d(s_q + kTileBytes, &tm_q, bar_q, 0, qrow + a.L);
      tma_load_2d(s_q + kTileBytes + kHalfBytes, &tm_q, bar_q, 64, qrow + a.L);
    }
    int nj[4] = {0, 0, 0, 0};
    uint32_t ntg[4] = {0u, 0u, 0u, 0u};
    int n_cur = 0;                             // union ordinal of the next selected tile
    int loc = 0;                               // local tiles issued
    // both heads keep every candidate (the union has every candidate and the
    // two lists never differ: the shared prefix is the whole union), so the
    // selected keys are [sink, ls), loaded as plain contiguous tiles without
    // reading the list
    const bool all_kept = n_total > 0 && n_total == max(0, it.ls - a.sink) &&
                          pi.split * a.list_unit >= n_total;
    if (n_total > 0 && !all_kept) fetch_at(0, nj, ntg);
    for (int t = 0;; ++t) {
      const int ks = t % kPairKStages, vs = t % kPairVStages;
      if (t >= kPairKStages &&
          !warp_wait(bar_kempty(ks), ((t / kPairKStages) - 1) & 1, wc))
        break;
      if (t >= kPairVStages &&
          !warp_wait(bar_vempty(vs), ((t / kPairVStages) - 1) & 1, wc))
        break;
      // tile t: sink tiles, then selected tiles while union keys remain, then
      // local tiles (there is always one: the diagonal)
      TileDesc td;
      bool last = false;
      if (t < it.n_sink_t) {
        td.gather = 0;
        td.key0 = t * 128;
        td.valid = min(128, it.sink_end - td.key0);
        td.causal = 0;
      } else if (n_cur < n_total && all_kept) {
        td.gather = 0;
        td.key0 = a.sink + n_cur;
        td.valid = min(128, n_total - n_cur);
        td.causal = 0;
        n_cur += td.valid;
      } else if (n_cur < n_total) {
        td.gather = 1;
        td.key0 = 0;
        td.valid = 128;
        td.causal = 0;
      } else {
        td.gather = 0;
        td.key0 = it.loc_start + loc * 128;
        td.valid = min(128, it.le - td.key0);
        td.causal = (td.key0 == it.row0);
        last = ++loc == it.n_loc_t;
      }
      const uint32_t kf = bar_kfull(ks), vf = bar_vfull(vs);
      bool contiguous = !td.gather;
      int key0 = td.key0;
      int j[4] = {nj[0], nj[1], nj[2], nj[3]};
      const uint32_t tg[4] = {ntg[0], ntg[1], ntg[2], ntg[3]};
      if (td.gather) {
        bool window;
        int k0;
        const int used = decide(n_cur, j, window, k0);
        n_cur += used;
        if (n_cur < n_total) fetch_at(n_cur, nj, ntg);   // the next selected tile's keys
        bool bad = false;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          if (j[r] < 0 || j[r] >= a.L) {
            bad = true;
            j[r] = 0;
          }
        }
        if (k0 < 0 || k0 >= a.L) {
          bad = true;
          k0 = 0;
        }
        if (bad) atomicOr(a.err, kErrBadIndex);
        // membership masks, bit c of word w <=> column 32w + c belongs to the head:
        // a window tile's column is key - k0, a gathered tile's its row 4 lane + r
        // (the slot's masks are free: the PV that read them has completed)
        if (lane < 8) tags[vs * 8 + lane] = 0u;
        __syncwarp();
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int ord = lane * 4 + r;
          const int col = window ? j[r] - k0 : ord;
          const bool in = window ? (ord < used) : true;   // padding rows carry tag 0
          if (in && (tg[r] & 1u)) atomicOr(&tags[(vs * 2 + 0) * 4 + (col >> 5)], 1u << (col & 31));
          if (in && (tg[r] & 2u)) atomicOr(&tags[(vs * 2 + 1) * 4 + (col >> 5)], 1u << (col & 31));
        }
        __syncwarp();
        contiguous = window;
        key0 = k0;
      }
      // every tile publishes its descriptor (and a selected tile its masks)
      if (lane == 0) {
        tdesc[vs] = static_cast<uint32_t>(td.valid) | (static_cast<uint32_t>(td.causal) << 9) |
                    (static_cast<uint32_t>(td.gather) << 10) | (last ? 1u << 11 : 0u);
        mbar_arrive(bar_tag0 + 8u * vs);
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_expect_tx(kf, kTileBytes);
        mbar_arrive_expect_tx(vf, kTileBytes);
      }
      __syncwarp();
      if (contiguous) {
        if (lane == 0) {
          tma_load_2d(s_k(ks), &tm_k, kf, 0, kv_row0 + key0);
          tma_load_2d(s_k(ks) + kHalfBytes, &tm_k, kf, 64, kv_row0 + key0);
          tma_load_2d(s_v(vs), &tm_v, vf, 0, kv_row0 + key0);
          tma_load_2d(s_v(vs) + kHalfBytes, &tm_v, vf, 64, kv_row0 + key0);
        }
      } else {
        const uint32_t roff = lane * 4u * 128u;
        tma_gather4(s_k(ks) + roff, &tm_kg, kf, 0, kv_row0 + j[0], kv_row0 + j[1],
                    kv_row0 + j[2], kv_row0 + j[3]);
        tma_gather4(s_k(ks) + kHalfBytes + roff, &tm_kg, kf, 64, kv_row0 + j[0],
                    kv_row0 + j[1], kv_row0 + j[2], kv_row0 + j[3]);
        tma_gather4(s_v(vs) + roff, &tm_vg, vf, 0, kv_row0 + j[0], kv_row0 + j[1],
                    kv_row0 + j[2], kv_row0 + j[3]);
        tma_gather4(s_v(vs) + kHalfBytes + roff, &tm_vg, vf, 64, kv_row0 + j[0],
                    kv_row0 + j[1], kv_row0 + j[2], kv_row0 + j[3]);
      }
      issued = t + 1;
      if (last) break;
    }
    if (lane == 0) {   // no copy may still be in flight when the CTA exits
      mbar_drain(bar_q, 0, a.wait_ns);
      for (int t = max(0, issued - kPairKStages); t < issued; ++t)
        mbar_drain(bar_kfull(t % kPairKStages), (t / kPairKStages) & 1, a.wait_ns);
      for (int t = max(0, issued - kPairVStages); t < issued; ++t)
        mbar_drain(bar_vfull(t % kPairVStages), (t / kPairVStages) & 1, a.wait_ns);
    }
  } else if (warp == 9) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = true;
      if (a.debug & 1u) ok = mbar_wait(bar_stall, 0, wc);   // never signalled: test hook
      if (ok) ok = mbar_wait(bar_q, 0, wc);
      auto qk = [&](int t, int hd) {
        const int ks = t % kPairKStages;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32u;
          mma_bf16_ss(tmem + 128u * hd, smem_desc_sw128(s_q + hd * kTileBytes + off, 16),
                      smem_desc_sw128(s_k(ks) + off, 16), kIdescQK, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar_sfull0 + 8u * hd);
      };
      auto pv = [&](int t, int hd) {
        const int vs = t % kPairVStages;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t bd = smem_desc_sw128(s_v(vs) + kk * 2048u, kHalfBytes);
          mma_bf16_ts(tmem + 256u + 128u * hd, tmem + 128u * hd + 8u * kk, bd, kIdescPV,
                      (t > 0 || kk > 0) ? 1u : 0u);
        }
      };
      if (ok) {
        if ((ok = mbar_wait(bar_kfull(0), 0, wc))) {
          tc_fence_after();
          qk(0, 0);
          qk(0, 1);
          mma_commit(bar_kempty(0));
        }
      }
      for (int t = 0; ok; ++t) {
        const int vs = t % kPairVStages;
        // tile t's descriptor was written before its K copy was armed, and
        // kfull of tile t has been observed (QK(t) is issued)
        const bool more = ((tdesc[vs] >> 11) & 1u) == 0u;
        // head A: PV(t), then QK(t+1)
        if (!(ok = mbar_wait(bar_pfull0, t & 1, wc))) break;
        if (!(ok = mbar_wait(bar_vfull(vs), (t / kPairVStages) & 1, wc))) break;
        tc_fence_after();
        pv(t, 0);
        if (more) {
          const int ks = (t + 1) % kPairKStages;
          if (!(ok = mbar_wait(bar_kfull(ks), ((t + 1) / kPairKStages) & 1, wc))) break;
          tc_fence_after();
          qk(t + 1, 0);
        }
        // head B: PV(t), then QK(t+1)
        if (!(ok = mbar_wait(bar_pfull0 + 8u, t & 1, wc))) break;
        tc_fence_after();
        pv(t, 1);
        mma_commit(bar_vempty(vs));
        if (more) {
          qk(t + 1, 1);
          mma_commit(bar_kempty((t + 1) % kPairKStages));
        } else {
          mma_commit(bar_odone);
          break;
        }
      }
      mma_commit(bar_drain);
      mbar_drain(bar_drain, 0, a.wait_ns);
    }
    __syncwarp();
  }   // warps 10-11 have no role
  } else {
    // ------------------------------------------------------------- softmax
    asm volatile("setmaxnreg.inc.sync.aligned.u32 208;" ::: "memory");
    const int hd = warp >> 2;                  // 0: head A (warps 0-3), 1: head B (4-7)
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t s_col = 128u * hd, o_col = 256u + 128u * hd;
    const float sl2 = a.sl2;
    float m_used = -INFINITY;
    float lsum = 0.f;
    bool ok = true;
    bool last = false;
    for (int t = 0; !last; ++t) {
      if (!(ok = warp_wait(bar_sfull0 + 8u * hd, t & 1, wc))) break;
      tc_fence_after();
      // every tile arrives once on its V slot's tag barrier
      const int vs = t % kPairVStages;
      if (!(ok = warp_wait(bar_tag0 + 8u * vs, (t / kPairVStages) & 1, wc))) break;
      const uint32_t dw = tdesc[vs];
      last = ((dw >> 11) & 1u) != 0u;
      const int valid = static_cast<int>(dw & 0x1FFu);
      const int limit = ((dw >> 9) & 1u) ? min(valid, r + 1) : valid;
      uint32_t tw[4] = {0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu};
      if ((dw >> 10) & 1u) {
#pragma unroll
        for (int w = 0; w < 4; ++w) tw[w] = tags[(vs * 2 + hd) * 4 + w];
      }
      uint32_t sr[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tmem + lane_off + s_col + 32u * c, sr[c]);
      tmem_ld_wait();
      const bool masked = (limit < 128) || ((tw[0] & tw[1] & tw[2] & tw[3]) != 0xffffffffu);
      if (masked) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const bool v = (c * 32 + e < limit) && ((tw[c] >> e) & 1u);
            if (!v) sr[c][e] = __float_as_uint(-INFINITY);
          }
      }
      float mxv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) mxv[u] = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int e = 0; e < 32; ++e) mxv[e & 7] = fmaxf(mxv[e & 7], __uint_as_float(sr[c][e]));
      const float mx = fmaxf(fmaxf(fmaxf(mxv[0], mxv[1]), fmaxf(mxv[2], mxv[3])),
                             fmaxf(fmaxf(mxv[4], mxv[5]), fmaxf(mxv[6], mxv[7])));
      const float mx2 = mx * sl2;
      const bool grow = mx2 > m_used + 8.0f;
      if (t == 0) {
        m_used = mx2;
      } else if (__any_sync(0xffffffffu, grow)) {
        // every PV of this head up to tile t-1 completed before S_t was ready
        const float f = grow ? fast_exp2(m_used - mx2) : 1.0f;
        if (grow) {
          lsum *= f;
          m_used = mx2;
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t ov[32];
          tmem_ld32(tmem + lane_off + o_col + 32u * c, ov);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * f);
          tmem_st32(tmem + lane_off + o_col + 32u * c, ov);
        }
        tmem_st_wait();
      }
      // p = 2^(s * scale * log2 e - m) -> P (bf16) into S's first 64 columns
      // (S is entirely in registers by now)
      const float neg_m = (m_used == -INFINITY) ? 0.f : -m_used;
      float ps[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) ps[u] = 0.f;
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int c = 2 * h2 + cc;
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const float x0 = fmaf(__uint_as_float(sr[c][e]), sl2, neg_m);
            const float x1 = fmaf(__uint_as_float(sr[c][e + 1]), sl2, neg_m);
#if SPA_EXP2_POLY_EVERY > 0
            const bool poly = ((e >> 1) % SPA_EXP2_POLY_EVERY) == SPA_EXP2_POLY_EVERY - 1;
#else
            const bool poly = false;
#endif
            const float p0 = poly ? poly_exp2(x0) : fast_exp2(x0);
            const float p1 = poly ? poly_exp2(x1) : fast_exp2(x1);
            ps[(e >> 1) & 7] += p0 + p1;
            sr[c][e >> 1] = pack_bf16x2(p0, p1);   // in place: index e/2 was consumed
          }
        }
        tmem_st32_halves(tmem + lane_off + s_col + 32u * h2, sr[2 * h2], sr[2 * h2 + 1]);
      }
      lsum += ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_pfull0 + 8u * hd);
    }
    if (ok) {
      ok = warp_wait(bar_odone, 0, wc);
      if (ok) {
        tc_fence_after();
        const int h = it.h + hd;
        const int row = it.row0 + r;
        const float inv = 1.0f / lsum;
        __nv_bfloat16* orow = a.o + (((long long)(it.b * a.Hq + h) * a.L) + row) * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t ov[32];
          tmem_ld32(tmem + lane_off + o_col + 32u * c, ov);
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
          a.lse[(long long)(it.b * a.Hq + h) * a.L + row] =
              m_used * 0.69314718055994531f + logf(lsum);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) tmem_dealloc(tmem, 512);
}

}  // namespace spa
