// attn_pair_fp8.cuh -- the paired attention (two q heads of one kv head per
// CTA, their softmaxes out of phase with the other head's GEMMs) with E4M3
// operands on the tcgen05 kind::f8f6f4 tensor cores: SALE's Computation Pass
// on quantised operands ("SageAttention-style", the review of SALE,
// Summary), at the schedule that keeps the bf16 kernel near peak.
//
// Relative to attn_pair.cuh: 16 KiB tiles (one TMA box, or one gather4 per
// four rows, per operand), rings of 4 K and 3 V stages; S = four SS MMAs of
// K = 32; P = 2^(x - m + 7) as E4M3 in the first 32 columns of S (the
// running max raised only past 1.75, so P < 448), O += P V as four TS MMAs
// with V MN-major; the scores carry s_q(block) s_k(head), the epilogue
// scales channel c by s_v[c] / l and adds the K-smoothing shift
// scale q^_r . mu back to the LSE.  Roles, barriers, masks and the register
// split are the paired kernel's.
#pragma once

#include "attn_fp8.cuh"
#include "attn_pair.cuh"

namespace spa {

constexpr int kPF8KStages = 4;
constexpr int kPF8VStages = 3;
constexpr uint32_t kPF8BarBytes = 2048u;      // barriers, masks, V scales, K mean
constexpr uint32_t kPF8SmemBytes =
    1024u + 2u * kTile8 + (kPF8KStages + kPF8VStages) * kTile8 + kPF8BarBytes;
static_assert(kPF8SmemBytes <= 232448u, "more shared memory than a CTA may use");

struct PairF8Args {
  AttnArgs base;              // geometry, lists, union lists, O, LSE, error word
  const float* qs;            // [B*Hq][nqb]
  const float* ks;            // [B*Hkv]
  const float* vs;            // [B*Hkv][128]
  const float* kmean;         // [B*Hkv][128]
  float scale;                // softmax scale (natural units), for the LSE shift
};

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
      : "memory");
}

__global__ void __launch_bounds__(kPairThreads, 1)
sparse_attn_pair_fp8_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_kg,
                        const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_vg, const PairF8Args f) {
  const AttnArgs& a = f.base;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t s_base = smem_u32(smem);
  const uint32_t s_q = s_base;                                      // Q_A, then Q_B
  auto s_k = [&](int st) { return s_base + kTile8 * (2 + st); };
  auto s_v = [&](int st) { return s_base + kTile8 * (2 + kPF8KStages + st); };
  uint8_t* bar_area = smem + kTile8 * (2 + kPF8KStages + kPF8VStages);
  const uint32_t b0 = smem_u32(bar_area);
  const uint32_t bar_q = b0;
  auto bar_kfull = [&](int st) { return b0 + 8u * (1 + st); };
  auto bar_kempty = [&](int st) { return b0 + 8u * (1 + kPF8KStages + st); };
  auto bar_vfull = [&](int st) { return b0 + 8u * (1 + 2 * kPF8KStages + st); };
  auto bar_vempty = [&](int st) { return b0 + 8u * (1 + 2 * kPF8KStages + kPF8VStages + st); };
  const uint32_t bar_sfull0 = b0 + 8u * (1 + 2 * kPF8KStages + 2 * kPF8VStages);   // [2 heads]
  const uint32_t bar_pfull0 = bar_sfull0 + 16u;                                       // [2 heads]
  const uint32_t bar_odone = bar_sfull0 + 32u;
  const uint32_t bar_drain = bar_sfull0 + 40u;
  const uint32_t bar_stall = bar_sfull0 + 48u;
  const uint32_t bar_tag0 = bar_sfull0 + 56u;                                         // [vstages]
  uint32_t* tags = reinterpret_cast<uint32_t*>(bar_area + 256);   // [vstage][head][4 words]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bar_area + 512);
  volatile uint32_t* abort_flag = tmem_holder + 1;
  float* vscale = reinterpret_cast<float*>(bar_area + 1024);   // 128 channel scales
  float* kmu = reinterpret_cast<float*>(bar_area + 1536);      // 128 K means
  static_assert(8 * (1 + 2 * kPF8KStages + 2 * kPF8VStages) + 56 + 8 * kPF8VStages <= 256,
                "barriers overlap the masks");
  static_assert(256 + kPF8VStages * 2 * 4 * 4 <= 512, "masks overlap the TMEM holder");
  static_assert(1536 + 512 <= kPF8BarBytes, "K means overflow the barrier area");

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int st = 0; st < kPF8KStages; ++st) {
      mbar_init(bar_kfull(st), 1);
      mbar_init(bar_kempty(st), 1);
    }
    for (int st = 0; st < kPF8VStages; ++st) {
      mbar_init(bar_vfull(st), 1);
      mbar_init(bar_vempty(st), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_sfull0 + 8u * i, 1);
      mbar_init(bar_pfull0 + 8u * i, 128);
    }
    for (int st = 0; st < kPF8VStages; ++st) mbar_init(bar_tag0 + 8u * st, 1);
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
  const int T = it.n_sink_t + it.n_sel_t + it.n_loc_t;
  const int kv_row0 = (it.b * a.Hkv + it.kvh) * a.L;
  if (threadIdx.x < 128) {       // the kv head's V scales and K mean, for the epilogue
    const long long c = (long long)(it.b * a.Hkv + it.kvh) * 128 + threadIdx.x;
    vscale[threadIdx.x] = f.vs[c];
    kmu[threadIdx.x] = f.kmean[c];
  }
  __syncthreads();

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
      mbar_arrive_expect_tx(bar_q, 2 * kTile8);
      const int qrow = (it.b * a.Hq + it.h) * a.L + it.row0;
      tma_load_2d(s_q, &tm_q, bar_q, 0, qrow);
      tma_load_2d(s_q + kTile8, &tm_q, bar_q, 0, qrow + a.L);
    }
    // Union entries of this lane's four rows of a selected tile, fetched one
    // tile ahead (padding rows repeat the first key with an empty tag).
    auto fetch = [&](int t, int (&j)[4], uint32_t (&tg)[4]) {
      const TileDesc td = tile_desc(it, t);
      if (!td.gather) return;
      int first;
      uint32_t ftag;
      pair_sel(a, pi, td.key0, first, ftag);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int row = lane * 4 + r;
        if (row < td.valid) {
          pair_sel(a, pi, td.key0 + row, j[r], tg[r]);
        } else {
          j[r] = first;
          tg[r] = 0u;
        }
      }
    };
    int nj[4] = {0, 0, 0, 0};
    uint32_t ntg[4] = {0u, 0u, 0u, 0u};
    if (T > 0) fetch(0, nj, ntg);
    for (int t = 0; t < T; ++t) {
      int j[4] = {nj[0], nj[1], nj[2], nj[3]};
      const uint32_t tg[4] = {ntg[0], ntg[1], ntg[2], ntg[3]};
      if (t + 1 < T) fetch(t + 1, nj, ntg);
      const int ks = t % kPF8KStages, vs = t % kPF8VStages;
      if (t >= kPF8KStages &&
          !warp_wait(bar_kempty(ks), ((t / kPF8KStages) - 1) & 1, wc))
        break;
      if (t >= kPF8VStages &&
          !warp_wait(bar_vempty(vs), ((t / kPF8VStages) - 1) & 1, wc))
        break;
      const TileDesc td = tile_desc(it, t);
      const uint32_t kf = bar_kfull(ks), vf = bar_vfull(vs);
      bool contiguous = !td.gather;
      int key0 = td.key0;
      if (td.gather) {
        bool bad = false;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          if (j[r] < 0 || j[r] >= a.L) {
            bad = true;
            j[r] = 0;
          }
        }
        if (bad) atomicOr(a.err, kErrBadIndex);
        // membership masks: bit c of word w <=> row 32w + c belongs to the head.
        // Lane l holds rows 4l..4l+3, i.e. bits 4(l%8)..4(l%8)+3 of word l/8.
        uint32_t ma = 0, mb = 0;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          ma |= (tg[r] & 1u) << r;
          mb |= ((tg[r] >> 1) & 1u) << r;
        }
        ma <<= 4 * (lane & 7);
        mb <<= 4 * (lane & 7);
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) {
          ma |= __shfl_xor_sync(0xffffffffu, ma, o);
          mb |= __shfl_xor_sync(0xffffffffu, mb, o);
        }
        if ((lane & 7) == 0) {
          tags[(vs * 2 + 0) * 4 + (lane >> 3)] = ma;
          tags[(vs * 2 + 1) * 4 + (lane >> 3)] = mb;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_tag0 + 8u * vs);   // publishes this tile's masks
        const int first = __shfl_sync(0xffffffffu, j[0], 0);
        const int last = __shfl_sync(0xffffffffu, j[3], 31);
        // 128 consecutive keys: every lane's four keys are exactly the next
        // ones (a list entry out of order or repeated keeps the gather path)
        contiguous = (td.valid == 128) && (last - first == 127) &&
                     __all_sync(0xffffffffu, j[0] == first + 4 * lane && j[1] == first + 4 * lane + 1 &&
                                                 j[2] == first + 4 * lane + 2 &&
                                                 j[3] == first + 4 * lane + 3);
        key0 = first;
      }
      if (lane == 0) {
        mbar_arrive_expect_tx(kf, kTile8);
        mbar_arrive_expect_tx(vf, kTile8);
      }
      __syncwarp();
      if (contiguous) {
        if (lane == 0) {
          tma_load_2d(s_k(ks), &tm_k, kf, 0, kv_row0 + key0);
          tma_load_2d(s_v(vs), &tm_v, vf, 0, kv_row0 + key0);
        }
      } else {
        const uint32_t roff = lane * 4u * 128u;
        tma_gather4(s_k(ks) + roff, &tm_kg, kf, 0, kv_row0 + j[0], kv_row0 + j[1],
                    kv_row0 + j[2], kv_row0 + j[3]);
        tma_gather4(s_v(vs) + roff, &tm_vg, vf, 0, kv_row0 + j[0], kv_row0 + j[1],
                    kv_row0 + j[2], kv_row0 + j[3]);
      }
      issued = t + 1;
    }
    if (lane == 0) {   // no copy may still be in flight when the CTA exits
      mbar_drain(bar_q, 0, a.wait_ns);
      for (int t = max(0, issued - kPF8KStages); t < issued; ++t)
        mbar_drain(bar_kfull(t % kPF8KStages), (t / kPF8KStages) & 1, a.wait_ns);
      for (int t = max(0, issued - kPF8VStages); t < issued; ++t)
        mbar_drain(bar_vfull(t % kPF8VStages), (t / kPF8VStages) & 1, a.wait_ns);
    }
  } else if (warp == 9) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = true;
      if (a.debug & 1u) ok = mbar_wait(bar_stall, 0, wc);   // never signalled: test hook
      if (ok) ok = mbar_wait(bar_q, 0, wc);
      auto qk = [&](int t, int hd) {
        const int ks = t % kPF8KStages;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          // 32 E4M3 elements = 32 bytes along the swizzled 128-byte row
          mma_f8_ss(tmem + 128u * hd, smem_desc_sw128(s_q + hd * kTile8 + kk * 32u, 16),
                    smem_desc_sw128(s_k(ks) + kk * 32u, 16), kIdescQK8, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar_sfull0 + 8u * hd);
      };
      auto pv = [&](int t, int hd) {
        const int vs = t % kPF8VStages;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          // 32 keys = 32 rows of the MN-major V tile; P in S's first 32 columns
          const uint64_t bd = smem_desc_sw128(s_v(vs) + kk * 4096u, kTile8);
          mma_f8_ts(tmem + 256u + 128u * hd, tmem + 128u * hd + 8u * kk, bd, kIdescPV8,
                    (t > 0 || kk > 0) ? 1u : 0u);
        }
      };
      if (ok && T > 0) {
        if ((ok = mbar_wait(bar_kfull(0), 0, wc))) {
          tc_fence_after();
          qk(0, 0);
          qk(0, 1);
          mma_commit(bar_kempty(0));
        }
      }
      for (int t = 0; ok && t < T; ++t) {
        const int vs = t % kPF8VStages;
        const bool more = t + 1 < T;
        // head A: PV(t), then QK(t+1)
        if (!(ok = mbar_wait(bar_pfull0, t & 1, wc))) break;
        if (!(ok = mbar_wait(bar_vfull(vs), (t / kPF8VStages) & 1, wc))) break;
        tc_fence_after();
        pv(t, 0);
        if (more) {
          const int ks = (t + 1) % kPF8KStages;
          if (!(ok = mbar_wait(bar_kfull(ks), ((t + 1) / kPF8KStages) & 1, wc))) break;
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
          mma_commit(bar_kempty((t + 1) % kPF8KStages));
        } else {
          mma_commit(bar_odone);
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
    const long long bh = (long long)it.b * a.Hq + it.h + hd;
    const float q_scale = f.qs[bh * a.nqb + it.qb];
    const float sl2 = a.sl2 * q_scale * f.ks[it.b * a.Hkv + it.kvh];
    float m_used = -INFINITY;
    float lsum = 0.f;
    uint32_t tag_phase = 0u;                   // bit vs: phase of tag barrier vs
    bool ok = true;
    for (int t = 0; t < T; ++t) {
      if (!(ok = warp_wait(bar_sfull0 + 8u * hd, t & 1, wc))) break;
      tc_fence_after();
      const TileDesc td = tile_desc(it, t);
      const int limit = td.causal ? min(td.valid, r + 1) : td.valid;
      uint32_t tw[4] = {0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu};
      if (td.gather) {
        const int vs = t % kPF8VStages;
        // tag barrier phases of this slot count the gathered tiles that used it
        if (!(ok = warp_wait(bar_tag0 + 8u * vs, (tag_phase >> vs) & 1u, wc))) break;
        tag_phase ^= 1u << vs;
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
      const bool grow = mx2 > m_used + kF8Lazy;
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
      // p = 2^(s * scale * log2 e - m + 7) < 2^8.75 -> P (E4M3, four per
      // column) into S's first 32 columns (S is entirely in registers by now)
      const float shift = (m_used == -INFINITY) ? 0.f : kF8PShift - m_used;
      float ps[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) ps[u] = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const float p0 = fast_exp2(fmaf(__uint_as_float(sr[c][e]), sl2, shift));
          const float p1 = fast_exp2(fmaf(__uint_as_float(sr[c][e + 1]), sl2, shift));
          const float p2 = fast_exp2(fmaf(__uint_as_float(sr[c][e + 2]), sl2, shift));
          const float p3 = fast_exp2(fmaf(__uint_as_float(sr[c][e + 3]), sl2, shift));
          ps[(e >> 2) & 7] += (p0 + p1) + (p2 + p3);
          sr[c][e >> 2] = e4m3x2(p0, p1) | (e4m3x2(p2, p3) << 16);   // index e/4 consumed
        }
        tmem_st8(tmem + lane_off + s_col + 8u * c, sr[c]);
      }
      lsum += ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_pfull0 + 8u * hd);
    }
    if (ok && T > 0) {
      ok = warp_wait(bar_odone, 0, wc);
      if (ok) {
        tc_fence_after();
        const int h = it.h + hd;
        const int row = it.row0 + r;
        const float inv = 1.0f / lsum;
        __nv_bfloat16* orow = a.o + (((long long)(it.b * a.Hq + h) * a.L) + row) * 128;
        const uint32_t own_q = hd * kTile8;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t ov[32];
          tmem_ld32(tmem + lane_off + o_col + 32u * c, ov);
          tmem_ld_wait();
          if (row < a.L) {
            uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
            const float* vsc = vscale + 32 * c;
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) {
              float x[8];
#pragma unroll
              for (int e = 0; e < 8; ++e)
                x[e] = __uint_as_float(ov[8 * v4 + e]) * (inv * vsc[8 * v4 + e]);
              uint4 w;
              w.x = pack_bf16x2(x[0], x[1]);
              w.y = pack_bf16x2(x[2], x[3]);
              w.z = pack_bf16x2(x[4], x[5]);
              w.w = pack_bf16x2(x[6], x[7]);
              dst[v4] = w;
            }
          }
        }
        // the Q tile is read with generic loads: observe its TMA completion
        if (a.lse != nullptr && !warp_wait(bar_q, 0, wc)) ok = false;
        if (ok && row < a.L && a.lse != nullptr) {
          // q^_r . mu from row r of this head's swizzled Q code tile
          float dot = 0.f;
#pragma unroll 4
          for (int c16 = 0; c16 < 8; ++c16) {
            const uint4 w = *reinterpret_cast<const uint4*>(smem + own_q + sw128_offset(r, c16 * 16));
            const uint32_t wd[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float2 lo = e4m3x2_to_f32(wd[i] & 0xffffu);
              const float2 hi = e4m3x2_to_f32(wd[i] >> 16);
              const float* mu = kmu + c16 * 16 + i * 4;
              dot = fmaf(lo.x, mu[0], dot);
              dot = fmaf(lo.y, mu[1], dot);
              dot = fmaf(hi.x, mu[2], dot);
              dot = fmaf(hi.y, mu[3], dot);
            }
          }
          a.lse[(long long)(it.b * a.Hq + h) * a.L + row] =
              (m_used - kF8PShift) * 0.69314718055994531f + logf(lsum) + f.scale * q_scale * dot;
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
