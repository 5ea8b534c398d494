// attn_pair.cuh -- sparse causal attention forward for two q heads of one GQA
// group at once, sharing every K/V tile (used when Hq / Hkv is even).
//
// Same computation as sparse_attn_kernel (AnchorAttention Sec. 3.4 /
// SALE Computation Pass, FlashAttention online softmax), organised so that
// the exponentials of one head overlap the tensor-core work of the other:
//
//   * one CTA = (b, kv head, query block, head pair (2p, 2p+1)); the key
//     sequence is sink tiles, the tiles of the pair's *union* list (every
//     entry carries which of the two heads kept it; up to the first entry
//     where the heads differ the union is head A's own list), and local
//     tiles;
//   * warp 8 loads Q of both heads once and K/V tiles into rings of 3 (K) and
//     2 (V) stages, gathering selected rows with TMA gather4, and publishes a
//     128-bit membership mask per head for each selected tile;
//   * warp 9 issues tcgen05.mma in the order PV_A(t), QK_A(t+1), PV_B(t),
//     QK_B(t+1): the tensor core runs one head's GEMMs while the other head's
//     softmax works.  P is written by the softmax into the first 64 columns of
//     its own S accumulator and read from there by the PV GEMM; the next QK
//     GEMM into the same columns is issued after that PV GEMM, and tcgen05
//     MMAs from one thread execute in issue order;
//   * warps 0-3 are head A's softmax and warps 4-7 head B's (thread = row =
//     TMEM lane).  Per tile: row max, then
//     exponentials + P: S is read once into registers (four TMEM loads, one
//     wait); P overwrites S's first 64 columns.
//
// TMEM columns: S_A [0,128) (P_A in [0,64)), S_B [128,256) (P_B in
// [128,192)), O_A [256,384), O_B [384,512).
#pragma once

#include "attn.cuh"
#include "ptx.cuh"

// One exponential pair in SPA_EXP2_POLY_EVERY goes through the FMA-pipe
// polynomial instead of MUFU (0: none).
#ifndef SPA_EXP2_POLY_EVERY
#define SPA_EXP2_POLY_EVERY 0
#endif

namespace spa {

constexpr int kPairKStages = 3;
constexpr int kPairVStages = 2;
constexpr int kPairThreads = 384;   // 3 warpgroups: softmax A, softmax B, load + MMA
constexpr uint32_t kPairBarBytes = 1024u;
constexpr uint32_t kPairSmemBytes =
    1024u + 2u * kTileBytes + (kPairKStages + kPairVStages) * kTileBytes + kPairBarBytes;
static_assert(kPairSmemBytes <= 232448u, "more shared memory than a CTA may use");

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

// 32 columns from the first 16 registers of two arrays.
__device__ __forceinline__ void tmem_st32_halves(uint32_t taddr, const uint32_t* a,
                                                 const uint32_t* b) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(a[4]), "r"(a[5]), "r"(a[6]), "r"(a[7]),
      "r"(a[8]), "r"(a[9]), "r"(a[10]), "r"(a[11]), "r"(a[12]), "r"(a[13]), "r"(a[14]),
      "r"(a[15]), "r"(b[0]), "r"(b[1]), "r"(b[2]), "r"(b[3]), "r"(b[4]), "r"(b[5]), "r"(b[6]),
      "r"(b[7]), "r"(b[8]), "r"(b[9]), "r"(b[10]), "r"(b[11]), "r"(b[12]), "r"(b[13]),
      "r"(b[14]), "r"(b[15])
      : "memory");
}

struct PairItem {
  AttnItem it;     // geometry; it.h is head A, it.n_sel counts union keys
  int pair;        // b * Hq / 2 + hA / 2
  int split;       // union entries before the two heads' lists first differ
  long long a_off; // head A's list of this block: the union's first `split` entries
};

__device__ __forceinline__ PairItem pair_item(const AttnArgs& a, int x) {
  PairItem pi;
  AttnItem& it = pi.it;
  const int ppk = a.group / 2;                 // head pairs per kv head
  const int per_kv = a.nqb * ppk;
  const int bkv = x / per_kv;
  const int rem = x - bkv * per_kv;
  it.qb = a.nqb - 1 - rem / ppk;
  const int pp = rem % ppk;
  it.b = bkv / a.Hkv;
  it.kvh = bkv - it.b * a.Hkv;
  it.h = it.kvh * a.group + 2 * pp;
  pi.pair = it.b * (a.Hq / 2) + it.h / 2;
  it.row0 = it.qb * 128;
  it.le = min(it.row0 + 128, a.L);
  it.ls = max(0, it.row0 + 128 - a.local);
  it.sink_end = min(a.sink, it.ls);
  pi.split = 0;
  pi.a_off = 0;
  if (a.mode == kModeDense) {
    it.n_sink_t = 0;
    it.n_sel = 0;
    it.loc_start = 0;
    it.list_off = 0;
  } else {
    it.n_sink_t = (it.sink_end + 127) / 128;
    const int cnt = a.pair_counts[(long long)pi.pair * a.nqb + it.qb];
    it.n_sel = cnt * a.list_unit;
    it.loc_start = it.ls;
    it.list_off = (long long)pi.pair * a.pair_per_head +
                  cap_prefix(it.qb, 128, a.cap_a) / a.list_unit;
    pi.split = a.pair_split[(long long)pi.pair * a.nqb + it.qb];
    pi.a_off = ((long long)it.b * a.Hq + it.h) * a.list_per_head +
               cap_prefix(it.qb, 128, a.cap_a) / a.list_unit;
  }
  it.n_sel_t = (it.n_sel + 127) / 128;
  it.n_loc_t = (it.le - it.loc_start + 127) / 128;
  return pi;
}

// Union entry of selected ordinal n: key index and 2-bit membership tag.
// While the two heads' lists agree, the union is head A's list (both heads
// keep every entry); the plan writes union entries only from the first
// difference on.
__device__ __forceinline__ void pair_sel(const AttnArgs& a, const PairItem& pi, int n, int& key,
                                         uint32_t& tag) {
  const int ne = n / a.list_unit;
  const bool shared = ne < pi.split;
  const uint32_t* src = shared ? reinterpret_cast<const uint32_t*>(a.lists) + pi.a_off
                               : a.pair_lists + pi.it.list_off;
  const uint32_t e = src[ne] | (shared ? (3u << 30) : 0u);
  tag = e >> 30;
  const int idx = static_cast<int>(e & 0x3FFFFFFFu);
  key = a.list_unit == 1 ? idx : idx * a.list_unit + n % a.list_unit;
}

__global__ void __launch_bounds__(kPairThreads, 1)
sparse_attn_pair_kernel(const __grid_constant__ CUtensorMap tm_q,
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
  const int T = it.n_sink_t + it.n_sel_t + it.n_loc_t;
  const int kv_row0 = (it.b * a.Hkv + it.kvh) * a.L;

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
      const int ks = t % kPairKStages, vs = t % kPairVStages;
      if (t >= kPairKStages &&
          !warp_wait(bar_kempty(ks), ((t / kPairKStages) - 1) & 1, wc))
        break;
      if (t >= kPairVStages &&
          !warp_wait(bar_vempty(vs), ((t / kPairVStages) - 1) & 1, wc))
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
      if (ok && T > 0) {
        if ((ok = mbar_wait(bar_kfull(0), 0, wc))) {
          tc_fence_after();
          qk(0, 0);
          qk(0, 1);
          mma_commit(bar_kempty(0));
        }
      }
      for (int t = 0; ok && t < T; ++t) {
        const int vs = t % kPairVStages;
        const bool more = t + 1 < T;
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
    uint32_t tag_phase = 0u;                   // bit vs: phase of tag barrier vs
    bool ok = true;
    for (int t = 0; t < T; ++t) {
      if (!(ok = warp_wait(bar_sfull0 + 8u * hd, t & 1, wc))) break;
      tc_fence_after();
      const TileDesc td = tile_desc(it, t);
      const int limit = td.causal ? min(td.valid, r + 1) : td.valid;
      uint32_t tw[4] = {0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu};
      if (td.gather) {
        const int vs = t % kPairVStages;
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
    if (ok && T > 0) {
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
