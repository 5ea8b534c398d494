// attn_fp8.cuh -- sparse causal attention over the kept keys with E4M3
// operands on the tcgen05 kind::f8f6f4 tensor cores (SALE's Computation Pass
// on quantised operands, "SageAttention-style": the review of SALE,
// Summary).
//
// Same schedule as the bf16 one-head kernel: one CTA = one 128-row query
// block of one q head; its key tiles are the sink tiles, the selected tiles
// (gathered rows, or two tiled loads when the 128 indices are consecutive)
// and the local tiles, the last one causally masked.  What changes with
// 8-bit operands:
//   * a 128 x 128 tile is 16 KiB and one 128-byte swizzle row holds a whole
//     128-dim row, so Q, K and V each move as one TMA box (and one gather4
//     per four rows);
//   * S = Q K^T is four MMAs of K = 32; the scores are in code units and
//     carry s_q(block) * s_k(head), folded into the softmax scale;
//   * P is written to TMEM as E4M3 (four per 32-bit column) and O += P V is
//     four TS MMAs of K = 32 with V as an MN-major operand (legal for E4M3);
//   * P = 2^(x - m + 7): the running max is only raised when it grows by more
//     than 1.75 (log2 units), so P stays below 2^8.75 < 448, the E4M3 range;
//     the factor 2^7 keeps small probabilities out of the subnormal range;
//   * the epilogue multiplies channel c by the V scale s_v[c] / l, and adds
//     back to the LSE the shift scale * q^_i . mu that the K smoothing took
//     out of every score of row i (from the Q codes still in shared memory),
//     so that LSE is that of the scores against the unsmoothed keys.
//
// TMEM columns: S0 [0,128)  S1 [128,256)  O [256,384)  P0 [384,416)  P1 [416,448).
#pragma once

#include "common.cuh"
#include "fp8_cvt.cuh"
#include "ptx.cuh"
#include "tiles.cuh"

namespace spa {

constexpr uint32_t kTile8 = 128u * 128u;                 // one 128 x 128 E4M3 tile
constexpr int kF8Stages = 4;
constexpr int kF8Threads = 192;
constexpr uint32_t kF8BarBytes = 1536u;     // barriers, V scales, K mean
constexpr uint32_t kF8SmemBytes = 1024u + kTile8 + kF8Stages * 2u * kTile8 + kF8BarBytes;
static_assert(kF8SmemBytes <= 232448u, "more shared memory than a CTA may use");
constexpr uint32_t kIdescQK8 = make_idesc(1, 0, 128, 128, 0, 0);   // E4M3 x E4M3 -> f32
constexpr uint32_t kIdescPV8 = make_idesc(1, 0, 128, 128, 0, 1);   // V MN-major
constexpr float kF8PShift = 7.0f;       // P = 2^(x - m + 7)
constexpr float kF8Lazy = 1.75f;        // raise m only when the max grows by more

// D[tmem] (+)= A[smem] * B[smem]^T, E4M3 inputs, fp32 accumulation.
__device__ __forceinline__ void mma_f8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

// D[tmem] (+)= A[tmem] * B[smem], E4M3 inputs, fp32 accumulation.
__device__ __forceinline__ void mma_f8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

struct F8Args {
  TileGeom g;                 // block geometry and the plan's lists
  float sl2;                  // softmax scale * log2(e), before the quantisation scales
  float scale;                // softmax scale (natural units), for the LSE shift
  const float* qs;            // [B*Hq][nqb]
  const float* ks;            // [B*Hkv]
  const float* vs;            // [B*Hkv][128]
  const float* kmean;         // [B*Hkv][128]: the mean the K codes were smoothed by
  __nv_bfloat16* o;
  float* lse;
  uint32_t* err;
  uint64_t wait_ns;
};

__global__ void __launch_bounds__(kF8Threads, 1)
sparse_attn_fp8_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_kg,
                       const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_vg, const F8Args a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t s_base = smem_u32(smem);
  const uint32_t s_q = s_base;
  auto s_k = [&](int st) { return s_base + kTile8 + st * 2u * kTile8; };
  auto s_v = [&](int st) { return s_base + kTile8 + st * 2u * kTile8 + kTile8; };
  uint8_t* bar_area = smem + kTile8 + kF8Stages * 2 * kTile8;
  const uint32_t b0 = smem_u32(bar_area);
  const uint32_t bar_q = b0;
  auto bar_kfull = [&](int s) { return b0 + 8u * (1 + s); };
  auto bar_vfull = [&](int s) { return b0 + 8u * (1 + kF8Stages + s); };
  auto bar_empty = [&](int s) { return b0 + 8u * (1 + 2 * kF8Stages + s); };
  const uint32_t bar_sfull0 = b0 + 8u * (1 + 3 * kF8Stages);
  const uint32_t bar_sfree0 = bar_sfull0 + 16u;
  const uint32_t bar_pfull0 = bar_sfull0 + 32u;
  const uint32_t bar_pvdone0 = bar_sfull0 + 48u;
  const uint32_t bar_drain = bar_sfull0 + 64u;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bar_area + 8 * (1 + 3 * kF8Stages) + 72);
  volatile uint32_t* abort_flag = tmem_holder + 1;
  float* vscale = reinterpret_cast<float*>(bar_area + 512);      // 128 channel scales
  float* kmu = reinterpret_cast<float*>(bar_area + 1024);        // 128 K means
  static_assert(8 * (1 + 3 * kF8Stages) + 72 + 8 <= 512, "barriers overlap the V scales");
  static_assert(1024 + 128 * 4 <= kF8BarBytes, "K means overflow the barrier area");

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < kF8Stages; ++s) {
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
  const BlockTiles it = block_tiles(a.g, blockIdx.x);
  if (threadIdx.x >= 64) {
    const long long c = (long long)(it.b * a.g.Hkv + it.kvh) * 128 + threadIdx.x - 64;
    vscale[threadIdx.x - 64] = a.vs[c];
    kmu[threadIdx.x - 64] = a.kmean[c];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitCtx wc{abort_flag, a.err, a.wait_ns};

  const int T = it.n_sink_t + it.n_sel_t + it.n_loc_t;
  const int kv_row0 = (it.b * a.g.Hkv + it.kvh) * a.g.L;

  if (warp == 0) {
    // ------------------------------------------------------------- producer
    int issued = 0;
    if (lane == 0) {
      mbar_arrive_expect_tx(bar_q, kTile8);
      tma_load_2d(s_q, &tm_q, bar_q, 0, (it.b * a.g.Hq + it.h) * a.g.L + it.row0);
    }
    auto fetch = [&](int t, int (&j)[4], int& first) {
      const Tile td = tile_of(it, t);
      if (!td.gather) return;
      first = selected_key(a.g, it, td.key0);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int row = lane * 4 + r;
        j[r] = row < td.valid ? selected_key(a.g, it, td.key0 + row) : first;
      }
    };
    int nj[4] = {0, 0, 0, 0}, nfirst = 0;
    if (T > 0) fetch(0, nj, nfirst);
    for (int t = 0; t < T; ++t) {
      int j[4] = {nj[0], nj[1], nj[2], nj[3]};
      const int first = nfirst;
      if (t + 1 < T) fetch(t + 1, nj, nfirst);
      const int st = t % kF8Stages;
      if (t >= kF8Stages) {
        if (!warp_wait(bar_empty(st), ((t / kF8Stages) - 1) & 1, wc)) break;
      }
      const Tile td = tile_of(it, t);
      const uint32_t kf = bar_kfull(st), vf = bar_vfull(st);
      if (!td.gather) {
        if (lane == 0) {
          mbar_arrive_expect_tx(kf, kTile8);
          tma_load_2d(s_k(st), &tm_k, kf, 0, kv_row0 + td.key0);
          mbar_arrive_expect_tx(vf, kTile8);
          tma_load_2d(s_v(st), &tm_v, vf, 0, kv_row0 + td.key0);
        }
      } else {
        bool bad = false;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          if (j[r] < 0 || j[r] >= a.g.L) {
            bad = true;
            j[r] = 0;
          }
        }
        if (bad) atomicOr(a.err, kErrBadIndex);
        const int last = __shfl_sync(0xffffffffu, j[3], 31);
        // 128 consecutive keys: every lane's four keys are exactly the next
        // ones (a list entry out of order or repeated keeps the gather path)
        const bool contiguous = (td.valid == 128) && (last - first == 127) && first >= 0 &&
                                first < a.g.L && last < a.g.L &&
                                __all_sync(0xffffffffu, j[0] == first + 4 * lane &&
                                                            j[1] == first + 4 * lane + 1 &&
                                                            j[2] == first + 4 * lane + 2 &&
                                                            j[3] == first + 4 * lane + 3);
        if (lane == 0) {
          mbar_arrive_expect_tx(kf, kTile8);
          mbar_arrive_expect_tx(vf, kTile8);
        }
        __syncwarp();
        if (contiguous) {
          if (lane == 0) {
            tma_load_2d(s_k(st), &tm_k, kf, 0, kv_row0 + first);
            tma_load_2d(s_v(st), &tm_v, vf, 0, kv_row0 + first);
          }
        } else {
          const uint32_t roff = lane * 4u * 128u;
          tma_gather4(s_k(st) + roff, &tm_kg, kf, 0, kv_row0 + j[0], kv_row0 + j[1],
                      kv_row0 + j[2], kv_row0 + j[3]);
          tma_gather4(s_v(st) + roff, &tm_vg, vf, 0, kv_row0 + j[0], kv_row0 + j[1],
                      kv_row0 + j[2], kv_row0 + j[3]);
        }
      }
      issued = t + 1;
    }
    if (lane == 0) {
      mbar_drain(bar_q, 0, a.wait_ns);
      for (int t = max(0, issued - kF8Stages); t < issued; ++t) {
        mbar_drain(bar_kfull(t % kF8Stages), (t / kF8Stages) & 1, a.wait_ns);
        mbar_drain(bar_vfull(t % kF8Stages), (t / kF8Stages) & 1, a.wait_ns);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(bar_q, 0, wc);
      auto issue_pv = [&](int u) -> bool {
        const int bu = u & 1, st = u % kF8Stages;
        if (!mbar_wait(bar_pfull0 + 8u * bu, (u >> 1) & 1, wc)) return false;
        if (!mbar_wait(bar_vfull(st), (u / kF8Stages) & 1, wc)) return false;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          // 32 keys = 32 rows of the MN-major V tile = 4 swizzle atoms
          const uint64_t bd = smem_desc_sw128(s_v(st) + ks * 4096u, kTile8);
          mma_f8_ts(tmem + 256u, tmem + 384u + 32u * bu + 8u * ks, bd, kIdescPV8,
                    (u > 0 || ks > 0) ? 1u : 0u);
        }
        mma_commit(bar_pvdone0 + 8u * bu);
        mma_commit(bar_empty(st));
        return true;
      };
      for (int t = 0; ok && t < T; ++t) {
        const int st = t % kF8Stages, b = t & 1;
        if (!(ok = mbar_wait(bar_kfull(st), (t / kF8Stages) & 1, wc))) break;
        if (t >= 2 && !(ok = mbar_wait(bar_sfree0 + 8u * b, ((t - 2) >> 1) & 1, wc))) break;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          // 32 E4M3 elements = 32 bytes along the swizzled 128-byte row
          mma_f8_ss(tmem + 128u * b, smem_desc_sw128(s_q + ks * 32u, 16),
                    smem_desc_sw128(s_k(st) + ks * 32u, 16), kIdescQK8, ks > 0 ? 1u : 0u);
        }
        mma_commit(bar_sfull0 + 8u * b);
        if (t >= 1) ok = issue_pv(t - 1);
      }
      if (ok && T > 0) issue_pv(T - 1);
      mma_commit(bar_drain);
      mbar_drain(bar_drain, 0, a.wait_ns);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------- softmax
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const int bh = it.b * a.g.Hq + it.h;
    const float sl2 =
        a.sl2 * a.qs[(long long)bh * a.g.nqb + it.qb] * a.ks[it.b * a.g.Hkv + it.kvh];
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

      const Tile td = tile_of(it, t);
      const int limit = td.causal ? min(td.valid, r + 1) : td.valid;
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
      const bool grow = mx2 > m_used + kF8Lazy;
      if (t == 0) {
        m_used = mx2;
      } else if (__any_sync(0xffffffffu, grow)) {
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
      // p = 2^(s * scale * log2 e - m + 7) < 2^8.75; masked entries give 0
      const float shift = kF8PShift - m_used;
      uint32_t pk[32];
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
          pk[c * 8 + (e >> 2)] = e4m3x2(p0, p1) | (e4m3x2(p2, p3) << 16);
        }
      }
      lsum += ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
      if (t >= 2 && !(ok = warp_wait(bar_pvdone0 + 8u * b, ((t - 2) >> 1) & 1, wc))) break;
      tc_fence_after();
      tmem_st32(tmem + lane_off + 384u + 32u * b, pk);
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
        __nv_bfloat16* orow = a.o + (((long long)bh * a.g.L) + row) * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t ov[32];
          tmem_ld32(tmem + lane_off + 256u + 32u * c, ov);
          tmem_ld_wait();
          if (row < a.g.L) {
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
        if (ok && row < a.g.L && a.lse != nullptr) {
          // q^_r . mu from row r of the swizzled Q code tile
          float dot = 0.f;
#pragma unroll 4
          for (int c16 = 0; c16 < 8; ++c16) {
            const uint4 w = *reinterpret_cast<const uint4*>(smem + sw128_offset(r, c16 * 16));
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
          const float q_scale = a.qs[(long long)bh * a.g.nqb + it.qb];
          a.lse[(long long)bh * a.g.L + row] = (m_used - kF8PShift) * 0.69314718055994531f +
                                             logf(lsum) + a.scale * q_scale * dot;
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
