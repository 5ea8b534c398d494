// decode.cuh -- decode-shaped reuse of a finished prefill plan.
//
// SpotAttention (Fig. 2 and Sec. 3) gives a decoding query a key set made of
// a sink prefix, a recency window and a set of selected blocks.  Here the
// selected part is the prefill plan's selection for the last prompt query
// block qb = (L - 1) / 128, so a query at absolute position pos >= L - 1
// attends to
//
//     D_h(pos) = [0, min(sink, pos + 1)) u sel_h(qb) u [max(ls_qb, sink'), pos]
//
// (ls_qb the local-window start of that block); at pos = L - 1 this is the
// prefill key set of the last prompt row.
//
// The q heads of one kv head select different keys, but they read the same
// K/V rows.  decode_union_kernel (once per plan) merges the selections of a
// group of up to eight q heads into one ascending list whose entries carry a
// byte of head bits; decode_attn_kernel (every step) walks sink + union +
// window once per group, loads each K/V row once for all the group's heads,
// and masks the scores of heads whose set does not hold the key.  The step is
// bound by HBM (512 bytes of K and V per key for up to eight q heads), so it
// runs on the CUDA cores, split over the key set with one fp32 partial
// (m, l, acc) per CTA and head that decode_combine_kernel merges.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "common.cuh"
#include "ptx.cuh"

namespace spa {

constexpr int kDecWarps = 4;
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kDecTileKeys = 16;                        // keys per warp per pipeline stage
constexpr int kDecStages = 3;
constexpr uint32_t kDecRowBytes = 256;                  // one 128-dim bf16 row
constexpr uint32_t kDecStageBytes = 2u * kDecTileKeys * kDecRowBytes;      // K + V
constexpr uint32_t kDecWarpBytes = kDecStages * kDecStageBytes;
constexpr uint32_t kDecRingBytes = kDecWarps * kDecWarpBytes;              // 96 KiB
constexpr int kDecQPad = 68;                            // floats per half row of q (64 + pad)
constexpr uint32_t kDecQBytes = 8u * 2u * kDecQPad * 4u;                   // up to 8 heads
constexpr uint32_t kDecPBytes = kDecWarps * kDecTileKeys * 8u * 4u;
constexpr uint32_t kDecMetaBytes = 2u * kDecWarps * 8u * 4u;               // m, l per warp
constexpr uint32_t kDecSmemBytes = kDecRingBytes + kDecQBytes + kDecPBytes + kDecMetaBytes;
static_assert(kDecWarps * 8u * 128u * 4u <= kDecRingBytes, "merge area fits in the ring");
static_assert(kDecSmemBytes <= 227u * 1024u, "decode smem");
constexpr int kDecPartFloats = 132;                     // acc[128], m, l, pad
constexpr int kDecUnionThreads = 1024;
constexpr uint32_t kDecKeyBits = 24;                    // union entry: unit index | heads << 24
constexpr uint32_t kDecKeyMask = (1u << kDecKeyBits) - 1u;

struct DecodeArgs {
  const __nv_bfloat16* q;     // [B, Hq, 128]
  const __nv_bfloat16* k;     // [B, Hkv, cap, 128]
  const __nv_bfloat16* v;
  const int* counts;          // plan counts (b, h, qb)
  const int* lists;           // plan lists
  long long list_per_head;    // list elements per (b, h)
  long long list_qb_off;      // P(qb) in list units: offset of the last block's list
  int B, Hq, Hkv, nqb, qb;    // qb = last prompt query block
  int group, hsub, gh;        // q heads per kv head, subgroups, heads per subgroup
  int cap;                    // kv cache capacity (rows per (b, kv head))
  int pos;                    // absolute position of the decoding query
  int sink, ls, mode, uk;     // uk: keys per list unit (1, or block_k in SALE mode)
  int cand_lo, cand_units;    // candidate range of block qb in list units
  int chunks;                 // CTAs per unit along the key set
  long long union_stride;     // union entries per unit (>= cand_units, multiple of 4)
  float sl2;                  // softmax scale * log2(e)
  const int* union_count;     // [units]
  const uint32_t* union_list; // [units][union_stride]
  float* part;                // [units][chunks][gh][kDecPartFloats]
  __nv_bfloat16* o;           // [B, Hq, 128]
  float* lse;                 // [B, Hq] or null
  uint32_t* err;
};

struct DecodeUnionArgs {
  const int* counts;
  const int* lists;
  long long list_per_head, list_qb_off, union_stride;
  int Hq, Hkv, nqb, qb, group, hsub, gh;
  int cand_lo, cand_units;
  int* union_count;
  uint32_t* union_list;
  uint32_t* tags;             // [units][union_stride / 4] scratch words
  uint32_t* err;
};

// ---------------------------------------------------------------------------
// Once per plan: the tagged union of the selections of a group of q heads.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int block_exclusive_scan(int x, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_sums[w] = incl;
  __syncthreads();
  if (w == 0) {
    const int nw = blockDim.x >> 5;
    int s = lane < nw ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < nw) warp_sums[lane] = s - (lane < nw ? warp_sums[lane] : 0);
    if (lane == nw - 1) *total = s;
  }
  __syncthreads();
  return warp_sums[w] + incl - x;
}

__global__ void __launch_bounds__(kDecUnionThreads) decode_union_kernel(DecodeUnionArgs a) {
  __shared__ int warp_sums[32];
  __shared__ int total;
  const int u = blockIdx.x;
  const int hs = u % a.hsub, bg = u / a.hsub;
  const int b = bg / a.Hkv, g = bg % a.Hkv;
  const long long words = (a.cand_units + 3) / 4;
  uint32_t* tw = a.tags + (long long)u * (a.union_stride / 4);
  for (long long w = threadIdx.x; w < words; w += blockDim.x) tw[w] = 0u;
  __syncthreads();
  for (int j = 0; j < a.gh; ++j) {
    const int h = g * a.group + hs * a.gh + j;
    const long long bh = (long long)b * a.Hq + h;
    int n = a.counts[bh * a.nqb + a.qb];
    if (n < 0 || n > a.cand_units) {
      if (threadIdx.x == 0) atomicOr(a.err, kErrBadIndex);
      n = n < 0 ? 0 : a.cand_units;
    }
    const int* lst = a.lists + bh * a.list_per_head + a.list_qb_off;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      const int idx = lst[i] - a.cand_lo;
      if (idx < 0 || idx >= a.cand_units) {
        atomicOr(a.err, kErrBadIndex);
        continue;
      }
      atomicOr(&tw[idx >> 2], (1u << j) << (8 * (idx & 3)));
    }
  }
  __syncthreads();
  uint32_t* out = a.union_list + (long long)u * a.union_stride;
  int running = 0;
  for (long long base = 0; base < words; base += blockDim.x) {
    const long long w = base + threadIdx.x;
    const uint32_t t = w < words ? tw[w] : 0u;
    int nz = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) nz += ((t >> (8 * i)) & 0xffu) != 0u;
    const int off = block_exclusive_scan(nz, warp_sums, &total);
    int at = running + off;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t tag = (t >> (8 * i)) & 0xffu;
      if (tag) out[at++] = (uint32_t)(a.cand_lo + 4 * w + i) | (tag << kDecKeyBits);
    }
    running += total;
    __syncthreads();                       // warp_sums / total reused next batch
  }
  if (threadIdx.x == 0) a.union_count[u] = running;
}

// ---------------------------------------------------------------------------
// Every step: split attention of one query per head over sink + union + window.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Position n of the unit's key set -> (key, head bits).  The set is the sink,
// then the union entries (each uk keys), then the window up to pos.
struct KeySet {
  int s1;          // sink keys present: min(sink, pos + 1)
  long long nsel;  // union keys: count * uk
  int lo_local;    // first window key
  const uint32_t* ul;
  int uk;
  uint32_t all;
  __device__ __forceinline__ void at(long long n, int& key, uint32_t& tag) const {
    if (n < s1) {
      key = (int)n;
      tag = all;
    } else if (n < s1 + nsel) {
      const long long m = n - s1;
      const uint32_t e = ul[m / uk];
      key = (int)(e & kDecKeyMask) * uk + (int)(m % uk);
      tag = e >> kDecKeyBits;
    } else {
      key = lo_local + (int)(n - s1 - nsel);
      tag = all;
    }
  }
};

template <int GH>
__global__ void __launch_bounds__(kDecThreads) decode_attn_kernel(DecodeArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  float* q_s = reinterpret_cast<float*>(smem + kDecRingBytes);
  float* p_s = reinterpret_cast<float*>(smem + kDecRingBytes + kDecQBytes);
  float* m_s = reinterpret_cast<float*>(smem + kDecRingBytes + kDecQBytes + kDecPBytes);
  float* l_s = m_s + kDecWarps * 8;

  const int u = blockIdx.x, c = blockIdx.y;
  const int hs = u % a.hsub, bg = u / a.hsub;
  const int b = bg / a.Hkv, g = bg % a.Hkv;
  const int h0 = g * a.group + hs * GH;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // the unit's key set
  KeySet ks;
  ks.uk = a.uk;
  ks.all = (1u << GH) - 1u;
  if (a.mode == kModeDense) {
    ks.s1 = 0;
    ks.nsel = 0;
    ks.lo_local = 0;
  } else {
    ks.s1 = a.sink < a.pos + 1 ? a.sink : a.pos + 1;
    int nu = a.union_count[u];
    if (nu < 0 || nu > a.cand_units) nu = 0;     // the union kernel wrote it; never expected
    ks.nsel = (long long)nu * a.uk;
    ks.lo_local = a.ls > ks.s1 ? a.ls : ks.s1;
  }
  ks.ul = a.union_list + (long long)u * a.union_stride;
  const long long N = ks.s1 + ks.nsel + (a.pos + 1 - ks.lo_local);
  const long long c0 = N * c / a.chunks, c1 = N * (c + 1) / a.chunks;
  const long long w0 = c0 + (c1 - c0) * warp / kDecWarps;
  const long long w1 = c0 + (c1 - c0) * (warp + 1) / kDecWarps;
  const int ntiles = (int)((w1 - w0 + kDecTileKeys - 1) / kDecTileKeys);

  // q of the GH heads, fp32, pre-scaled to log2 units; half rows padded
  for (int i = threadIdx.x; i < GH * 128; i += kDecThreads) {
    const int j = i >> 7, d = i & 127;
    const float x = __bfloat162float(a.q[((long long)b * a.Hq + h0 + j) * 128 + d]);
    q_s[(j * 2 + (d >> 6)) * kDecQPad + (d & 63)] = x * a.sl2;
  }
  __syncthreads();

  const long long kv_base = ((long long)b * a.Hkv + g) * (long long)a.cap;
  const uint32_t ring = smem_u32(smem) + warp * kDecWarpBytes;
  float* pw = p_s + warp * kDecTileKeys * 8;

  // issue the copies of tile t into stage t % kDecStages
  auto issue = [&](int t) {
    const long long n = w0 + (long long)t * kDecTileKeys + (lane & 15);
    int key = 0;
    uint32_t tag = 0;
    if (n < w1) ks.at(n, key, tag);
    if (key < 0 || key > a.pos) {
      atomicOr(a.err, kErrBadIndex);
      key = 0;
    }
    const uint32_t st = ring + (uint32_t)(t % kDecStages) * kDecStageBytes;
    const int cc = lane & 15;
#pragma unroll
    for (int i = 0; i < kDecTileKeys / 2; ++i) {
      const int r = (lane >> 4) + 2 * i;
      const int kr = __shfl_sync(0xffffffffu, key, r);
      const long long row = (kv_base + kr) * 128 + cc * 8;
      const uint32_t off = (uint32_t)r * kDecRowBytes + (uint32_t)((cc ^ r) * 16);
      cp_async16(st + off, a.k + row);
      cp_async16(st + kDecTileKeys * kDecRowBytes + off, a.v + row);
    }
  };

  float m[GH], lrow[GH], acc[GH][4];
#pragma unroll
  for (int j = 0; j < GH; ++j) {
    m[j] = -INFINITY;
    lrow[j] = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[j][e] = 0.f;
  }

#pragma unroll
  for (int t = 0; t < kDecStages - 1; ++t) {
    if (t < ntiles) issue(t);
    cp_async_commit();
  }
  const int kk = lane >> 1, hh = lane & 1;
  for (int t = 0; t < ntiles; ++t) {
    if (t + kDecStages - 1 < ntiles) issue(t + kDecStages - 1);
    cp_async_commit();
    cp_async_wait<kDecStages - 1>();
    __syncwarp();
    const uint8_t* st = smem + warp * kDecWarpBytes + (t % kDecStages) * kDecStageBytes;

    // this thread's key of the tile and its head bits
    const long long n_me = w0 + (long long)t * kDecTileKeys + (lane & 15);
    int key_me = 0;
    uint32_t tag_me = 0;
    if (n_me < w1) ks.at(n_me, key_me, tag_me);
    const uint32_t tag = __shfl_sync(0xffffffffu, tag_me, kk);   // lane kk holds key kk

    // scores: thread (kk, hh) covers dims [64 hh, 64 hh + 64) of key kk
    float s[GH];
#pragma unroll
    for (int j = 0; j < GH; ++j) s[j] = 0.f;
    const uint8_t* krow = st + kk * kDecRowBytes;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int cch = hh * 8 + i;
      const uint4 kv = *reinterpret_cast<const uint4*>(krow + ((cch ^ kk) * 16));
      const float k0 = bf16lo(kv.x), k1 = bf16hi(kv.x), k2 = bf16lo(kv.y), k3 = bf16hi(kv.y);
      const float k4 = bf16lo(kv.z), k5 = bf16hi(kv.z), k6 = bf16lo(kv.w), k7 = bf16hi(kv.w);
#pragma unroll
      for (int j = 0; j < GH; ++j) {
        const float* qp = q_s + (j * 2 + hh) * kDecQPad + i * 8;
        const float4 qa = *reinterpret_cast<const float4*>(qp);
        const float4 qb = *reinterpret_cast<const float4*>(qp + 4);
        float x = s[j];
        x = fmaf(qa.x, k0, x); x = fmaf(qa.y, k1, x); x = fmaf(qa.z, k2, x); x = fmaf(qa.w, k3, x);
        x = fmaf(qb.x, k4, x); x = fmaf(qb.y, k5, x); x = fmaf(qb.z, k6, x); x = fmaf(qb.w, k7, x);
        s[j] = x;
      }
    }
    float alpha[GH];
#pragma unroll
    for (int j = 0; j < GH; ++j) {
      float x = s[j] + __shfl_xor_sync(0xffffffffu, s[j], 1);
      if (!((tag >> j) & 1u)) x = -INFINITY;     // key not in head j's set (or past the slice)
      float tmax = x;
#pragma unroll
      for (int o = 2; o < 32; o <<= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
      const float mn = fmaxf(m[j], tmax);
      float p;
      if (mn == -INFINITY) {
        alpha[j] = 1.f;
        p = 0.f;
      } else {
        alpha[j] = exp2f(m[j] - mn);
        p = exp2f(x - mn);
      }
      m[j] = mn;
      lrow[j] = lrow[j] * alpha[j] + p;
      if (hh == 0) pw[kk * 8 + j] = p;
    }
    __syncwarp();

    // acc[j][dims 4 lane .. 4 lane + 3] += p[key][j] * V[key]
    const uint8_t* vt = st + kDecTileKeys * kDecRowBytes;
    const int vc = lane >> 1;
#pragma unroll
    for (int j = 0; j < GH; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[j][e] *= alpha[j];
#pragma unroll 4
    for (int r = 0; r < kDecTileKeys; ++r) {
      const uint2 vv =
          *reinterpret_cast<const uint2*>(vt + r * kDecRowBytes + ((vc ^ r) * 16) + (lane & 1) * 8);
      const float v0 = bf16lo(vv.x), v1 = bf16hi(vv.x), v2 = bf16lo(vv.y), v3 = bf16hi(vv.y);
#pragma unroll
      for (int j = 0; j < GH; ++j) {
        const float p = pw[r * 8 + j];
        acc[j][0] = fmaf(p, v0, acc[j][0]);
        acc[j][1] = fmaf(p, v1, acc[j][1]);
        acc[j][2] = fmaf(p, v2, acc[j][2]);
        acc[j][3] = fmaf(p, v3, acc[j][3]);
      }
    }
    __syncwarp();                          // the stage and pw are rewritten next
  }
  cp_async_wait<0>();

  // row sums over the warp's 16 key slots (each slot is held by two lanes)
#pragma unroll
  for (int j = 0; j < GH; ++j) {
    float x = lrow[j];
#pragma unroll
    for (int o = 2; o < 32; o <<= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    lrow[j] = x;
  }
  __syncthreads();                         // every warp is done with its ring
  float* acc_s = reinterpret_cast<float*>(smem);     // [warp][GH][128]
#pragma unroll
  for (int j = 0; j < GH; ++j) {
    *reinterpret_cast<float4*>(acc_s + (warp * GH + j) * 128 + 4 * lane) =
        make_float4(acc[j][0], acc[j][1], acc[j][2], acc[j][3]);
    if (lane == 0) {
      m_s[warp * 8 + j] = m[j];
      l_s[warp * 8 + j] = lrow[j];
    }
  }
  __syncthreads();
  const int d = threadIdx.x;
#pragma unroll
  for (int j = 0; j < GH; ++j) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, m_s[w * 8 + j]);
    float Ls = 0.f, A = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kDecWarps; ++w) {
        const float f = exp2f(m_s[w * 8 + j] - M);
        Ls += l_s[w * 8 + j] * f;
        A += acc_s[(w * GH + j) * 128 + d] * f;
      }
    }
    float* part = a.part + (((long long)u * a.chunks + c) * GH + j) * kDecPartFloats;
    part[d] = A;
    if (d == 0) {
      part[128] = M;
      part[129] = Ls;
    }
  }
}

// Merge the per-CTA partials of one (b, q head): O = sum_c 2^(m_c - M) acc_c /
// sum_c 2^(m_c - M) l_c, LSE = ln 2 * (M + log2 l).
__global__ void __launch_bounds__(128) decode_combine_kernel(DecodeArgs a) {
  const int bh = blockIdx.x;
  const int b = bh / a.Hq, h = bh % a.Hq;
  const int g = h / a.group, hs = (h % a.group) / a.gh, j = (h % a.group) % a.gh;
  const int u = (b * a.Hkv + g) * a.hsub + hs;
  const int d = threadIdx.x;
  float m = -INFINITY, l = 0.f, acc = 0.f;
  for (int c = 0; c < a.chunks; ++c) {
    const float* part = a.part + (((long long)u * a.chunks + c) * a.gh + j) * kDecPartFloats;
    const float mc = part[128];
    if (mc == -INFINITY) continue;
    const float mn = fmaxf(m, mc);
    const float fo = exp2f(m - mn), fn = exp2f(mc - mn);
    l = l * fo + part[129] * fn;
    acc = acc * fo + part[d] * fn;
    m = mn;
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
  a.o[(long long)bh * 128 + d] = __float2bfloat16(acc * inv);
  if (a.lse && d == 0) a.lse[bh] = (m + log2f(l)) * 0.6931471805599453f;
}

}  // namespace spa
