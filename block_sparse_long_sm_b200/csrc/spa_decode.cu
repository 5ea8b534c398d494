// spa_decode.cu -- sparse_decode_scratch_bytes / sparse_decode_prepare /
// sparse_decode_attn (include/spa.h): decode-shaped reuse of a prefill plan
// (SpotAttention, Fig. 2 and Sec. 3: sink prefix + recency window + selected
// blocks).  Nothing here allocates device memory.
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/spa.h"
#include "decode.cuh"
#include "host.cuh"

namespace {

using namespace spa;

// CTAs one decode step aims at: four waves of two CTAs per SM on 148 SMs, so
// that the tail of the last wave is at most a quarter of the step.
constexpr long long kDecTargetCtas = 148LL * 2 * 4;
constexpr int kDecMinKeysPerCta = 64;
constexpr int kDecMaxCapacity = 1 << 24;        // union entries keep 24 bits of index

struct DecodeLayout {
  int qb = 0, ls = 0, uk = 1, cand_lo = 0, cand_units = 0;
  int group = 1, gh = 1, hsub = 1;
  long long units = 0, list_qb_off = 0, union_stride = 0;
  int max_chunks = 1;
  size_t union_count = 0, union_list = 0, tags = 0, part = 0, total = 0;
};

int heads_per_cta(int group) {
  for (int d = 8; d > 1; --d)
    if (group % d == 0) return d;
  return 1;
}

int chunks_for(long long units, long long keys_bound) {
  long long c = (kDecTargetCtas + units - 1) / units;
  const long long by_keys = (keys_bound + kDecMinKeysPerCta - 1) / kDecMinKeysPerCta;
  if (c > by_keys) c = by_keys;
  if (c < 1) c = 1;
  if (c > 65535) c = 65535;
  return (int)c;
}

// Scratch layout (byte offsets, each region 256-aligned): 256 reserved bytes
// (so that every valid parameter set has a non-zero size); union counts
// int32[units]; union lists uint32[units][union_stride]; tag words
// uint32[units][union_stride / 4]; partials float[units][max_chunks][gh][132].
DecodeLayout decode_layout(const spa_params* p, int kv_capacity) {
  DecodeLayout d;
  const int L = p->seq_len;
  d.qb = L > 0 ? (L - 1) / 128 : 0;
  const int lse_ = (d.qb + 1) * 128 - p->local;
  d.ls = lse_ > 0 ? lse_ : 0;
  d.uk = p->mode == SPA_MODE_SALE ? p->block_k : 1;
  if (p->mode != SPA_MODE_DENSE && d.ls > p->sink) {
    d.cand_lo = p->sink / d.uk;
    d.cand_units = (d.ls - p->sink) / d.uk;
  }
  d.group = p->heads_q / p->heads_kv;
  d.gh = heads_per_cta(d.group);
  d.hsub = d.group / d.gh;
  d.units = (long long)p->batch * p->heads_kv * d.hsub;
  d.list_qb_off = cap_prefix(d.qb, 128, (long long)p->local + p->sink) / d.uk;
  d.union_stride = ((long long)d.cand_units + 3) / 4 * 4;
  d.max_chunks = chunks_for(d.units > 0 ? d.units : 1, kv_capacity);
  size_t off = kHeaderBytes;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes);
    return at;
  };
  d.union_count = take((size_t)d.units * 4);
  d.union_list = take((size_t)d.units * d.union_stride * 4);
  d.tags = take((size_t)d.units * (d.union_stride / 4) * 4);
  d.part = take((size_t)d.units * d.max_chunks * d.gh * kDecPartFloats * 4);
  d.total = off;
  return d;
}

spa_status decode_checks(const spa_params* p, int kv_capacity, const void* workspace,
                         size_t ws_bytes, const void* scratch, size_t scratch_bytes, Layout* lo,
                         DecodeLayout* dl) {
  spa_status st = common_checks(p, workspace, ws_bytes, lo);
  if (st != SPA_OK) return st;
  if (p->seq_len < 1) return SPA_ERR_INVALID;
  if (kv_capacity < p->seq_len) return SPA_ERR_INVALID;
  if (kv_capacity > kDecMaxCapacity) return SPA_ERR_UNSUPPORTED;
  *dl = decode_layout(p, kv_capacity);
  if (!scratch || !aligned16(scratch)) return SPA_ERR_INVALID;
  if (scratch_bytes < dl->total) return SPA_ERR_WORKSPACE;
  return SPA_OK;
}

template <int GH>
cudaError_t launch_decode(const DecodeArgs& a, dim3 grid, cudaStream_t stream) {
  cudaError_t e = set_smem(decode_attn_kernel<GH>, kDecSmemBytes);
  if (e != cudaSuccess) return e;
  decode_attn_kernel<GH><<<grid, kDecThreads, kDecSmemBytes, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

extern "C" {

SPA_API size_t sparse_decode_scratch_bytes(const spa_params* p, int32_t kv_capacity) {
  if (validate(p) != SPA_OK || p->seq_len < 1 || kv_capacity < p->seq_len ||
      kv_capacity > kDecMaxCapacity)
    return 0;
  return decode_layout(p, kv_capacity).total;
}

SPA_API spa_status sparse_decode_prepare(const spa_params* p, int32_t kv_capacity,
                                         void* workspace, size_t workspace_bytes, void* scratch,
                                         size_t scratch_bytes, cudaStream_t stream) {
  Layout lo;
  DecodeLayout dl;
  spa_status st =
      decode_checks(p, kv_capacity, workspace, workspace_bytes, scratch, scratch_bytes, &lo, &dl);
  if (st != SPA_OK) return st;
  if (dl.units == 0) return SPA_OK;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* sc = static_cast<uint8_t*>(scratch);
  if (p->mode == SPA_MODE_DENSE || dl.cand_units == 0) {
    if (cudaMemsetAsync(sc + dl.union_count, 0, (size_t)dl.units * 4, stream) != cudaSuccess)
      return SPA_ERR_CUDA;
    return SPA_OK;
  }
  DecodeUnionArgs a;
  a.counts = reinterpret_cast<const int*>(ws + lo.counts);
  a.lists = reinterpret_cast<const int*>(ws + lo.lists);
  a.list_per_head = lo.list_per_head;
  a.list_qb_off = dl.list_qb_off;
  a.union_stride = dl.union_stride;
  a.Hq = p->heads_q; a.Hkv = p->heads_kv; a.nqb = lo.nqb; a.qb = dl.qb;
  a.group = dl.group; a.hsub = dl.hsub; a.gh = dl.gh;
  a.cand_lo = dl.cand_lo; a.cand_units = dl.cand_units;
  a.union_count = reinterpret_cast<int*>(sc + dl.union_count);
  a.union_list = reinterpret_cast<uint32_t*>(sc + dl.union_list);
  a.tags = reinterpret_cast<uint32_t*>(sc + dl.tags);
  a.err = reinterpret_cast<uint32_t*>(ws);
  decode_union_kernel<<<(unsigned)dl.units, kDecUnionThreads, 0, stream>>>(a);
  if (cudaGetLastError() != cudaSuccess) return SPA_ERR_CUDA;
  return SPA_OK;
}

SPA_API spa_status sparse_decode_attn(const spa_params* p, const void* q, const void* k_cache,
                                      const void* v_cache, int32_t kv_capacity, int32_t pos,
                                      void* workspace, size_t workspace_bytes, void* scratch,
                                      size_t scratch_bytes, void* o, float* lse,
                                      cudaStream_t stream) {
  Layout lo;
  DecodeLayout dl;
  spa_status st =
      decode_checks(p, kv_capacity, workspace, workspace_bytes, scratch, scratch_bytes, &lo, &dl);
  if (st != SPA_OK) return st;
  if (pos < p->seq_len - 1 || pos >= kv_capacity) return SPA_ERR_INVALID;
  if (dl.units == 0) return SPA_OK;
  if (!q || !k_cache || !v_cache || !o || !aligned16(q) || !aligned16(k_cache) ||
      !aligned16(v_cache) || !aligned16(o))
    return SPA_ERR_INVALID;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return SPA_ERR_INVALID;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* sc = static_cast<uint8_t*>(scratch);
  DecodeArgs a;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k = static_cast<const __nv_bfloat16*>(k_cache);
  a.v = static_cast<const __nv_bfloat16*>(v_cache);
  a.counts = reinterpret_cast<const int*>(ws + lo.counts);
  a.lists = reinterpret_cast<const int*>(ws + lo.lists);
  a.list_per_head = lo.list_per_head;
  a.list_qb_off = dl.list_qb_off;
  a.B = p->batch; a.Hq = p->heads_q; a.Hkv = p->heads_kv; a.nqb = lo.nqb; a.qb = dl.qb;
  a.group = dl.group; a.hsub = dl.hsub; a.gh = dl.gh;
  a.cap = kv_capacity;
  a.pos = pos;
  a.sink = p->sink;
  a.ls = dl.ls;
  a.mode = p->mode == SPA_MODE_ANCHOR ? kModeAnchor : (p->mode == SPA_MODE_SALE ? kModeSale : kModeDense);
  a.uk = dl.uk;
  a.cand_lo = dl.cand_lo;
  a.cand_units = dl.cand_units;
  a.chunks = chunks_for(dl.units, (long long)pos + 1);
  a.union_stride = dl.union_stride;
  a.sl2 = eff_scale(p) * 1.4426950408889634f;
  a.union_count = reinterpret_cast<const int*>(sc + dl.union_count);
  a.union_list = reinterpret_cast<const uint32_t*>(sc + dl.union_list);
  a.part = reinterpret_cast<float*>(sc + dl.part);
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.err = reinterpret_cast<uint32_t*>(ws);
  const dim3 grid((unsigned)dl.units, (unsigned)a.chunks);
  cudaError_t e;
  switch (dl.gh) {
    case 1: e = launch_decode<1>(a, grid, stream); break;
    case 2: e = launch_decode<2>(a, grid, stream); break;
    case 3: e = launch_decode<3>(a, grid, stream); break;
    case 4: e = launch_decode<4>(a, grid, stream); break;
    case 5: e = launch_decode<5>(a, grid, stream); break;
    case 6: e = launch_decode<6>(a, grid, stream); break;
    case 7: e = launch_decode<7>(a, grid, stream); break;
    default: e = launch_decode<8>(a, grid, stream); break;
  }
  if (e != cudaSuccess) return SPA_ERR_CUDA;
  decode_combine_kernel<<<(unsigned)((long long)p->batch * p->heads_q), 128, 0, stream>>>(a);
  if (cudaGetLastError() != cudaSuccess) return SPA_ERR_CUDA;
  return SPA_OK;
}

}  // extern "C"
