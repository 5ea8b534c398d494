// spa_attn.cu -- sparse_prefill_attn and sparse_prefill_attn_fp8
// (include/spa.h): the attention kernels and their launch, in a translation
// unit of their own.
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/spa.h"
#include "attn.cuh"
#include "attn_pair.cuh"
#include "attn_pair_fp8.cuh"
#include "attn_pair_win.cuh"
#include "host.cuh"

namespace {
using namespace spa;
}  // namespace

extern "C" {

SPA_API spa_status sparse_prefill_attn(const spa_params* p, const void* q, const void* k, const void* v,
                               void* workspace, size_t workspace_bytes, void* o, float* lse,
                               cudaStream_t stream) {
  Layout lo;
  spa_status st = common_checks(p, workspace, workspace_bytes, &lo);
  if (st != SPA_OK) return st;
  const int B = p->batch, Hq = p->heads_q, Hkv = p->heads_kv, L = p->seq_len;
  if (B == 0 || L == 0) return SPA_OK;
  if (!q || !k || !v || !o || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return SPA_ERR_INVALID;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return SPA_ERR_INVALID;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const long long BH = (long long)B * Hq, BKV = (long long)B * Hkv;
  CUtensorMap tq, tk, tkg, tv, tvg;
  if (!map_2d(&tq, kBF16, 2, q, 128, BH * L, 64, 128, kSW128) ||
      !map_2d(&tk, kBF16, 2, k, 128, BKV * L, 64, 128, kSW128) ||
      !map_2d(&tkg, kBF16, 2, k, 128, BKV * L, 64, 1, kSW128) ||
      !map_2d(&tv, kBF16, 2, v, 128, BKV * L, 64, 128, kSW128) ||
      !map_2d(&tvg, kBF16, 2, v, 128, BKV * L, 64, 1, kSW128))
    return SPA_ERR_CUDA;
  AttnArgs aa;
  aa.B = B; aa.Hq = Hq; aa.Hkv = Hkv; aa.L = L; aa.nqb = lo.nqb; aa.group = lo.group;
  aa.sink = p->sink; aa.local = p->local;
  aa.mode = p->mode == SPA_MODE_ANCHOR ? kModeAnchor : (p->mode == SPA_MODE_SALE ? kModeSale : kModeDense);
  aa.bk = p->block_k;
  aa.sl2 = eff_scale(p) * 1.4426950408889634f;
  aa.counts = reinterpret_cast<const int*>(ws + lo.counts);
  aa.lists = reinterpret_cast<const int*>(ws + lo.lists);
  aa.list_per_head = lo.list_per_head;
  aa.cap_a = lo.cap_a;
  aa.list_unit = lo.unit;
  aa.pair_counts = reinterpret_cast<const int*>(ws + lo.pair_counts);
  aa.pair_lists = reinterpret_cast<const uint32_t*>(ws + lo.pair_lists);
  aa.pair_split = reinterpret_cast<const int*>(ws + lo.pair_split);
  aa.pair_per_head = lo.list_per_head;
  aa.o = static_cast<__nv_bfloat16*>(o);
  aa.lse = lse;
  aa.err = reinterpret_cast<uint32_t*>(ws);
  aa.wait_ns = wait_ns(p);
  aa.debug = p->debug_flags;
  if (lo.paired && (p->debug_flags & SPA_DEBUG_WINDOW_TILES)) {
    if (set_smem(sparse_attn_pair_win_kernel, kPairSmemBytes) != cudaSuccess) return SPA_ERR_CUDA;
    sparse_attn_pair_win_kernel<<<(unsigned)(lo.nb / 2), kPairThreads, kPairSmemBytes, stream>>>(
        tq, tk, tkg, tv, tvg, aa);
  } else if (lo.paired) {
    if (set_smem(sparse_attn_pair_kernel, kPairSmemBytes) != cudaSuccess) return SPA_ERR_CUDA;
    sparse_attn_pair_kernel<<<(unsigned)(lo.nb / 2), kPairThreads, kPairSmemBytes, stream>>>(
        tq, tk, tkg, tv, tvg, aa);
  } else {
    if (set_smem(sparse_attn_kernel, kAttnSmemBytes) != cudaSuccess) return SPA_ERR_CUDA;
    sparse_attn_kernel<<<(unsigned)lo.nb, kAttnThreads, kAttnSmemBytes, stream>>>(tq, tk, tkg,
                                                                                 tv, tvg, aa);
  }
  if (cudaGetLastError() != cudaSuccess) return SPA_ERR_CUDA;
  return SPA_OK;
}

SPA_API spa_status sparse_prefill_attn_fp8(const spa_params* p, const void* q8, const void* k8,
                                           const void* v8, const float* scales, void* workspace,
                                           size_t workspace_bytes, void* o, float* lse,
                                           cudaStream_t stream) {
  Layout lo;
  spa_status st = common_checks(p, workspace, workspace_bytes, &lo);
  if (st != SPA_OK) return st;
  const int B = p->batch, Hq = p->heads_q, Hkv = p->heads_kv, L = p->seq_len;
  if (B == 0 || L == 0) return SPA_OK;
  if (!q8 || !k8 || !v8 || !scales || !o || !aligned16(q8) || !aligned16(k8) || !aligned16(v8) ||
      !aligned16(o) || (reinterpret_cast<uintptr_t>(scales) & 3u))
    return SPA_ERR_INVALID;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return SPA_ERR_INVALID;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const long long BH = (long long)B * Hq, BKV = (long long)B * Hkv;
  CUtensorMap tq, tk, tkg, tv, tvg;
  if (!map_2d(&tq, kI8, 1, q8, 128, BH * L, 128, 128, kSW128) ||
      !map_2d(&tk, kI8, 1, k8, 128, BKV * L, 128, 128, kSW128) ||
      !map_2d(&tkg, kI8, 1, k8, 128, BKV * L, 128, 1, kSW128) ||
      !map_2d(&tv, kI8, 1, v8, 128, BKV * L, 128, 128, kSW128) ||
      !map_2d(&tvg, kI8, 1, v8, 128, BKV * L, 128, 1, kSW128))
    return SPA_ERR_CUDA;
  // scales: qs [B*Hq*nqb], ks [B*Hkv], vs [B*Hkv*128], K mean [B*Hkv*128]
  const long long n_qs = BH * lo.nqb;
  F8Args a;
  a.g = tile_geom(p, lo, ws);
  a.scale = eff_scale(p);
  a.sl2 = a.scale * 1.4426950408889634f;
  a.qs = scales;
  a.ks = scales + n_qs;
  a.vs = scales + n_qs + BKV;
  a.kmean = scales + n_qs + BKV + BKV * 128;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.err = reinterpret_cast<uint32_t*>(ws);
  a.wait_ns = wait_ns(p);
  if (lo.paired && p->mode != SPA_MODE_DENSE) {
    // two q heads per CTA over the pair's union lists
    PairF8Args pa;
    pa.base.B = B; pa.base.Hq = Hq; pa.base.Hkv = Hkv; pa.base.L = L; pa.base.nqb = lo.nqb;
    pa.base.group = lo.group; pa.base.sink = p->sink; pa.base.local = p->local;
    pa.base.mode = a.g.mode; pa.base.bk = p->block_k;
    pa.base.sl2 = a.sl2;
    pa.base.counts = a.g.counts; pa.base.lists = a.g.lists;
    pa.base.list_per_head = lo.list_per_head; pa.base.cap_a = lo.cap_a;
    pa.base.list_unit = lo.unit;
    pa.base.pair_counts = reinterpret_cast<const int*>(ws + lo.pair_counts);
    pa.base.pair_lists = reinterpret_cast<const uint32_t*>(ws + lo.pair_lists);
    pa.base.pair_split = reinterpret_cast<const int*>(ws + lo.pair_split);
    pa.base.pair_per_head = lo.list_per_head;
    pa.base.o = a.o; pa.base.lse = lse; pa.base.err = a.err; pa.base.wait_ns = a.wait_ns;
    pa.base.debug = 0;
    pa.qs = a.qs; pa.ks = a.ks; pa.vs = a.vs; pa.kmean = a.kmean; pa.scale = a.scale;
    if (set_smem(sparse_attn_pair_fp8_kernel, kPF8SmemBytes) != cudaSuccess) return SPA_ERR_CUDA;
    sparse_attn_pair_fp8_kernel<<<(unsigned)(lo.nb / 2), kPairThreads, kPF8SmemBytes, stream>>>(
        tq, tk, tkg, tv, tvg, pa);
  } else {
    if (set_smem(sparse_attn_fp8_kernel, kF8SmemBytes) != cudaSuccess) return SPA_ERR_CUDA;
    sparse_attn_fp8_kernel<<<(unsigned)lo.nb, kF8Threads, kF8SmemBytes, stream>>>(tq, tk, tkg,
                                                                                 tv, tvg, a);
  }
  if (cudaGetLastError() != cudaSuccess) return SPA_ERR_CUDA;
  return SPA_OK;
}

}  // extern "C"
