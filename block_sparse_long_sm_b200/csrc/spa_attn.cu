// spa_attn.cu -- sparse_prefill_attn and sparse_prefill_attn_fp8
// (include/spa.h): the attention kernels and their launch, in a translation
// unit of their own.
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/spa.h"
#include "attn.cuh"
#include "attn_pair.cuh"
#include "attn_fp8.cuh"
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
  CUtensorMap tq, tk, tkg, tv, tvg, tk16, tv16;
  if (!map_2d(&tq, kBF16, 2, q, 128, BH * L, 64, 128, kSW128) ||
      !map_2d(&tk, kBF16, 2, k, 128, BKV * L, 64, 128, kSW128) ||
      !map_2d(&tkg, kBF16, 2, k, 128, BKV * L, 64, 1, kSW128) ||
      !map_2d(&tv, kBF16, 2, v, 128, BKV * L, 64, 128, kSW128) ||
      !map_2d(&tvg, kBF16, 2, v, 128, BKV * L, 64, 1, kSW128) ||
      !map_2d(&tk16, kBF16, 2, k, 128, BKV * L, 64, 16, kSW128) ||
      !map_2d(&tv16, kBF16, 2, v, 128, BKV * L, 64, 16, kSW128))
    return SPA_ERR_CUDA;
  AttnArgs aa{};
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
  aa.tmask = reinterpret_cast<const uint4*>(ws + lo.tmask);
  aa.tmask_per_head = lo.tmask_per_head;
  aa.tc = lo.tc;
  aa.tbits = reinterpret_cast<const uint32_t*>(ws + lo.tbits);
  aa.tbit_words = lo.tbit_words;
  aa.k = static_cast<const __nv_bfloat16*>(k);
  aa.v = static_cast<const __nv_bfloat16*>(v);
  aa.o = static_cast<__nv_bfloat16*>(o);
  aa.lse = lse;
  aa.err = reinterpret_cast<uint32_t*>(ws);
  aa.wait_ns = wait_ns(p);
  aa.debug = p->debug_flags;
  if (lo.paired) {
    if (set_smem(sparse_attn_pair_kernel, kPairSmemBytes) != cudaSuccess) return SPA_ERR_CUDA;
    sparse_attn_pair_kernel<<<(unsigned)(lo.nb / 2), kPairThreads, kPairSmemBytes, stream>>>(
        tq, tk, tkg, tv, tvg, tk16, tv16, aa);
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
  if (set_smem(sparse_attn_fp8_kernel, kF8SmemBytes) != cudaSuccess) return SPA_ERR_CUDA;
  sparse_attn_fp8_kernel<<<(unsigned)lo.nb, kF8Threads, kF8SmemBytes, stream>>>(tq, tk, tkg, tv,
                                                                               tvg, a);
  if (cudaGetLastError() != cudaSuccess) return SPA_ERR_CUDA;
  return SPA_OK;
}

}  // extern "C"
