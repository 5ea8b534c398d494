// spa_fp8.cu -- sparse_prefill_attn_fp8 (include/spa.h): the E4M3 attention
// kernel and its launch, in a translation unit of their own.
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/spa.h"
#include "attn_fp8.cuh"
#include "host.cuh"

namespace {
using namespace spa;
}  // namespace

extern "C" {

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
