// spa_mass.cu -- sparse_key_mass (include/spa.h): attention mass per key from
// the prefill rows, reusing the prefill LSE (KVpop, Sec. 3).
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/spa.h"
#include "host.cuh"
#include "key_mass.cuh"

namespace {
using namespace spa;
}  // namespace

extern "C" {

SPA_API spa_status sparse_key_mass(const spa_params* p, const void* q, const void* k,
                                   const float* lse, int32_t window, void* workspace,
                                   size_t workspace_bytes, float* mass, cudaStream_t stream) {
  Layout lo;
  spa_status st = common_checks(p, workspace, workspace_bytes, &lo);
  if (st != SPA_OK) return st;
  if (window < 0) return SPA_ERR_INVALID;
  if (p->mode != SPA_MODE_DENSE && window > p->local - p->block_q) return SPA_ERR_UNSUPPORTED;
  const int B = p->batch, Hq = p->heads_q, Hkv = p->heads_kv, L = p->seq_len;
  if (B == 0 || L == 0) return SPA_OK;
  if (!q || !k || !lse || !mass || !aligned16(q) || !aligned16(k) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u) || (reinterpret_cast<uintptr_t>(mass) & 3u))
    return SPA_ERR_INVALID;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const long long BH = (long long)B * Hq, BKV = (long long)B * Hkv;
  CUtensorMap tq, tk, tkg;
  if (!map_2d(&tq, kBF16, 2, q, 128, BH * L, 64, 128, kSW128) ||
      !map_2d(&tk, kBF16, 2, k, 128, BKV * L, 64, 128, kSW128) ||
      !map_2d(&tkg, kBF16, 2, k, 128, BKV * L, 64, 1, kSW128))
    return SPA_ERR_CUDA;
  if (cudaMemsetAsync(mass, 0, (size_t)BKV * L * sizeof(float), stream) != cudaSuccess)
    return SPA_ERR_CUDA;
  MassArgs a;
  a.g = tile_geom(p, lo, ws);
  a.sl2 = eff_scale(p) * 1.4426950408889634f;
  a.window = window;
  a.lse = lse;
  a.mass = mass;
  a.err = reinterpret_cast<uint32_t*>(ws);
  a.wait_ns = wait_ns(p);
  if (set_smem(key_mass_kernel, kMassSmemBytes) != cudaSuccess) return SPA_ERR_CUDA;
  key_mass_kernel<<<(unsigned)lo.nb, kMassThreads, kMassSmemBytes, stream>>>(tq, tk, tkg, a);
  if (cudaGetLastError() != cudaSuccess) return SPA_ERR_CUDA;
  return SPA_OK;
}

}  // extern "C"
