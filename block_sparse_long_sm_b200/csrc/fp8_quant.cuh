// fp8_quant.cuh -- E4M3 quantisation of Q, K and V for the FP8 attention.
//
// SALE runs its Computation Pass on quantised operands in the manner of
// SageAttention (the review of SALE, Summary).  For the tcgen05 kind::f8f6f4
// tensor cores the operands are OCP E4M3 ("fn": bias 7, 3 mantissa bits,
// largest finite 448), rounded to nearest even and saturated:
//   Q   one scale per (b, q head, 128-row block);
//   K   smoothed by its per-(b, kv head) sequence mean (a constant shift of
//       every score of a row, which the softmax cancels), then one scale per
//       (b, kv head);
//   V   one scale per (b, kv head, channel).
// scale = absmax / 448 in IEEE fp32 (1 for an all-zero group) and
// code = E4M3(x / scale) with an IEEE fp32 division.
//
//   fp8_quant_q_kernel     grid (nqb, B*Hq): absmax and codes of one Q block;
//   fp8_kv_absmax_kernel   grid (chunks, B*Hkv): absmax of smoothed K per head
//                          and of V per channel, merged with atomicMax on the
//                          bits of non-negative floats;
//   fp8_kv_quant_kernel    grid (chunks, B*Hkv): K and V codes.
// The K mean comes from the SALE K-mean kernels (the same smoothing).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "common.cuh"
#include "fp8_cvt.cuh"

namespace spa {

constexpr int kFp8Chunks = 64;      // row chunks per (b, kv head) for K and V

__device__ __forceinline__ float fp8_scale(float amax) {
  return amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
}

struct Fp8QuantArgs {
  const __nv_bfloat16* q;     // [B*Hq][L][128]
  const __nv_bfloat16* k;     // [B*Hkv][L][128]
  const __nv_bfloat16* v;
  const float* kmean;         // [B*Hkv][128]
  int L, nqb;
  uint8_t* q8;                // codes, same layouts as q, k, v
  uint8_t* k8;
  uint8_t* v8;
  float* qs;                  // [B*Hq][nqb]
  float* ks;                  // [B*Hkv]
  float* vs;                  // [B*Hkv][128]
  uint32_t* kabs;             // [B*Hkv]       absmax bits, zeroed before the absmax pass
  uint32_t* vabs;             // [B*Hkv][128]
};

__device__ __forceinline__ float block_max128(float x, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = x;
  __syncthreads();
  return fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
}

// thread d owns column d of the block
__global__ void __launch_bounds__(128) fp8_quant_q_kernel(const Fp8QuantArgs a) {
  __shared__ float red[4];
  const int bh = blockIdx.y, qb = blockIdx.x, d = threadIdx.x;
  const int r0 = qb * 128, r1 = min(r0 + 128, a.L);
  const __nv_bfloat16* xp = a.q + (long long)bh * a.L * 128 + d;
  float amax = 0.f;
  for (int r = r0; r < r1; ++r) amax = fmaxf(amax, fabsf(__bfloat162float(xp[(long long)r * 128])));
  const float s = fp8_scale(block_max128(amax, red));
  uint8_t* cp = a.q8 + (long long)bh * a.L * 128 + d;
  for (int r = r0; r < r1; ++r)
    cp[(long long)r * 128] = e4m3(__fdiv_rn(__bfloat162float(xp[(long long)r * 128]), s));
  if (d == 0) a.qs[(long long)bh * a.nqb + qb] = s;
}

__global__ void __launch_bounds__(128) fp8_kv_absmax_kernel(const Fp8QuantArgs a) {
  __shared__ float red[4];
  const int bkv = blockIdx.y, chunk = blockIdx.x, d = threadIdx.x;
  const int per = (a.L + kFp8Chunks - 1) / kFp8Chunks;
  const int r0 = chunk * per, r1 = min(r0 + per, a.L);
  const long long base = (long long)bkv * a.L * 128 + d;
  const float mu = a.kmean[(long long)bkv * 128 + d];
  float ak = 0.f, av = 0.f;
  for (int r = r0; r < r1; ++r) {
    const long long i = base + (long long)r * 128;
    ak = fmaxf(ak, fabsf(__fsub_rn(__bfloat162float(a.k[i]), mu)));
    av = fmaxf(av, fabsf(__bfloat162float(a.v[i])));
  }
  ak = block_max128(ak, red);
  if (d == 0 && ak > 0.f) atomicMax(&a.kabs[bkv], __float_as_uint(ak));
  if (av > 0.f) atomicMax(&a.vabs[(long long)bkv * 128 + d], __float_as_uint(av));
}

__global__ void __launch_bounds__(128) fp8_kv_quant_kernel(const Fp8QuantArgs a) {
  const int bkv = blockIdx.y, chunk = blockIdx.x, d = threadIdx.x;
  const int per = (a.L + kFp8Chunks - 1) / kFp8Chunks;
  const int r0 = chunk * per, r1 = min(r0 + per, a.L);
  const long long base = (long long)bkv * a.L * 128 + d;
  const float mu = a.kmean[(long long)bkv * 128 + d];
  const float sk = fp8_scale(__uint_as_float(a.kabs[bkv]));
  const float sv = fp8_scale(__uint_as_float(a.vabs[(long long)bkv * 128 + d]));
  for (int r = r0; r < r1; ++r) {
    const long long i = base + (long long)r * 128;
    a.k8[i] = e4m3(__fdiv_rn(__fsub_rn(__bfloat162float(a.k[i]), mu), sk));
    a.v8[i] = e4m3(__fdiv_rn(__bfloat162float(a.v[i]), sv));
  }
  if (chunk == 0) {
    a.vs[(long long)bkv * 128 + d] = sv;
    if (d == 0) a.ks[bkv] = sk;
  }
}

}  // namespace spa
