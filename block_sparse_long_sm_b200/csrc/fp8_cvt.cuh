// fp8_cvt.cuh -- E4M3 conversions (OCP "fn": bias 7, 3 mantissa bits,
// largest finite 448) shared by the quantisation and attention kernels.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>

namespace spa {

// Two floats to E4M3 (lo in bits 0-7), round to nearest even, saturating.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  unsigned short r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ uint8_t e4m3(float x) { return static_cast<uint8_t>(e4m3x2(x, 0.f)); }

// Two E4M3 codes (bits 0-7 -> .x, bits 8-15 -> .y) to fp32, exactly (every
// E4M3 value is an fp16 value).
__device__ __forceinline__ float2 e4m3x2_to_f32(uint32_t codes) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(static_cast<unsigned short>(codes)));
  return __half22float2(*reinterpret_cast<const __half2*>(&h2));
}

}  // namespace spa
