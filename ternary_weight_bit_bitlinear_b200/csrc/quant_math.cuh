// quant_math.cuh -- the per-token absmax int8 quantiser's arithmetic, shared
// by the quantiser kernels (quant.cuh) and the fused decode kernels: one
// element, four elements packed into a 32-bit word, and the absolute maximum
// of a float4.  q = clamp(rint(x * s), -128, 127) with s = 127 / amax, ties
// to even ("Bitnet.cpp" reading notes, section 2.3: int8 activations with an
// absmax scale).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace bl {

__device__ __forceinline__ int quant_one(float x, float s) {
  int v = __float2int_rn(__fmul_rn(x, s));   // NaN (0 * inf) -> 0; +-inf saturate
  return max(-128, min(127, v));
}

__device__ __forceinline__ uint32_t quant_pack4(float4 v, float s, int& sum) {
  const int a = quant_one(v.x, s), b = quant_one(v.y, s), c = quant_one(v.z, s),
            d = quant_one(v.w, s);
  sum += a + b + c + d;
  return (static_cast<uint32_t>(a) & 0xFFu) | ((static_cast<uint32_t>(b) & 0xFFu) << 8) |
         ((static_cast<uint32_t>(c) & 0xFFu) << 16) | (static_cast<uint32_t>(d) << 24);
}

__device__ __forceinline__ float absmax4(float4 v) {
  return fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
}

}  // namespace bl
