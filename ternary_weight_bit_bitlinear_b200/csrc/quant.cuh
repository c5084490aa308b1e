// quant.cuh -- per-token absmax int8 activation quantisation.
//
// The I2_S setting quantises activations to int8 with an absmax scale
// ("Bitnet.cpp" reading notes, section 2.3 and section 4.1); here one scale
// per token row.  q = clamp(rint(x * (127/amax)), -128, 127), ties to even.
// One CTA per token: a warp-shuffle max reduction, then a second pass that
// quantises, stores four int8 per 32-bit word and reduces the row sum.
#pragma once

#include "ptx.cuh"

namespace bl {

constexpr int kQuantThreads = 512;

__device__ __forceinline__ int quant_one(float x, float s) {
  int v = __float2int_rn(__fmul_rn(x, s));   // NaN (0 * inf) -> 0; +-inf saturate
  return max(-128, min(127, v));
}

__global__ void __launch_bounds__(kQuantThreads)
quant_act_kernel(const float* __restrict__ x, int K, int8_t* __restrict__ xq,
                 float* __restrict__ amax_out, int32_t* __restrict__ xsum_out) {
  __shared__ float red_f[kQuantThreads / 32];
  __shared__ int red_i[kQuantThreads / 32];
  const int n = blockIdx.x;
  const float4* row = reinterpret_cast<const float4*>(x + static_cast<int64_t>(n) * K);
  const int K4 = K / 4;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

  float m = 0.0f;
  for (int i = threadIdx.x; i < K4; i += blockDim.x) {
    float4 v = __ldg(row + i);
    m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if (lane == 0) red_f[warp] = m;
  __syncthreads();
  float amax = 0.0f;
#pragma unroll
  for (int w = 0; w < kQuantThreads / 32; ++w) amax = fmaxf(amax, red_f[w]);

  uint32_t* out = reinterpret_cast<uint32_t*>(xq + static_cast<int64_t>(n) * K);
  int sum = 0;
  if (amax == 0.0f) {
    for (int i = threadIdx.x; i < K4; i += blockDim.x) out[i] = 0u;
  } else {
    const float s = __fdiv_rn(127.0f, amax);
    for (int i = threadIdx.x; i < K4; i += blockDim.x) {
      float4 v = __ldg(row + i);
      int a = quant_one(v.x, s), b = quant_one(v.y, s), c = quant_one(v.z, s),
          d = quant_one(v.w, s);
      sum += a + b + c + d;
      out[i] = (static_cast<uint32_t>(a) & 0xFFu) | ((static_cast<uint32_t>(b) & 0xFFu) << 8) |
               ((static_cast<uint32_t>(c) & 0xFFu) << 16) | (static_cast<uint32_t>(d) << 24);
    }
  }
  if (threadIdx.x == 0) amax_out[n] = amax;
  if (xsum_out) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
    if (lane == 0) red_i[warp] = sum;
    __syncthreads();
    if (threadIdx.x == 0) {
      int t = 0;
#pragma unroll
      for (int w = 0; w < kQuantThreads / 32; ++w) t += red_i[w];
      xsum_out[n] = t;
    }
  }
}

}  // namespace bl
