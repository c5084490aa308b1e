// gemv.cuh -- decode mpGEMM for a few tokens (N <= 16) on the CUDA cores.
//
// The reading notes' I2_S kernel is MAD-based: int8 multiply-adds of
// activations against ternary weights ("Bitnet.cpp" reading notes, section 4.1
// item 3); the FairyFuse "fused kernel design" unpacks the bit-packed codes
// and accumulates in the same loop with no intermediate writes.  Here each
// 16-byte load brings 64 weights; (word >> 2j) & 0x03030303 puts four codes+1
// in byte lanes that line up with four int8 activations, so one dp4a does four
// multiply-adds.  The +1 offset is removed once per output with the token's
// activation sum: acc = dp4a_total - xsum.
#pragma once

#include "ptx.cuh"

namespace bl {

constexpr int kGemvThreads = 256;
constexpr int kGemvRows = 4;   // rows per warp

__device__ __forceinline__ uint4 ld_stream_u4(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

template <int NT>
__global__ void __launch_bounds__(kGemvThreads)
gemv_kernel(const uint4* __restrict__ wq, int M, int cpr,      // cpr = K / 64 chunks per row
            const uint4* __restrict__ xq4,                       // [N, 4*cpr] uint4
            const float* __restrict__ alpha_ptr, const float* __restrict__ amax,
            const int32_t* __restrict__ xsum, float* __restrict__ y,
            int32_t* __restrict__ acc_out) {
  constexpr int R = kGemvRows;
  const int lane = threadIdx.x & 31;
  const int warp_global = (blockIdx.x * kGemvThreads + threadIdx.x) >> 5;
  const int row0 = warp_global * R;
  if (row0 >= M) return;

  int acc[R][NT];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[r][t] = 0;

  for (int c = lane; c < cpr; c += 32) {
    uint32_t u[R][16];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      uint4 w = make_uint4(0x55555555u, 0x55555555u, 0x55555555u, 0x55555555u);
      if (row0 + r < M) w = ld_stream_u4(wq + static_cast<int64_t>(row0 + r) * cpr + c);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) u[r][4 * i + j] = (ws[i] >> (2 * j)) & 0x03030303u;
    }
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const uint4* xa = xq4 + static_cast<int64_t>(t) * 4 * cpr + 4 * c;
      int a[16];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint4 v = __ldg(xa + i);
        a[4 * i + 0] = static_cast<int>(v.x);
        a[4 * i + 1] = static_cast<int>(v.y);
        a[4 * i + 2] = static_cast<int>(v.z);
        a[4 * i + 3] = static_cast<int>(v.w);
      }
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[r][t] = __dp4a(static_cast<int>(u[r][e]), a[e], acc[r][t]);
    }
  }

#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[r][t] += __shfl_xor_sync(0xFFFFFFFFu, acc[r][t], o);

  const float alpha = *alpha_ptr;
#pragma unroll
  for (int r = 0; r < R; ++r) {
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      if (lane == ((r * NT + t) & 31) && row0 + r < M) {
        const int a = acc[r][t] - xsum[t];
        const float scale = __fmul_rn(alpha, __fdiv_rn(amax[t], 127.0f));
        const int64_t o = static_cast<int64_t>(t) * M + row0 + r;
        y[o] = __fmul_rn(__int2float_rn(a), scale);
        if (acc_out) acc_out[o] = a;
      }
    }
  }
}

}  // namespace bl
