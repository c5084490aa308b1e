// quant.cuh -- per-token absmax int8 activation quantisation.
//
// The I2_S setting quantises activations to int8 with an absmax scale
// ("Bitnet.cpp" reading notes, section 2.3 and section 4.1); here one scale
// per token row.  q = clamp(rint(x * (127/amax)), -128, 127), ties to even.
//
// One CTA per token row, rows of several matrices numbered across one launch.
// Each thread loads its float4s of the row once and keeps up to kQuantRegF4 of
// them in registers; the maximum is reduced with warp shuffles and one
// shared-memory exchange, the row is quantised from registers, stored four
// int8 per 32-bit word, and the row sum reduced the same way.  Launches of
// many rows use 256-thread CTAs (rows up to 8192 wide read exactly once, and
// several rows in flight per SM).  Launches of fewer rows than SMs (a
// decoder's one token) take the fewest threads, from 256 up to 1024, that
// hold the widest row in registers (quant_wide_threads), so a row's latency
// is one read and two block reductions; more threads than that only lengthen
// the reductions.
//
// Per-tensor mode (the reading notes' own I2_S setting, section 2.3 and
// section 4.1: one int8 scale for the whole activation tensor): a first
// kernel folds max|x| over the matrix into one word, and the row kernel takes
// that maximum instead of the row's.
#pragma once

#include "ptx.cuh"
#include "quant_math.cuh"

namespace bl {

constexpr int kQuantThreads = 256;        // row-kernel CTA size for launches of many rows
constexpr int kQuantRegF4 = 8;             // float4 per thread kept in registers
constexpr int kQuantMaxMatrices = 64;

struct QuantMatrix {
  const float* x;
  int8_t* xq;
  float* amax;
  int32_t* xsum;   // may be null
  const unsigned int* tensor_amax;   // per-tensor mode: bits of max|x| over the matrix
  int K;
  int row_begin;   // first global row of this matrix
};

struct QuantParams {
  QuantMatrix m[kQuantMaxMatrices];
  int count;
};

template <int kThreads>
static __global__ void __launch_bounds__(kThreads)
quant_rows_kernel(const __grid_constant__ QuantParams p) {
  __shared__ float red_f[kThreads / 32];
  __shared__ int red_i[kThreads / 32];
  pdl_wait_prior_grid();
  pdl_allow_next_grid();
  const int g = blockIdx.x;
  int mi = 0;
  while (mi + 1 < p.count && g >= p.m[mi + 1].row_begin) ++mi;
  const QuantMatrix A = p.m[mi];   // by value: registers, not parameter-space reloads
  const int n = g - A.row_begin;
  const int K4 = A.K / 4;
  const float4* row = reinterpret_cast<const float4*>(A.x + static_cast<int64_t>(n) * A.K);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

  float4 v[kQuantRegF4];
  float m = 0.0f;
#pragma unroll
  for (int j = 0; j < kQuantRegF4; ++j) {
    const int i = threadIdx.x + j * kThreads;
    v[j] = i < K4 ? __ldg(row + i) : make_float4(0.f, 0.f, 0.f, 0.f);
    m = fmaxf(m, absmax4(v[j]));
  }
  float amax = 0.0f;
  if (A.tensor_amax) {
    amax = __uint_as_float(*A.tensor_amax);
  } else {
    for (int i = threadIdx.x + kQuantRegF4 * kThreads; i < K4; i += kThreads)
      m = fmaxf(m, absmax4(__ldg(row + i)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if (lane == 0) red_f[warp] = m;
    __syncthreads();
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) amax = fmaxf(amax, red_f[w]);
  }

  uint32_t* out = reinterpret_cast<uint32_t*>(A.xq + static_cast<int64_t>(n) * A.K);
  int sum = 0;
  if (amax == 0.0f) {
    for (int i = threadIdx.x; i < K4; i += kThreads) out[i] = 0u;
  } else {
    const float s = __fdiv_rn(127.0f, amax);
#pragma unroll
    for (int j = 0; j < kQuantRegF4; ++j) {
      const int i = threadIdx.x + j * kThreads;
      if (i < K4) out[i] = quant_pack4(v[j], s, sum);
    }
    for (int i = threadIdx.x + kQuantRegF4 * kThreads; i < K4; i += kThreads)
      out[i] = quant_pack4(__ldg(row + i), s, sum);
  }
  if (threadIdx.x == 0) A.amax[n] = amax;
  if (A.xsum) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
    if (lane == 0) red_i[warp] = sum;
    __syncthreads();
    if (threadIdx.x == 0) {
      int t = 0;
#pragma unroll
      for (int w = 0; w < kThreads / 32; ++w) t += red_i[w];
      A.xsum[n] = t;
    }
  }
}

// CTA size of a launch of fewer rows than SMs whose widest row is kmax wide.
inline int quant_wide_threads(int64_t kmax) {
  return kmax <= 4 * kQuantRegF4 * 256 ? 256 : kmax <= 4 * kQuantRegF4 * 512 ? 512 : 1024;
}

// Per-tensor maximum of |x| over n4 float4s, folded into *out (the bits of a
// non-negative float order like unsigned integers, so atomicMax on them is
// the float maximum).  *out must start at 0.
static __global__ void __launch_bounds__(kQuantThreads)
tensor_absmax_kernel(const float4* __restrict__ x, int64_t n4, unsigned int* __restrict__ out) {
  __shared__ float red[kQuantThreads / 32];
  pdl_wait_prior_grid();
  pdl_allow_next_grid();
  float m = 0.0f;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += stride)
    m = fmaxf(m, absmax4(__ldg(x + i)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float b = 0.0f;
#pragma unroll
    for (int w = 0; w < kQuantThreads / 32; ++w) b = fmaxf(b, red[w]);
    atomicMax(out, __float_as_uint(b));
  }
}

}  // namespace bl
