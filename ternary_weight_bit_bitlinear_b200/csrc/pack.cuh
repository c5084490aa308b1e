// pack.cuh -- weight absmean, ternarisation and 2-bit packing.
//
// BitNet b1.58 weights are ternary with one per-tensor scale ("Bitnet.cpp:
// Efficient Edge Inference for Ternary LLMs" reading notes, section 1.1 and
// section 4.1 "lossless inference conditions"; I2_S stores them at 2.0 bits per
// weight, section 2.3 method table).  The scale is alpha = mean|W|.
//
// Three launches:
//   1. abs_bins:  exact sum of |W| as integer significands binned by exponent
//                 (integer adds commute, so the sum is order-free);
//   2. alpha_finalize: one thread turns the bins into mean|W| rounded once to
//                 fp32 (binary long division, round half to even);
//   3. ternarize_pack: c = clamp(rint(W/alpha), -1, 1), 16 weights per word.
#pragma once

#include "ptx.cuh"

namespace bl {

// Workspace layout of bitlinear_pack_weights: 256 uint64 bins, then a flag.
constexpr int kBins = 256;
constexpr size_t kPackWorkspaceBytes = kBins * sizeof(unsigned long long) + 16;

constexpr int kBinsThreads = 256;
constexpr int kBinsWarps = kBinsThreads / 32;

// Per-warp shared histograms keep same-address atomics inside one warp.
static __global__ void __launch_bounds__(kBinsThreads)
abs_bins_kernel(const float4* __restrict__ w4, int64_t n4,
                unsigned long long* __restrict__ bins, unsigned int* __restrict__ flag) {
  __shared__ unsigned long long hist[kBinsWarps][kBins];
  for (int i = threadIdx.x; i < kBinsWarps * kBins; i += blockDim.x) (&hist[0][0])[i] = 0ull;
  __syncthreads();
  unsigned long long* mine = hist[threadIdx.x / 32];
  unsigned int bad = 0;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += stride) {
    float4 v = __ldcs(w4 + i);
    float e4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t bits = __float_as_uint(e4[j]);
      uint32_t ex = (bits >> 23) & 0xFFu;
      uint32_t frac = bits & 0x7FFFFFu;
      if (ex == 0xFFu) {
        bad = 1;
      } else {
        uint32_t sig = ex ? (frac | 0x800000u) : frac;   // value = sig * 2^(max(ex,1) - 150)
        if (sig) atomicAdd(&mine[ex ? ex : 1u], static_cast<unsigned long long>(sig));
      }
    }
  }
  if (bad) atomicOr(flag, 1u);
  __syncthreads();
  for (int b = threadIdx.x; b < kBins; b += blockDim.x) {
    unsigned long long s = 0;
#pragma unroll
    for (int w = 0; w < kBinsWarps; ++w) s += hist[w][b];
    if (s) atomicAdd(&bins[b], s);
  }
}

// Single thread.  mean|W| = (sum_e bins[e] * 2^(e-1)) * 2^-149 / count.
// The numerator is a 384-bit integer D; restoring division by `count`, one
// quotient bit per numerator bit from the top, continued into fractional bit
// positions until the bit below the fp32 unit in the last place is known.
static __global__ void alpha_finalize_kernel(const unsigned long long* __restrict__ bins,
                                      const unsigned int* __restrict__ flag, uint64_t count,
                                      float* __restrict__ alpha) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  if (*flag) {
    *alpha = __int_as_float(0x7FC00000);   // NaN marks a non-finite weight
    atomicOr(&g_device_error, kDeviceNonFinite);
    return;
  }
  constexpr int kLimbs = 12;   // 384 bits; the numerator needs < 320
  uint32_t D[kLimbs];
#pragma unroll
  for (int i = 0; i < kLimbs; ++i) D[i] = 0;
  for (int e = 1; e < 255; ++e) {
    unsigned long long v = bins[e];
    if (!v) continue;
    int pos = e - 1;   // add v << pos
    int limb = pos >> 5, sh = pos & 31;
    unsigned long long carry = 0;
    // split v << sh into three 32-bit pieces
    uint32_t piece[3];
    piece[0] = static_cast<uint32_t>(v << sh);
    piece[1] = static_cast<uint32_t>(sh ? (v >> (32 - sh)) : (v >> 32));
    piece[2] = static_cast<uint32_t>(sh ? (v >> (64 - sh)) : 0ull);
    for (int i = limb; i < kLimbs; ++i) {
      unsigned long long add = (i - limb < 3) ? piece[i - limb] : 0u;
      unsigned long long s = static_cast<unsigned long long>(D[i]) + add + carry;
      D[i] = static_cast<uint32_t>(s);
      carry = s >> 32;
    }
  }
  int top = -1;
  for (int i = kLimbs - 1; i >= 0 && top < 0; --i)
    if (D[i]) top = i * 32 + 31 - __clz(D[i]);
  if (top < 0) {
    *alpha = 0.0f;
    return;
  }
  // Quotient bit produced at numerator position p weighs 2^(p - 149).
  unsigned long long rem = 0;
  int lead = INT_MIN;          // position of the leading quotient 1
  int ulp_pos = 0;             // position of the fp32 last place
  uint64_t mant = 0;
  int guard = 0;
  int p = top;
  for (;; --p) {
    int bit = (p >= 0) ? static_cast<int>((D[p >> 5] >> (p & 31)) & 1u) : 0;
    rem = (rem << 1) | static_cast<unsigned long long>(bit);
    int q = 0;
    if (rem >= count) {
      rem -= count;
      q = 1;
    }
    if (q && lead == INT_MIN) {
      lead = p;
      ulp_pos = (lead - 149 >= -126) ? (lead - 23) : 0;
    }
    int ulp_now = (lead == INT_MIN) ? 0 : ulp_pos;
    if (p >= ulp_now) {
      mant = (mant << 1) | static_cast<uint64_t>(q);
    } else {          // p == ulp_now - 1: the guard bit
      guard = q;
      break;
    }
  }
  // Sticky: remainder, or numerator bits not yet brought down.
  bool sticky = rem != 0;
  for (int b = p - 1; b >= 0 && !sticky; --b) sticky = (D[b >> 5] >> (b & 31)) & 1u;
  if (guard && (sticky || (mant & 1u))) ++mant;
  int ulp_final = (lead == INT_MIN) ? 0 : ulp_pos;
  *alpha = static_cast<float>(ldexp(static_cast<double>(mant), ulp_final - 149));
}

// One thread per packed word.  A row holds `wp` words: the first `kw` =
// K/16 carry 16 consecutive weights each, the rest (when K is not a multiple
// of 64) pad the row to a 16-byte boundary with code-0 fields (01).
static __global__ void __launch_bounds__(256)
ternarize_pack_kernel(const float4* __restrict__ w4, int64_t rows, int kw, int wp,
                      const float* __restrict__ alpha_ptr, uint32_t* __restrict__ packed) {
  const float alpha = *alpha_ptr;
  const int64_t words = rows * wp;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t w = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; w < words;
       w += stride) {
    int64_t src = 4 * w;                  // float4 index of the word's first weight
    if (wp != kw) {
      const int64_t m = w / wp;
      const int r = static_cast<int>(w - m * wp);
      if (r >= kw) {
        packed[w] = 0x55555555u;
        continue;
      }
      src = 4 * (m * kw + r);
    }
    uint32_t word = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {          // weights 4j .. 4j+3 of the word
      float4 v = __ldcs(w4 + src + j);
      float e4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        int c = 0;
        if (alpha != 0.0f) {
          c = __float2int_rn(__fdiv_rn(e4[b], alpha));   // NaN -> 0, +-inf saturate
          c = max(-1, min(1, c));
        }
        word |= static_cast<uint32_t>(c + 1) << (8 * b + 2 * j);
      }
    }
    packed[w] = word;
  }
}

}  // namespace bl
