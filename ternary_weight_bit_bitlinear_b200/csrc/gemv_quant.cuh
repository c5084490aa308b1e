// gemv_quant.cuh -- decode GEMV with the per-token activation quantiser fused
// into its prologue: fp32 activations in, fp32 outputs out, no int8 round trip
// through global memory and no second launch.
//
// The fusion follows the FairyFuse "fused kernel design" (activation handling,
// unpacking and accumulation in one kernel, no intermediate writes) and keeps
// the I2_S arithmetic of the "Bitnet.cpp" reading notes (section 2.3, section
// 4.1): per-token absmax int8 activations, ternary weights, int32 sums, one
// fp32 rescale.  The quantised values are the ones quant.cuh produces:
//   amax = max_k |x[k]|,  s = 127 / amax,  q = clamp(rint(x * s), -128, 127).
//
// Work split: one warp per CTA.  A launch's problems form segments: runs of
// consecutive problems that read the same input (pointer and K; q, k and v,
// or gate and up, when given side by side).  The host gives every segment a
// number of warps in proportion to its k-chunk count (at least one, at most
// its unit count), and each warp takes an equal share of its segment's units
// (32 rows x all of K, as in gemv.cuh).  A warp therefore quantises exactly
// one input, once, before it streams any weights:
//   1. the first weight stages are prefetched into L2 (their addresses do not
//      depend on the input), and when the staging below leaves the ring's
//      space alone, the ring's first stages are already copied in;
//   2. each token's fp32 row is copied into the warp's shared memory with
//      16-byte cp.async copies, all in flight at once;
//   3. amax is reduced from shared memory and the row is quantised, four int8
//      per 32-bit word;
//   4. the weight ring of gemv.cuh (weights only, 4 stages of 4 KB) streams
//      the warp's units, with activations read as broadcasts from the int8
//      copy.
// Shared memory of a CTA: the int8 copy [NT][xstride] at the start, the ring
// at the end.  When a token's fp32 row fits between its own int8 row and the
// end of the area it is staged there and quantised in place; otherwise it
// passes through the ring's space in pieces, once for the maximum and once to
// quantise.
#pragma once

#include "gemv.cuh"
#include "quant_math.cuh"

namespace bl {

constexpr int kGqStages = 4;                                          // power of two
constexpr int kGqStageBytes = kGemvTileRows * kGemvChunkBytes;        // 4 KB of weights
constexpr int kGqRingBytes = kGqStages * kGqStageBytes;
constexpr int kGqMaxProblems = 256;
constexpr int kGqMaxXBytes = 65536;   // tokens x K (rounded up to 512) held per warp

struct GqProblem {
  const uint32_t* packed;
  const float* alpha;
  float* y;                // fp32 [NT][M]
  int32_t* acc;            // int32 [NT][M] or null
  int M, W;                // W = K / 16 words per row
  int unit_begin;          // first unit of this problem
};

// A run of problems that read one input.  Its units all have the same K.
struct GqSegment {
  const float* x;          // fp32 [NT][K]
  int K;
  int chunks;              // k-chunks per unit: ceil(K / 512)
  int unit_begin, units;   // the segment's units, numbered across the launch
  int warp_begin, warps;   // the warps (CTAs) that share them
  int prob_begin;          // first problem of the segment
};

struct GqParams {
  GqProblem prob[kGqMaxProblems];
  GqSegment seg[kGqMaxProblems];
  int num_problems;
  int num_segments;
  int xstride;             // bytes per token of the int8 copy: 512 x the launch's largest chunks
  int area;                // dynamic shared memory bytes: >= NT * xstride + kGqRingBytes;
                           // the ring takes the last kGqRingBytes
};

// Quantise x [NT][K] (fp32, 16-byte aligned rows) into xs [NT][xstride] int8,
// zero from K up to kpad; amax / 127 and the sum of q of token t go to
// s_a127[t] and s_xsum[t].  Run by the whole warp.
//
// In place: token t's row is staged at xs + t * xstride; in round r each lane
// reads float4 32r + lane and then writes the word of the same index, i.e.
// bytes below 128r + 128, which only reach float4s that an earlier round (or
// this round, before the __syncwarp) has read.
// In pieces: the window [win, win + win_bytes) takes up to win_bytes / 4
// floats at a time, once for the maximum, once for the quantisation.
//
// With first_staged, token 0's row was staged in place already (gq_stage_first)
// as the oldest of kGqStages cp.async groups still pending; the others belong
// to the weight ring.
template <int NT>
__device__ __forceinline__ void gq_quantise(const float* __restrict__ x, int K, int kpad,
                                            int xstride, uint8_t* xs, uint8_t* win,
                                            int win_bytes, int area, float* s_a127,
                                            int* s_xsum, bool first_staged, int lane) {
  const int K4 = K / 4;
#pragma unroll 1
  for (int t = 0; t < NT; ++t) {
    uint8_t* row8 = xs + t * xstride;
    uint32_t* out = reinterpret_cast<uint32_t*>(row8);
    const float* row = x + static_cast<int64_t>(t) * K;
    float m = 0.0f;
    int sum = 0;
    if (t * xstride + 4 * K <= area) {
      if (t == 0 && first_staged) {
        cp_async_wait<kGqStages - 1>();
      } else {
        for (int i = lane; i < K4; i += 32) cp_async16(row8 + 16 * i, row + 4 * i, 16u);
        cp_async_commit();
        cp_async_wait<0>();
      }
      __syncwarp();
      const float4* v4 = reinterpret_cast<const float4*>(row8);
      for (int i = lane; i < K4; i += 32) m = fmaxf(m, absmax4(v4[i]));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
      const float s = m == 0.0f ? 0.0f : __fdiv_rn(127.0f, m);
      for (int base = 0; base < K4; base += 32) {   // uniform trip count: __syncwarp inside
        const int i = base + lane;
        const float4 v = i < K4 ? v4[i] : make_float4(0.f, 0.f, 0.f, 0.f);
        __syncwarp();
        if (i < K4) out[i] = m == 0.0f ? 0u : quant_pack4(v, s, sum);
      }
      __syncwarp();
    } else {
      const int P4 = win_bytes / 16;   // float4s per piece
      const float4* w4 = reinterpret_cast<const float4*>(win);
#pragma unroll 1
      for (int b = 0; b < K4; b += P4) {
        const int n = min(P4, K4 - b);
        for (int i = lane; i < n; i += 32) cp_async16(win + 16 * i, row + 4 * (b + i), 16u);
        cp_async_commit();
        cp_async_wait<0>();
        __syncwarp();
        for (int i = lane; i < n; i += 32) m = fmaxf(m, absmax4(w4[i]));
        __syncwarp();   // the window is read before the next piece lands
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
      const float s = m == 0.0f ? 0.0f : __fdiv_rn(127.0f, m);
#pragma unroll 1
      for (int b = 0; b < K4; b += P4) {
        const int n = min(P4, K4 - b);
        if (m != 0.0f) {
          for (int i = lane; i < n; i += 32) cp_async16(win + 16 * i, row + 4 * (b + i), 16u);
          cp_async_commit();
          cp_async_wait<0>();
          __syncwarp();
        }
        for (int i = lane; i < n; i += 32) out[b + i] = m == 0.0f ? 0u : quant_pack4(w4[i], s, sum);
        __syncwarp();
      }
    }
    for (int i = K4 + lane; i < kpad / 4; i += 32) out[i] = 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
    if (lane == 0) {
      s_a127[t] = __fdiv_rn(m, 127.0f);
      s_xsum[t] = sum;
    }
    __syncwarp();
  }
}

// Token 0's fp32 row staged in place at xs, as one cp.async group.
__device__ __forceinline__ void gq_stage_first(const float* __restrict__ x, int K, uint8_t* xs,
                                               int lane) {
  for (int i = lane; i < K / 4; i += 32) cp_async16(xs + 16 * i, x + 4 * i, 16u);
  cp_async_commit();
}

// Segment that warp b belongs to (the last one whose warp_begin <= b).
__device__ __forceinline__ int gq_segment_of(const GqParams& p, int b) {
  int lo = 0, hi = p.num_segments - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.seg[mid].warp_begin <= b) lo = mid; else hi = mid - 1;
  }
  return lo;
}

template <int NT>
__global__ void __launch_bounds__(32)
gemv_quant_kernel(const __grid_constant__ GqParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ float s_a127[NT];
  __shared__ int s_xsum[NT];
  const int lane = threadIdx.x;
  const uint32_t sw = static_cast<uint32_t>(lane & 7);
  uint8_t* xs = smem;
  uint8_t* ring = smem + p.area - kGqRingBytes;

  // This warp's units: an equal share of its segment's.
  const GqSegment sg = p.seg[gq_segment_of(p, blockIdx.x)];
  const int wi = blockIdx.x - sg.warp_begin;
  const int u_begin =
      sg.unit_begin + static_cast<int>(static_cast<int64_t>(sg.units) * wi / sg.warps);
  const int u_end =
      sg.unit_begin + static_cast<int>(static_cast<int64_t>(sg.units) * (wi + 1) / sg.warps);
  int pi = sg.prob_begin;
  while (pi + 1 < p.num_problems && p.prob[pi + 1].unit_begin <= u_begin) ++pi;

  // Copy plan of the first unit.  Its first stages are prefetched into L2
  // before the wait on the preceding kernel: that kernel may write the input,
  // and a prefetch is only a cache hint, so nothing is read too early.
  GqProblem ipr = p.prob[pi];
  GemvCopyPlan icp = gemv_plan(ipr, (u_begin - ipr.unit_begin) * kGemvTileRows, lane);
  if (u_begin < u_end) {
#pragma unroll 1
    for (int kc = 0; kc < kGqStages - 1 && kc < sg.chunks; ++kc) {
      if (kc * (kGemvChunkBytes / 4) + icp.wword < ipr.W) {
        const uint8_t* src = icp.wsrc + kc * kGemvChunkBytes;
#pragma unroll 1
        for (int i = 0; i < icp.vrows; ++i)
          asm volatile("prefetch.global.L2 [%0];" ::"l"(src + i * icp.wstep) : "memory");
      }
    }
  }
  pdl_wait_prior_grid();
  pdl_allow_next_grid();
  if (u_begin >= u_end) return;

  // Copy side: weights of (unit, k-chunk) pairs, running ahead across units.
  int iu = u_begin, ic = 0, ipi = pi;
  int slot = 0;
  auto issue_next = [&]() {
    if (iu < u_end) {
      gemv_issue_weights(ipr.W, icp, ic, ring + slot * kGqStageBytes);
      if (++ic == sg.chunks) {
        ic = 0;
        if (++iu < u_end) {
          while (ipi + 1 < p.num_problems && p.prob[ipi + 1].unit_begin <= iu) ++ipi;
          ipr = p.prob[ipi];
          icp = gemv_plan(ipr, (iu - ipr.unit_begin) * kGemvTileRows, lane);
        }
      }
    }
    cp_async_commit();   // one group per stage, empty once the run is done
    slot = (slot + 1) & (kGqStages - 1);
  };
  // The ring's first stages go in before the quantisation when every token's
  // staged row ends below the ring.  Token 0's row is copied first, so that its
  // quantisation waits for that copy alone, not for the weights behind it.
  const bool early_ring = (NT - 1) * p.xstride + 4 * sg.K <= p.area - kGqRingBytes;
  if (early_ring) {
    gq_stage_first(sg.x, sg.K, xs, lane);
#pragma unroll 1
    for (int s = 0; s < kGqStages - 1; ++s) issue_next();
  }
  gq_quantise<NT>(sg.x, sg.K, sg.chunks * kGemvChunkK, p.xstride, xs, smem + NT * p.xstride,
                  p.area - NT * p.xstride, p.area, s_a127, s_xsum, early_ring, lane);
  if (!early_ring) {
#pragma unroll 1
    for (int s = 0; s < kGqStages - 1; ++s) issue_next();
  }

  int cslot = 0;
  for (int cu = u_begin; cu < u_end; ++cu) {
    while (pi + 1 < p.num_problems && p.prob[pi + 1].unit_begin <= cu) ++pi;
    const GqProblem pr = p.prob[pi];   // by value: registers, not parameter-space reloads
    const int row0 = (cu - pr.unit_begin) * kGemvTileRows;

    int acc[NT][4];
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[t][j] = 0;

    for (int kc = 0; kc < sg.chunks; ++kc) {
      issue_next();
      cp_async_wait<kGqStages - 1>();
      __syncwarp();
      const uint8_t* st = ring + cslot * kGqStageBytes;
      cslot = (cslot + 1) & (kGqStages - 1);
      gemv_chunk_dot<NT>(st + lane * kGemvChunkBytes, sw, xs + kc * kGemvChunkK, p.xstride, acc);
      __syncwarp();   // every lane is done with this stage before it is refilled
    }

    const int row = row0 + lane;
    if (row < pr.M) {
      const float alpha = *pr.alpha;
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        const int a = acc[t][0] + (acc[t][1] >> 2) + (acc[t][2] >> 4) + (acc[t][3] >> 6) -
                      s_xsum[t];
        const float scale = __fmul_rn(alpha, s_a127[t]);
        const int64_t o = static_cast<int64_t>(t) * pr.M + row;
        pr.y[o] = __fmul_rn(__int2float_rn(a), scale);
        if (pr.acc) pr.acc[o] = a;
      }
    }
  }
  cp_async_wait<0>();
}

// ---------------------------------------------------------------------------
// Split-unit variant, for launches with fewer units than the kernel above has
// warp slots (one layer, or one input group of a layer, per launch: the order
// of a real decoder).  There every warp above would own one unit and work
// alone on its SM, so one warp's quantisation of a whole input row and its
// walk through all k-chunks of the unit would be the launch's latency.  Here
// one CTA of kGqsWarps warps takes one unit:
//   1. each warp prefetches its share of the k-chunks into L2 (before the
//      dependent-launch wait) and issues its ring's first stages;
//   2. all threads reduce amax per token, combine it through shared memory
//      and quantise their float4s into the shared int8 copy; x is read once
//      into registers when every token's row fits 16 float4s per thread in
//      total, twice (the second time from L2) otherwise;
//   3. warp w streams k-chunks [C w / S, C (w + 1) / S) through its own ring
//      (gemv.cuh's layout and arithmetic);
//   4. the other warps leave their int32 sums in their rings, and warp 0 adds
//      them (integers: the order does not matter) and writes y as above.
// Shared memory: the int8 copy [NT][xstride], then kGqsWarps rings.

constexpr int kGqsWarps = 4;
constexpr int kGqsThreads = 32 * kGqsWarps;
constexpr int kGqsMaxTokens = 4;
constexpr int kGqsRegF4 = 16;   // float4s per thread held in registers, over all tokens
constexpr int kGqsPrefetchChunks = 8;

__host__ __device__ constexpr int gqs_smem_bytes(int nt, int xstride) {
  return nt * xstride + kGqsWarps * kGqRingBytes;
}

// Problem and segment of unit u: the last whose unit_begin <= u.
__device__ __forceinline__ int gq_problem_of_unit(const GqParams& p, int u) {
  int lo = 0, hi = p.num_problems - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.prob[mid].unit_begin <= u) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ int gq_segment_of_unit(const GqParams& p, int u) {
  int lo = 0, hi = p.num_segments - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.seg[mid].unit_begin <= u) lo = mid; else hi = mid - 1;
  }
  return lo;
}

template <int NT>
__global__ void __launch_bounds__(kGqsThreads)
gemv_quant_split_kernel(const __grid_constant__ GqParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ float s_m[kGqsWarps][NT];
  __shared__ int s_q[kGqsWarps][NT];
  __shared__ float s_a127[NT];
  __shared__ int s_xsum[NT];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t sw = static_cast<uint32_t>(lane & 7);
  const int unit = blockIdx.x;
  const GqProblem pr = p.prob[gq_problem_of_unit(p, unit)];
  const GqSegment sg = p.seg[gq_segment_of_unit(p, unit)];
  const int row0 = (unit - pr.unit_begin) * kGemvTileRows;
  const int kc0 = sg.chunks * warp / kGqsWarps;
  const int kc1 = sg.chunks * (warp + 1) / kGqsWarps;
  uint8_t* xs = smem;
  uint8_t* ring = smem + NT * p.xstride + warp * kGqRingBytes;

  // 1. L2 prefetch of this warp's k-chunks, up to kGqsPrefetchChunks (a hint:
  //    nothing is read before the wait), then the ring's first stages after it.
  const GemvCopyPlan cp = gemv_plan(pr, row0, lane);
#pragma unroll 1
  for (int kc = kc0; kc < kc1 && kc < kc0 + kGqsPrefetchChunks; ++kc) {
    if (kc * (kGemvChunkBytes / 4) + cp.wword < pr.W) {
      const uint8_t* src = cp.wsrc + kc * kGemvChunkBytes;
#pragma unroll 1
      for (int i = 0; i < cp.vrows; ++i)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(src + i * cp.wstep) : "memory");
    }
  }
  pdl_wait_prior_grid();
  pdl_allow_next_grid();
  int ic = kc0, slot = 0;
  auto issue_next = [&]() {
    if (ic < kc1) gemv_issue_weights(pr.W, cp, ic++, ring + slot * kGqStageBytes);
    cp_async_commit();   // one group per stage, empty past this warp's chunks
    slot = (slot + 1) & (kGqStages - 1);
  };
#pragma unroll 1
  for (int st = 0; st < kGqStages - 1; ++st) issue_next();

  // 2. amax per token over the whole CTA, then the quantisation.  Rows with
  //    K <= 4 * kGqsRegF4 / NT * kGqsThreads are read once, into registers;
  //    otherwise x is read twice (the second time from L2).
  const int K4 = sg.K / 4, P4 = sg.chunks * (kGemvChunkK / 4);
  constexpr int R = kGqsRegF4 / NT;   // float4s per thread and token
  if (K4 <= R * kGqsThreads) {
    float4 v[NT][R];
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const float4* x4 = reinterpret_cast<const float4*>(sg.x + static_cast<int64_t>(t) * sg.K);
      float m = 0.0f;
#pragma unroll
      for (int j = 0; j < R; ++j) {
        const int i = tid + j * kGqsThreads;
        v[t][j] = i < K4 ? x4[i] : make_float4(0.f, 0.f, 0.f, 0.f);
        m = fmaxf(m, absmax4(v[t][j]));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
      if (lane == 0) s_m[warp][t] = m;
    }
    __syncthreads();
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      float m = 0.0f;
#pragma unroll
      for (int w = 0; w < kGqsWarps; ++w) m = fmaxf(m, s_m[w][t]);
      const float s = m == 0.0f ? 0.0f : __fdiv_rn(127.0f, m);
      uint32_t* out = reinterpret_cast<uint32_t*>(xs + t * p.xstride);
      int sum = 0;
#pragma unroll
      for (int j = 0; j < R; ++j) {
        const int i = tid + j * kGqsThreads;
        if (i < K4) out[i] = m == 0.0f ? 0u : quant_pack4(v[t][j], s, sum);
      }
      for (int i = K4 + tid; i < P4; i += kGqsThreads) out[i] = 0u;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
      if (lane == 0) s_q[warp][t] = sum;
    }
  } else {
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const float4* x4 = reinterpret_cast<const float4*>(sg.x + static_cast<int64_t>(t) * sg.K);
      float m = 0.0f;
      for (int i = tid; i < K4; i += kGqsThreads) m = fmaxf(m, absmax4(x4[i]));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
      if (lane == 0) s_m[warp][t] = m;
    }
    __syncthreads();
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      float m = 0.0f;
#pragma unroll
      for (int w = 0; w < kGqsWarps; ++w) m = fmaxf(m, s_m[w][t]);
      const float s = m == 0.0f ? 0.0f : __fdiv_rn(127.0f, m);
      const float4* x4 = reinterpret_cast<const float4*>(sg.x + static_cast<int64_t>(t) * sg.K);
      uint32_t* out = reinterpret_cast<uint32_t*>(xs + t * p.xstride);
      int sum = 0;
      for (int i = tid; i < K4; i += kGqsThreads)
        out[i] = m == 0.0f ? 0u : quant_pack4(x4[i], s, sum);
      for (int i = K4 + tid; i < P4; i += kGqsThreads) out[i] = 0u;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
      if (lane == 0) s_q[warp][t] = sum;
    }
  }
  __syncthreads();   // the int8 copy and the partial sums are complete
  if (tid < NT) {
    float m = 0.0f;
    int sum = 0;
#pragma unroll
    for (int w = 0; w < kGqsWarps; ++w) {
      m = fmaxf(m, s_m[w][tid]);
      sum += s_q[w][tid];
    }
    s_a127[tid] = __fdiv_rn(m, 127.0f);
    s_xsum[tid] = sum;
  }

  // 3. This warp's k-chunks.
  int acc[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[t][j] = 0;
  int cslot = 0;
  for (int kc = kc0; kc < kc1; ++kc) {
    issue_next();
    cp_async_wait<kGqStages - 1>();
    __syncwarp();
    const uint8_t* st = ring + cslot * kGqStageBytes;
    cslot = (cslot + 1) & (kGqStages - 1);
    gemv_chunk_dot<NT>(st + lane * kGemvChunkBytes, sw, xs + kc * kGemvChunkK, p.xstride, acc);
    __syncwarp();   // every lane is done with this stage before it is refilled
  }
  cp_async_wait<0>();
  __syncwarp();

  // 4. Partial sums through the rings, the epilogue by warp 0.
  int* red = reinterpret_cast<int*>(ring);   // [NT][4][32]
  if (warp > 0) {
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
      for (int j = 0; j < 4; ++j) red[(t * 4 + j) * 32 + lane] = acc[t][j];
  }
  __syncthreads();
  if (warp != 0) return;
#pragma unroll 1
  for (int w = 1; w < kGqsWarps; ++w) {
    const int* o = reinterpret_cast<const int*>(smem + NT * p.xstride + w * kGqRingBytes);
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[t][j] += o[(t * 4 + j) * 32 + lane];
  }
  const int row = row0 + lane;
  if (row < pr.M) {
    const float alpha = *pr.alpha;
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const int a = acc[t][0] + (acc[t][1] >> 2) + (acc[t][2] >> 4) + (acc[t][3] >> 6) -
                    s_xsum[t];
      const float scale = __fmul_rn(alpha, s_a127[t]);
      const int64_t o = static_cast<int64_t>(t) * pr.M + row;
      pr.y[o] = __fmul_rn(__int2float_rn(a), scale);
      if (pr.acc) pr.acc[o] = a;
    }
  }
}

}  // namespace bl
