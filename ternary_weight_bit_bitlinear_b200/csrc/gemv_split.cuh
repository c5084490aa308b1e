// gemv_split.cuh -- the decode GEMV of gemv.cuh for launches too small to fill
// the GPU with one unit per warp.
#pragma once

#include "gemv.cuh"

namespace bl {

// For launches with fewer units than gemv_tile_kernel has warps resident (one
// layer, or one input group of a layer, per launch), each of its warps would
// walk all k-chunks of its single unit alone.  Here one CTA of kGemvWarps
// warps takes one unit: warp w streams k-chunks [C w / 4, C (w + 1) / 4) of
// its C through its own ring (same layout, copies and arithmetic), the other
// warps leave their int32 sums in their rings, and warp 0 adds them (integers:
// the order does not matter) and writes y as gemv_tile_kernel does.
template <int NT>
__global__ void __launch_bounds__(kGemvThreads)
gemv_split_kernel(const __grid_constant__ GemvParams p) {
  using C = GemvCfg<NT>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* ring = smem + warp * C::kWarpBytes;
  const uint32_t sw = static_cast<uint32_t>(lane & 7);
  const int unit = blockIdx.x;
  const GemvProblem pr = p.prob[gemv_locate(p, unit)];
  const int row0 = (unit - pr.unit_begin) * kGemvTileRows;
  const int nchunks = (pr.K + kGemvChunkK - 1) / kGemvChunkK;
  const int kc0 = nchunks * warp / kGemvWarps, kc1 = nchunks * (warp + 1) / kGemvWarps;
  const GemvCopyPlan cp = gemv_plan(pr, row0, lane);

  // The weights of this warp's first k-chunks go to L2 before the wait on
  // the preceding kernel (a hint: nothing is read before the wait).
#pragma unroll 1
  for (int kc = kc0; kc < kc1 && kc < kc0 + 8; ++kc) {
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
    if (ic < kc1) gemv_issue<NT>(pr, cp, ic++, ring + slot * C::kStageBytes, lane);
    cp_async_commit();   // one group per stage, empty past this warp's chunks
    slot = (slot + 1) & (C::kStages - 1);
  };
#pragma unroll 1
  for (int s = 0; s < C::kStages - 1; ++s) issue_next();

  int acc[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[t][j] = 0;
  int cslot = 0;
  for (int kc = kc0; kc < kc1; ++kc) {
    issue_next();
    cp_async_wait<C::kStages - 1>();
    __syncwarp();
    const uint8_t* st = ring + cslot * C::kStageBytes;
    cslot = (cslot + 1) & (C::kStages - 1);
    gemv_chunk_dot<NT>(st + lane * kGemvChunkBytes, sw, st + C::kWeightBytes, kGemvChunkK, acc);
    __syncwarp();   // every lane is done with this stage before it is refilled
  }
  cp_async_wait<0>();
  __syncwarp();

  int* red = reinterpret_cast<int*>(ring);   // [NT][4][32], within this warp's ring
  if (warp > 0) {
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
      for (int j = 0; j < 4; ++j) red[(t * 4 + j) * 32 + lane] = acc[t][j];
  }
  __syncthreads();
  if (warp != 0) return;
#pragma unroll 1
  for (int w = 1; w < kGemvWarps; ++w) {
    const int* o = reinterpret_cast<const int*>(smem + w * C::kWarpBytes);
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
                    pr.xsum[t];
      const float scale = __fmul_rn(alpha, __fdiv_rn(pr.amax[t], 127.0f));
      const int64_t o = static_cast<int64_t>(t) * pr.M + row;
      pr.y[o] = __fmul_rn(__int2float_rn(a), scale);
      if (pr.acc) pr.acc[o] = a;
    }
  }
}

}  // namespace bl
