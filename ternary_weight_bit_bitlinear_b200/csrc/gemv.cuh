// gemv.cuh -- decode mpGEMM for a few tokens (N <= 16) on the CUDA cores.
//
// The reading notes' I2_S kernel is MAD-based: int8 multiply-adds of
// activations against ternary weights ("Bitnet.cpp" reading notes, section 4.1
// item 3); the FairyFuse "fused kernel design" unpacks the bit-packed codes and
// accumulates in the same loop, with no intermediate writes.
//
// Work unit: 32 consecutive rows of one layer, one row per lane, all of its K
// (layers of one launch may differ in K).
// Each warp runs its own pipeline of k-chunks (512 weights = 128 bytes per row,
// plus the matching 512 int8 activations of every token), brought in with
// 16-byte cp.async copies into a STAGES-deep ring in shared memory.  A row's
// 16-byte chunks are stored XOR-swizzled by row (chunk c of row r at c ^ r%8),
// so the per-lane 16-byte reads of 8 consecutive lanes hit all 32 banks once.
// Activations are read as broadcasts (every lane wants the same k).
//
// Arithmetic per 32-bit packed word (16 weights): byte lane b of field j
// (bits 2j..2j+1) holds code+1 of weight 4j+b, so
//   w & (0x03030303 << 2j)  =  4^j * (codes+1 of weights 4j..4j+3, one per byte)
// and one dp4a (unsigned bytes x signed int8) against activations 4j..4j+3
// accumulates 4^j times their dot product.  Four accumulators, one per j, are
// combined exactly at the end (acc_j is a multiple of 4^j), and the +1 offset
// is removed with the token's activation sum: acc = sum - xsum.  No shifts in
// the inner loop and no cross-lane reduction at all.
#pragma once

#include "ptx.cuh"

namespace bl {

constexpr int kGemvTileRows = 32;        // rows per unit: one per lane
constexpr int kGemvChunkBytes = 128;     // packed bytes per row per k-chunk (512 weights)
constexpr int kGemvChunkK = 512;
constexpr int kGemvWarps = 4;            // warps per CTA
constexpr int kGemvThreads = kGemvWarps * 32;
constexpr int kGemvMaxTokens = 16;
constexpr int kGemvMaxProblems = 256;

template <int NT>
struct GemvCfg {
  static constexpr int kStages = NT <= 4 ? 4 : (NT <= 8 ? 3 : 2);
  static constexpr int kWeightBytes = kGemvTileRows * kGemvChunkBytes;    // 4 KB
  static constexpr int kStageBytes = kWeightBytes + NT * kGemvChunkK;
  static constexpr int kWarpBytes = kStages * kStageBytes;
  static constexpr int kSmemBytes = kGemvWarps * kWarpBytes;
};

struct GemvProblem {
  const uint32_t* packed;
  const float* alpha;
  const int8_t* xq;
  const float* amax;
  const int32_t* xsum;
  float* y;
  int32_t* acc;
  int M, K, W;      // W = K / 16 words per row
  int unit_begin;   // first unit of this problem
};

struct GemvParams {
  GemvProblem prob[kGemvMaxProblems];
  int num_problems;
  int total_units;
};

__device__ __forceinline__ int gemv_locate(const GemvParams& p, int unit) {
  int lo = 0, hi = p.num_problems - 1;
  while (lo < hi) {   // last problem whose unit_begin <= unit
    const int mid = (lo + hi + 1) >> 1;
    if (p.prob[mid].unit_begin <= unit) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Issue the copies of k-chunk `kc` of the unit starting at row0 into `st`.
template <int NT>
__device__ __forceinline__ void gemv_issue(const GemvProblem& pr, int row0, int kc, uint8_t* st,
                                           int lane) {
  // weights: 32 rows x 8 sixteen-byte chunks; a warp instruction copies 4
  // whole 128-byte row segments (coalesced)
  const int c = lane & 7;
  const int word = kc * (kGemvChunkBytes / 4) + c * 4;
  const bool kval = word < pr.W;
#pragma unroll
  for (int i = 0; i < kGemvTileRows / 4; ++i) {
    const int r = i * 4 + (lane >> 3);
    const int row = row0 + r;
    const bool ok = kval && row < pr.M;
    const uint32_t* src = ok ? pr.packed + static_cast<int64_t>(row) * pr.W + word : pr.packed;
    cp_async16(st + r * kGemvChunkBytes + ((c ^ (r & 7)) << 4), src, ok ? 16u : 0u);
  }
  // activations: 512 bytes per token, 16 per lane
  const int k0 = kc * kGemvChunkK + lane * 16;
  const bool xval = k0 < pr.K;
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    const int8_t* src = xval ? pr.xq + static_cast<int64_t>(t) * pr.K + k0 : pr.xq;
    cp_async16(st + GemvCfg<NT>::kWeightBytes + t * kGemvChunkK + lane * 16, src,
               xval ? 16u : 0u);
  }
}

template <int NT>
__global__ void __launch_bounds__(kGemvThreads)
gemv_tile_kernel(const __grid_constant__ GemvParams p) {
  using C = GemvCfg<NT>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* ring = smem + warp * C::kWarpBytes;
  const int total_warps = gridDim.x * kGemvWarps;
  const uint32_t sw = static_cast<uint32_t>(lane & 7);

  for (int u = blockIdx.x * kGemvWarps + warp; u < p.total_units; u += total_warps) {
    const GemvProblem& pr = p.prob[gemv_locate(p, u)];
    const int row0 = (u - pr.unit_begin) * kGemvTileRows;
    const int nchunks = (pr.K + kGemvChunkK - 1) / kGemvChunkK;

    int acc[NT][4];
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[t][j] = 0;

#pragma unroll
    for (int s = 0; s < C::kStages - 1; ++s) {
      if (s < nchunks) gemv_issue<NT>(pr, row0, s, ring + s * C::kStageBytes, lane);
      cp_async_commit();
    }
    for (int kc = 0; kc < nchunks; ++kc) {
      const int nxt = kc + C::kStages - 1;
      if (nxt < nchunks)
        gemv_issue<NT>(pr, row0, nxt, ring + (nxt % C::kStages) * C::kStageBytes, lane);
      cp_async_commit();
      cp_async_wait<C::kStages - 1>();
      __syncwarp();
      const uint8_t* st = ring + (kc % C::kStages) * C::kStageBytes;
      const uint8_t* wrow = st + lane * kGemvChunkBytes;
      const uint8_t* xs = st + C::kWeightBytes;
#pragma unroll
      for (int c = 0; c < kGemvChunkBytes / 16; ++c) {
        const uint4 w = *reinterpret_cast<const uint4*>(wrow + ((static_cast<uint32_t>(c) ^ sw) << 4));
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const uint4* xp = reinterpret_cast<const uint4*>(xs + t * kGemvChunkK + c * 64);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint4 xa = xp[i];
            acc[t][0] = dp4a_us(ws[i] & 0x03030303u, xa.x, acc[t][0]);
            acc[t][1] = dp4a_us(ws[i] & 0x0C0C0C0Cu, xa.y, acc[t][1]);
            acc[t][2] = dp4a_us(ws[i] & 0x30303030u, xa.z, acc[t][2]);
            acc[t][3] = dp4a_us(ws[i] & 0xC0C0C0C0u, xa.w, acc[t][3]);
          }
        }
      }
      __syncwarp();   // every lane is done with this stage before it is refilled
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
  cp_async_wait<0>();
}

}  // namespace bl
