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
// continuing from one unit into the next without draining,
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
  static constexpr int kStages = NT <= 4 ? 4 : 2;   // powers of two: the ring index is a mask
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

// Per-lane copy plan of one unit, fixed for all its k-chunks.  Lane l copies
// the 16-byte chunk (l % 8) of rows row0 + 4i + l/8, i = 0..7.
struct GemvCopyPlan {
  const uint8_t* wsrc;     // chunk (l % 8) of row row0 + l/8 at k-chunk 0
  int64_t wstep;           // bytes from one of this lane's rows to the next (4 rows)
  uint32_t dst_even;       // stage offset of copy i = 0 (even i add i * 512)
  uint32_t dst_odd;        // stage offset of copy i = 1 minus 512 (odd i add (i-1) * 512)
  int vrows;               // copies i < vrows have a row inside the layer
  int wword;               // word index of this lane's chunk within a k-chunk
};

template <class Problem>   // any problem type with packed, M and W
__device__ __forceinline__ GemvCopyPlan gemv_plan(const Problem& pr, int row0, int lane) {
  GemvCopyPlan cp;
  const int rr = lane >> 3, c = lane & 7;
  cp.wsrc = reinterpret_cast<const uint8_t*>(pr.packed) +
            static_cast<int64_t>(row0 + rr) * pr.W * 4 + c * 16;
  cp.wstep = static_cast<int64_t>(pr.W) * 16;
  cp.dst_even = rr * kGemvChunkBytes + ((c ^ rr) << 4);
  cp.dst_odd = 512 + rr * kGemvChunkBytes + ((c ^ (rr + 4)) << 4);
  cp.vrows = max(0, min(8, (pr.M - row0 - rr + 3) / 4));
  cp.wword = 4 * c;
  return cp;
}

// Issue the weight copies of k-chunk `kc` (W words per row) into stage buffer
// `st`.  Weight chunks outside the layer are skipped (rows past M are never
// stored; past the last word, the activations are zero, so stale bytes
// multiply zeros).  Each copy asks L2 for the aligned 256 bytes around it, so
// the row's next k-chunk is already on its way when its stage is issued.
__device__ __forceinline__ void gemv_issue_weights(int W, const GemvCopyPlan& cp, int kc,
                                                   uint8_t* st) {
  if (kc * (kGemvChunkBytes / 4) + cp.wword < W) {
    const uint8_t* src = cp.wsrc + kc * kGemvChunkBytes;
#pragma unroll
    for (int i = 0; i < kGemvTileRows / 4; ++i) {
      if (i < cp.vrows)
        cp_async16_l2_256(st + ((i & 1) ? cp.dst_odd + (i - 1) * 512 : cp.dst_even + i * 512),
                          src);
      src += cp.wstep;
    }
  }
}

// Weights and int8 activations of k-chunk `kc` into stage buffer `st`.
template <int NT>
__device__ __forceinline__ void gemv_issue(const GemvProblem& pr, const GemvCopyPlan& cp, int kc,
                                           uint8_t* st, int lane) {
  gemv_issue_weights(pr.W, cp, kc, st);
  // activations: 512 bytes per token, 16 per lane, zero-filled past K
  const int k0 = kc * kGemvChunkK + lane * 16;
  const bool xval = k0 < pr.K;
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    const int8_t* src = xval ? pr.xq + static_cast<int64_t>(t) * pr.K + k0 : pr.xq;
    cp_async16(st + GemvCfg<NT>::kWeightBytes + t * kGemvChunkK + lane * 16, src,
               xval ? 16u : 0u);
  }
}

// One k-chunk of this lane's row against every token: `wrow` is the row's
// 128 swizzled bytes in a stage, `xs` the chunk's 512 int8 activations of
// token 0 (token t at xs + t * xstride), read as broadcasts.
template <int NT>
__device__ __forceinline__ void gemv_chunk_dot(const uint8_t* wrow, uint32_t sw, const uint8_t* xs,
                                               int xstride, int (&acc)[NT][4]) {
#pragma unroll
  for (int c = 0; c < kGemvChunkBytes / 16; ++c) {
    const uint4 w = *reinterpret_cast<const uint4*>(wrow + ((static_cast<uint32_t>(c) ^ sw) << 4));
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const uint4* xp = reinterpret_cast<const uint4*>(xs + t * xstride + c * 64);
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
}

template <int NT>
__global__ void __launch_bounds__(kGemvThreads)
gemv_tile_kernel(const __grid_constant__ GemvParams p) {
  using C = GemvCfg<NT>;
  extern __shared__ __align__(128) uint8_t smem[];
  pdl_wait_prior_grid();
  pdl_allow_next_grid();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* ring = smem + warp * C::kWarpBytes;
  const int stride = gridDim.x * kGemvWarps;
  const uint32_t sw = static_cast<uint32_t>(lane & 7);

  // The copy side runs ahead of the compute side through this warp's whole
  // sequence of (unit, k-chunk) pairs, across unit boundaries, so the ring
  // stays full from the first unit to the last.
  int iu = blockIdx.x * kGemvWarps + warp;   // unit and chunk to issue next
  int ic = 0;
  GemvProblem ipr;
  GemvCopyPlan icp;
  int inchunks = 0;
  if (iu < p.total_units) {
    ipr = p.prob[gemv_locate(p, iu)];
    icp = gemv_plan(ipr, (iu - ipr.unit_begin) * kGemvTileRows, lane);
    inchunks = (ipr.K + kGemvChunkK - 1) / kGemvChunkK;
  }
  int slot = 0;
  auto issue_next = [&]() {
    if (iu < p.total_units) {
      gemv_issue<NT>(ipr, icp, ic, ring + slot * C::kStageBytes, lane);
      if (++ic == inchunks) {
        ic = 0;
        iu += stride;
        if (iu < p.total_units) {
          ipr = p.prob[gemv_locate(p, iu)];
          icp = gemv_plan(ipr, (iu - ipr.unit_begin) * kGemvTileRows, lane);
          inchunks = (ipr.K + kGemvChunkK - 1) / kGemvChunkK;
        }
      }
    }
    cp_async_commit();   // one group per stage, empty once the sequence is done
    slot = (slot + 1) & (C::kStages - 1);
  };
#pragma unroll 1
  for (int s = 0; s < C::kStages - 1; ++s) issue_next();

  int cslot = 0;
  for (int cu = blockIdx.x * kGemvWarps + warp; cu < p.total_units; cu += stride) {
    // by value: registers, not re-read from parameter space after each store
    const GemvProblem pr = p.prob[gemv_locate(p, cu)];
    const int row0 = (cu - pr.unit_begin) * kGemvTileRows;
    const int nchunks = (pr.K + kGemvChunkK - 1) / kGemvChunkK;

    int acc[NT][4];
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[t][j] = 0;

    for (int kc = 0; kc < nchunks; ++kc) {
      issue_next();
      cp_async_wait<C::kStages - 1>();
      __syncwarp();
      const uint8_t* st = ring + cslot * C::kStageBytes;
      cslot = (cslot + 1) & (C::kStages - 1);
      gemv_chunk_dot<NT>(st + lane * kGemvChunkBytes, sw, st + C::kWeightBytes, kGemvChunkK, acc);
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
