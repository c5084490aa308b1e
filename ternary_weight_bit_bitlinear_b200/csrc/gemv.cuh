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

// ---------------------------------------------------------------- generic
// Any N <= 16 and any K: each warp takes 4 rows; lanes stride over 16-byte
// chunks (64 weights) and read the matching activations through L1.

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
gemv_generic_kernel(const uint4* __restrict__ wq, int M, int cpr,      // cpr = K / 64 chunks per row
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

// ---------------------------------------------------------------- streaming
// N <= 4.  One launch covers a group of problems that share K (and N).  Work
// is cut into units of consecutive rows of one problem; since rows are stored
// back to back, a unit is one contiguous byte range, copied into a 4-stage
// shared-memory ring by one producer thread with bulk async copies.  Eight
// consumer warps read it: warp w owns k-slice (w % ksplit) -- every lane keeps
// the int8 activations of its 32-word-strided slice in registers for the whole
// unit -- and rows w / ksplit, + 8/ksplit, ...; a row's partial dot product is
// reduced over the warp, and with ksplit > 1 combined in shared memory.

constexpr int kStreamStages = 4;
constexpr int kStreamStageBytes = 16384;
constexpr int kStreamConsumerWarps = 8;
constexpr int kStreamThreads = (kStreamConsumerWarps + 1) * 32;
constexpr int kStreamMaxUnitRows = 1024;
constexpr int kStreamMaxTokens = 4;
constexpr int kStreamMaxProblems = 256;

struct GemvProblem {
  const uint32_t* packed;
  const float* alpha;
  const int8_t* xq;
  const float* amax;
  const int32_t* xsum;
  float* y;
  int32_t* acc;
  int M;
  int unit_begin;   // first unit of this problem
};

struct GemvParams {
  GemvProblem prob[kStreamMaxProblems];
  int num_problems;
  int total_units;
  int K, W;              // W = K / 16 words per row
  int rows_per_stage;    // RS
  int unit_rows;         // RS * stages per unit
  int ksplit;            // 1, 2, 4 or 8 k-slices
};

constexpr size_t stream_smem_bytes() {
  return kStreamStages * kStreamStageBytes + 2 * kStreamStages * sizeof(uint64_t) +
         kStreamMaxUnitRows * kStreamMaxTokens * sizeof(int) + 16;
}

__device__ __forceinline__ int stream_locate(const GemvParams& p, int unit) {
  int lo = 0, hi = p.num_problems - 1;
  while (lo < hi) {   // last problem whose unit_begin <= unit
    const int mid = (lo + hi + 1) >> 1;
    if (p.prob[mid].unit_begin <= unit) lo = mid; else hi = mid - 1;
  }
  return lo;
}

template <int NT, int S>
__global__ void __launch_bounds__(kStreamThreads, 2)
gemv_stream_kernel(const __grid_constant__ GemvParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint32_t* ring = reinterpret_cast<uint32_t*>(smem);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStreamStages * kStreamStageBytes);
  uint64_t* empty = full + kStreamStages;
  int* part = reinterpret_cast<int*>(empty + kStreamStages);
  __shared__ int abort_flag;
  volatile int* abort = &abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kStageWords = kStreamStageBytes / 4;
  const int W = p.W, RS = p.rows_per_stage, UR = p.unit_rows;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStreamStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kStreamConsumerWarps);
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kStreamConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t slot = 0, phase = 0;
      for (int u = blockIdx.x; u < p.total_units; u += gridDim.x) {
        const GemvProblem& pr = p.prob[stream_locate(p, u)];
        const int r0 = (u - pr.unit_begin) * UR;
        const int r1 = min(r0 + UR, pr.M);
        for (int rs = r0; rs < r1; rs += RS) {
          const int nrows = min(RS, r1 - rs);
          if (!mbar_wait(&empty[slot], phase ^ 1u, abort)) return;
          const uint32_t bytes = static_cast<uint32_t>(nrows) * W * 4u;
          mbar_arrive_expect_tx(&full[slot], bytes);
          bulk_load(ring + slot * kStageWords, pr.packed + static_cast<int64_t>(rs) * W, bytes,
                    &full[slot]);
          if (++slot == kStreamStages) { slot = 0; phase ^= 1u; }
        }
      }
    }
    return;
  }

  // ------------------------------------------------------------ consumers
  const int ks = p.ksplit;
  const int slice = warp % ks, group = warp / ks, groups = kStreamConsumerWarps / ks;
  const int word0 = slice * S * 32 + lane;   // this lane's first word within a row
  uint32_t slot = 0, phase = 0;
  int cur = -1;
  uint32_t xr[NT][S][4];
  float scale = 0.0f;   // lane t < NT: alpha * (amax_t / 127)
  int xs = 0;           // lane t < NT: sum of token t's activations

  for (int u = blockIdx.x; u < p.total_units; u += gridDim.x) {
    const int pi = stream_locate(p, u);
    const GemvProblem& pr = p.prob[pi];
    const int r0 = (u - pr.unit_begin) * UR;
    const int r1 = min(r0 + UR, pr.M);
    if (pi != cur) {
      cur = pi;
#pragma unroll
      for (int t = 0; t < NT; ++t) {
#pragma unroll
        for (int j = 0; j < S; ++j) {
          const int wi = word0 + 32 * j;
          uint4 v = make_uint4(0u, 0u, 0u, 0u);
          if (wi < W)
            v = __ldg(reinterpret_cast<const uint4*>(pr.xq + static_cast<int64_t>(t) * p.K) + wi);
          xr[t][j][0] = v.x;
          xr[t][j][1] = v.y;
          xr[t][j][2] = v.z;
          xr[t][j][3] = v.w;
        }
      }
      if (lane < NT) {
        scale = __fmul_rn(*pr.alpha, __fdiv_rn(pr.amax[lane], 127.0f));
        xs = pr.xsum[lane];
      }
    }
    if (ks > 1) {
      for (int i = threadIdx.x; i < (r1 - r0) * NT; i += kStreamConsumerWarps * 32) part[i] = 0;
      named_barrier(1, kStreamConsumerWarps * 32);
    }
    for (int rs = r0; rs < r1; rs += RS) {
      const int nrows = min(RS, r1 - rs);
      // On a timeout the stage is skipped but the loop (and its named
      // barriers) still runs to the end, so no warp is left waiting.
      const bool ready = mbar_wait(&full[slot], phase, abort);
      const uint32_t* st = ring + slot * kStageWords;
      for (int i = group; ready && i < nrows; i += groups) {
        int acc[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) acc[t] = 0;
        const uint32_t* row = st + i * W;
#pragma unroll
        for (int j = 0; j < S; ++j) {
          const int wi = word0 + 32 * j;
          if (wi < W) {
            const uint32_t w = row[wi];
            const uint32_t q0 = w & 0x03030303u, q1 = (w >> 2) & 0x03030303u,
                           q2 = (w >> 4) & 0x03030303u, q3 = (w >> 6) & 0x03030303u;
#pragma unroll
            for (int t = 0; t < NT; ++t) {
              acc[t] = __dp4a(static_cast<int>(q0), static_cast<int>(xr[t][j][0]), acc[t]);
              acc[t] = __dp4a(static_cast<int>(q1), static_cast<int>(xr[t][j][1]), acc[t]);
              acc[t] = __dp4a(static_cast<int>(q2), static_cast<int>(xr[t][j][2]), acc[t]);
              acc[t] = __dp4a(static_cast<int>(q3), static_cast<int>(xr[t][j][3]), acc[t]);
            }
          }
        }
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) acc[t] += __shfl_xor_sync(0xFFFFFFFFu, acc[t], o);
        int mine = acc[0];
#pragma unroll
        for (int t = 1; t < NT; ++t)
          if (lane == t) mine = acc[t];
        if (lane < NT) {
          const int row_idx = rs + i;
          if (ks == 1) {
            const int a = mine - xs;
            const int64_t o = static_cast<int64_t>(lane) * pr.M + row_idx;
            pr.y[o] = __fmul_rn(__int2float_rn(a), scale);
            if (pr.acc) pr.acc[o] = a;
          } else {
            atomicAdd(&part[(row_idx - r0) * NT + lane], mine);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
      if (++slot == kStreamStages) { slot = 0; phase ^= 1u; }
    }
    if (ks > 1) {
      named_barrier(1, kStreamConsumerWarps * 32);
      const float alpha = *pr.alpha;
      for (int i = threadIdx.x; i < (r1 - r0) * NT; i += kStreamConsumerWarps * 32) {
        const int t = i % NT, row_idx = r0 + i / NT;
        const int a = part[i] - pr.xsum[t];
        const float sc = __fmul_rn(alpha, __fdiv_rn(pr.amax[t], 127.0f));
        const int64_t o = static_cast<int64_t>(t) * pr.M + row_idx;
        pr.y[o] = __fmul_rn(__int2float_rn(a), sc);
        if (pr.acc) pr.acc[o] = a;
      }
      named_barrier(1, kStreamConsumerWarps * 32);
    }
  }
}

}  // namespace bl
