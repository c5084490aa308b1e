// tl2.cuh -- TL2-style weight storage at 5/3 bits per weight, and the decode
// GEMV that reads it.
//
// The reading notes ("Bitnet.cpp" dual-mode reading report, section 2.3
// "technical details") store three ternary weights in 5 bits: a 1-bit sign
// and a 4-bit index, after folding each of the 27 combinations onto its mirror
// image, and split K into a part stored in threes and a remainder.  This
// project's layout (one row of TL2 bytes per weight row, 16-byte aligned):
//   index plane  16 bytes per block of 96 weights; group g (weights 3g..3g+2
//                of the block) has its index in byte g/2, low nibble for even g
//   sign plane   one little-endian uint32 per block (bit g), padded to 16 B
//   remainder    the last K % 96 weights in the 2-bit layout of pack.cuh
// For a group with v = 9(c0+1) + 3(c1+1) + (c2+1): index |v - 13|, sign
// (v < 13).  Negating the codes of a group flips its sign only.
//
// Conversion: from the 2-bit rows (pack.cuh) with the same codes; one thread
// per block of 96 weights or per 16-byte unit of the remainder.
//
// GEMV (N <= 16 tokens): as gemv.cuh, one row per lane and units of 32 rows,
// with a per-warp ring of k-chunks of 4 blocks (384 weights: 64 index bytes
// and 16 sign bytes per row, plus the 384 int8 activations of every token).
// Per chunk the warp regroups the activations into words of three int8
// (q[3g], q[3g+1], q[3g+2], 0); per group each lane forms the 5-bit code
// (sign, index), reads the three signed codes from a 32-entry table in shared
// memory (distinct entries sit in distinct banks) and accumulates one signed
// dp4a per token.  The remainder is read straight from global memory at the
// end of the unit and handled like gemv.cuh's words (codes+1 against the
// activations, minus their sum).
#pragma once

#include "gemv.cuh"

namespace bl {

constexpr int kTl2Block = 96;            // weights per block (32 groups of 3)
constexpr int kTl2ChunkBlocks = 4;       // blocks per ring stage
constexpr int kTl2ChunkK = kTl2Block * kTl2ChunkBlocks;   // 384
constexpr int kTl2Warps = 4;
constexpr int kTl2Threads = kTl2Warps * 32;
constexpr int kTl2Stages = 4;            // power of two
constexpr int kTl2MaxProblems = 256;

__host__ __device__ constexpr int64_t tl2_blocks(int64_t K) { return K / kTl2Block; }
__host__ __device__ constexpr int64_t tl2_sign_offset(int64_t K) { return 16 * tl2_blocks(K); }
__host__ __device__ constexpr int64_t tl2_tail_offset(int64_t K) {
  return tl2_sign_offset(K) + 16 * ((tl2_blocks(K) + 3) / 4);
}
__host__ __device__ constexpr int64_t tl2_row_bytes(int64_t K) {
  return tl2_tail_offset(K) + 16 * ((K - kTl2Block * tl2_blocks(K) + 63) / 64);
}

// ---------------------------------------------------------------- conversion

// Field of weight k in a 2-bit row (pack.cuh layout): code + 1.
__device__ __forceinline__ int i2_field(const uint32_t* row, int64_t k) {
  return (row[k >> 4] >> (8 * (k & 3) + 2 * ((k & 15) >> 2))) & 3;
}

static __global__ void __launch_bounds__(256)
tl2_convert_kernel(const uint32_t* __restrict__ packed, int64_t rows, int64_t K, int wp,
                   uint8_t* __restrict__ out) {
  const int64_t nb = tl2_blocks(K);
  const int64_t k3 = kTl2Block * nb, k2 = K - k3;
  const int64_t tail_units = (k2 + 63) / 64;
  const int64_t per_row = nb + tail_units;
  const int64_t rb = tl2_row_bytes(K);
  const int64_t total = rows * per_row;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t it = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; it < total;
       it += stride) {
    const int64_t m = it / per_row;
    const int64_t u = it - m * per_row;
    const uint32_t* src = packed + m * wp;
    uint8_t* row = out + m * rb;
    if (u < nb) {
      uint32_t idx[4] = {0u, 0u, 0u, 0u};
      uint32_t signs = 0u;
      for (int g = 0; g < 32; ++g) {
        const int64_t k = kTl2Block * u + 3 * g;
        const int v = 9 * i2_field(src, k) + 3 * i2_field(src, k + 1) + i2_field(src, k + 2);
        const int s = v < 13;
        const int i = s ? 13 - v : v - 13;
        idx[g >> 3] |= static_cast<uint32_t>(i) << (4 * (g & 7));
        signs |= static_cast<uint32_t>(s) << g;
      }
      *reinterpret_cast<uint4*>(row + 16 * u) = make_uint4(idx[0], idx[1], idx[2], idx[3]);
      uint32_t* sp = reinterpret_cast<uint32_t*>(row + tl2_sign_offset(K));
      sp[u] = signs;
      if (u == nb - 1)   // zero the sign plane's padding words
        for (int64_t w = nb; w < 4 * ((nb + 3) / 4); ++w) sp[w] = 0u;
    } else {
      // a 16-byte unit of the remainder: the 2-bit words, code-0 padding past K
      const int64_t t = u - nb;
      uint32_t w4[4];
      for (int j = 0; j < 4; ++j) {
        uint32_t word = 0x55555555u;
        for (int i = 0; i < 16; ++i) {
          const int64_t j2 = 64 * t + 16 * j + i;
          if (j2 >= k2) break;
          const int bit = 8 * (j2 & 3) + 2 * ((j2 & 15) >> 2);
          word = (word & ~(3u << bit)) | (static_cast<uint32_t>(i2_field(src, k3 + j2)) << bit);
        }
        w4[j] = word;
      }
      *reinterpret_cast<uint4*>(row + tl2_tail_offset(K) + 16 * t) =
          make_uint4(w4[0], w4[1], w4[2], w4[3]);
    }
  }
}

// ---------------------------------------------------------------------- GEMV

struct Tl2Problem {
  const uint8_t* tl2;      // [M][row_bytes]
  const float* alpha;
  const int8_t* xq;        // [NT][K]
  const float* amax;
  float* y;
  int32_t* acc;
  int M, K;
  int nb;                  // blocks of 96
  int row_bytes, sign_off, tail_off;
  int unit_begin;
};

struct Tl2Params {
  Tl2Problem prob[kTl2MaxProblems];
  int num_problems;
  int total_units;
};

template <int NT>
struct Tl2Cfg {
  static constexpr int kIdxBytes = kGemvTileRows * 16 * kTl2ChunkBlocks;   // 2 KB
  static constexpr int kSignBytes = kGemvTileRows * 16;                    // 512 B
  static constexpr int kStageBytes = kIdxBytes + kSignBytes + NT * kTl2ChunkK;
  static constexpr int kGroupBytes = NT * 4 * (kTl2ChunkK / 3);            // regrouped x
  static constexpr int kWarpBytes = kTl2Stages * kStageBytes + kGroupBytes;
  static constexpr int kSmemBytes = kTl2Warps * kWarpBytes;
};

__device__ __forceinline__ int dp4a_ss(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.s32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__device__ __forceinline__ int tl2_locate(const Tl2Params& p, int unit) {
  int lo = 0, hi = p.num_problems - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.prob[mid].unit_begin <= unit) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Copies of chunk kc of the unit whose first row is row0: each lane moves 4
// index pieces (rows lane/4 + 8i, piece lane%4), the sign piece of row lane,
// and up to 24 activation pieces per token.  Index piece c of row r goes to
// slot c ^ ((r >> 1) & 3), so 8 consecutive lanes reading one block hit
// distinct banks.
template <int NT>
__device__ __forceinline__ void tl2_issue(const Tl2Problem& pr, int row0, int kc, uint8_t* st,
                                          int lane) {
  using C = Tl2Cfg<NT>;
  const int piece = lane & 3;
  const int blk = kc * kTl2ChunkBlocks + piece;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = (lane >> 2) + 8 * i;
    if (row0 + r < pr.M && blk < pr.nb)
      cp_async16(st + r * 64 + ((piece ^ ((r >> 1) & 3)) << 4),
                 pr.tl2 + static_cast<int64_t>(row0 + r) * pr.row_bytes + 16 * blk, 16u);
  }
  if (row0 + lane < pr.M)
    cp_async16(st + C::kIdxBytes + lane * 16,
               pr.tl2 + static_cast<int64_t>(row0 + lane) * pr.row_bytes + pr.sign_off + 16 * kc,
               16u);
  if (lane < kTl2ChunkK / 16) {
    const int k = kc * kTl2ChunkK + lane * 16;
    const bool ok = k < kTl2Block * pr.nb;
#pragma unroll
    for (int t = 0; t < NT; ++t)
      cp_async16(st + C::kIdxBytes + C::kSignBytes + t * kTl2ChunkK + lane * 16,
                 ok ? pr.xq + static_cast<int64_t>(t) * pr.K + k : pr.xq, ok ? 16u : 0u);
  }
}

template <int NT>
__global__ void __launch_bounds__(kTl2Threads)
gemv_tl2_kernel(const __grid_constant__ Tl2Params p) {
  using C = Tl2Cfg<NT>;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint32_t lut[32];
  pdl_wait_prior_grid();
  pdl_allow_next_grid();
  if (threadIdx.x < 32) {   // (sign, index) -> three signed bytes
    const int s = threadIdx.x >> 4, i = threadIdx.x & 15;
    uint32_t e = 0u;
    if (i <= 13) {
      const int v = s ? 13 - i : 13 + i;
      const int c0 = v / 9 - 1, c1 = (v / 3) % 3 - 1, c2 = v % 3 - 1;
      e = (static_cast<uint32_t>(c0) & 0xFFu) | ((static_cast<uint32_t>(c1) & 0xFFu) << 8) |
          ((static_cast<uint32_t>(c2) & 0xFFu) << 16);
    }
    lut[threadIdx.x] = e;
  }
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* ring = smem + warp * C::kWarpBytes;
  uint32_t* xg = reinterpret_cast<uint32_t*>(ring + kTl2Stages * C::kStageBytes);
  const int stride = gridDim.x * kTl2Warps;

  int iu = blockIdx.x * kTl2Warps + warp, ic = 0, inchunks = 0, irow0 = 0;
  Tl2Problem ipr;
  if (iu < p.total_units) {
    ipr = p.prob[tl2_locate(p, iu)];
    irow0 = (iu - ipr.unit_begin) * kGemvTileRows;
    inchunks = (ipr.nb + kTl2ChunkBlocks - 1) / kTl2ChunkBlocks;
  }
  int slot = 0;
  auto issue_next = [&]() {
    // units with no whole block (K < 96) have no chunks: skip them here
    while (iu < p.total_units && inchunks == 0) {
      iu += stride;
      if (iu < p.total_units) {
        ipr = p.prob[tl2_locate(p, iu)];
        irow0 = (iu - ipr.unit_begin) * kGemvTileRows;
        inchunks = (ipr.nb + kTl2ChunkBlocks - 1) / kTl2ChunkBlocks;
      }
    }
    if (iu < p.total_units) {
      tl2_issue<NT>(ipr, irow0, ic, ring + slot * C::kStageBytes, lane);
      if (++ic == inchunks) {
        ic = 0;
        iu += stride;
        if (iu < p.total_units) {
          ipr = p.prob[tl2_locate(p, iu)];
          irow0 = (iu - ipr.unit_begin) * kGemvTileRows;
          inchunks = (ipr.nb + kTl2ChunkBlocks - 1) / kTl2ChunkBlocks;
        }
      }
    }
    cp_async_commit();
    slot = (slot + 1) & (kTl2Stages - 1);
  };
#pragma unroll 1
  for (int s = 0; s < kTl2Stages - 1; ++s) issue_next();

  const uint32_t sw = static_cast<uint32_t>((lane >> 1) & 3);
  int cslot = 0;
  for (int cu = blockIdx.x * kTl2Warps + warp; cu < p.total_units; cu += stride) {
    const Tl2Problem pr = p.prob[tl2_locate(p, cu)];
    const int row0 = (cu - pr.unit_begin) * kGemvTileRows;
    const int nchunks = (pr.nb + kTl2ChunkBlocks - 1) / kTl2ChunkBlocks;
    int acc[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[t] = 0;

    for (int kc = 0; kc < nchunks; ++kc) {
      issue_next();
      cp_async_wait<kTl2Stages - 1>();
      __syncwarp();
      const uint8_t* st = ring + cslot * C::kStageBytes;
      cslot = (cslot + 1) & (kTl2Stages - 1);
      // regroup the chunk's activations: word g = (q[3g], q[3g+1], q[3g+2], 0)
      const uint32_t* x8 = reinterpret_cast<const uint32_t*>(st + C::kIdxBytes + C::kSignBytes);
#pragma unroll
      for (int t = 0; t < NT; ++t) {
#pragma unroll
        for (int i = 0; i < kTl2ChunkK / 3 / 32; ++i) {
          const int g = lane + 32 * i;
          const int b = 3 * g;
          const uint32_t lo = x8[t * (kTl2ChunkK / 4) + (b >> 2)];
          const uint32_t hi = x8[t * (kTl2ChunkK / 4) + (b >> 2) + 1];
          xg[t * (kTl2ChunkK / 3) + g] = __funnelshift_r(lo, hi, 8 * (b & 3)) & 0x00FFFFFFu;
        }
      }
      __syncwarp();
      const uint4 sg4 = *reinterpret_cast<const uint4*>(st + C::kIdxBytes + lane * 16);
      const uint32_t sgn[4] = {sg4.x, sg4.y, sg4.z, sg4.w};
      const int nblk = min(kTl2ChunkBlocks, pr.nb - kc * kTl2ChunkBlocks);
#pragma unroll
      for (int bi = 0; bi < kTl2ChunkBlocks; ++bi) {
        if (bi < nblk) {
          const uint4 iv = *reinterpret_cast<const uint4*>(st + lane * 64 +
                                                           ((static_cast<uint32_t>(bi) ^ sw) << 4));
          const uint32_t iw[4] = {iv.x, iv.y, iv.z, iv.w};
          const uint32_t s = sgn[bi];
#pragma unroll
          for (int w = 0; w < 4; ++w) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {   // groups 8w + 4h .. 8w + 4h + 3
              uint32_t e[4];
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const int g = 8 * w + 4 * h + q;
                const uint32_t code = ((iw[w] >> (4 * (4 * h + q))) & 15u) | (((s >> g) & 1u) << 4);
                e[q] = lut[code];
              }
#pragma unroll
              for (int t = 0; t < NT; ++t) {
                const uint4 xv = *reinterpret_cast<const uint4*>(
                    xg + t * (kTl2ChunkK / 3) + 32 * bi + 8 * w + 4 * h);
                acc[t] = dp4a_ss(e[0], xv.x, acc[t]);
                acc[t] = dp4a_ss(e[1], xv.y, acc[t]);
                acc[t] = dp4a_ss(e[2], xv.z, acc[t]);
                acc[t] = dp4a_ss(e[3], xv.w, acc[t]);
              }
            }
          }
        }
      }
      __syncwarp();   // stage and regrouped activations are read before they are refilled
    }

    const int row = row0 + lane;
    const int k3 = kTl2Block * pr.nb;
    if (pr.K > k3) {   // the remainder, straight from global memory
      const uint32_t* tw = reinterpret_cast<const uint32_t*>(
          pr.tl2 + static_cast<int64_t>(min(row, pr.M - 1)) * pr.row_bytes + pr.tail_off);
      for (int w = 0; w < (pr.K - k3) / 16; ++w) {
        const uint32_t word = __ldg(tw + w);
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const uint32_t* xr = reinterpret_cast<const uint32_t*>(
              pr.xq + static_cast<int64_t>(t) * pr.K + k3 + 16 * w);
          int a = 0, xs = 0;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t xv = __ldg(xr + j);
            a = dp4a_us((word >> (2 * j)) & 0x03030303u, xv, a);
            xs = dp4a_ss(0x01010101u, xv, xs);
          }
          acc[t] += a - xs;
        }
      }
    }
    if (row < pr.M) {
      const float alpha = *pr.alpha;
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        const float scale = __fmul_rn(alpha, __fdiv_rn(pr.amax[t], 127.0f));
        const int64_t o = static_cast<int64_t>(t) * pr.M + row;
        pr.y[o] = __fmul_rn(__int2float_rn(acc[t]), scale);
        if (pr.acc) pr.acc[o] = acc[t];
      }
    }
  }
  cp_async_wait<0>();
}

}  // namespace bl
