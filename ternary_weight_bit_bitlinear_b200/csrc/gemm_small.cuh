// gemm_small.cuh -- the ternary x int8 product for a few tokens (N <= 32) on
// the 5th-generation tensor cores, at the rate the weights stream from HBM.
//
// With few tokens the MMAs are short and the work is moving the packed
// weights (2 bits each) and expanding them to int8 codes.  The reading notes'
// I2_S kernel is MAD-based (section 4.1 item 3): int8 multiply-adds of the
// activations against the ternary codes; here the multiply-adds are
// tcgen05.mma kind::i8 with the weights as the M = 128 side (one 128-row block
// per tile) and the tokens as N (16 or 32, zero past N).  What differs from
// the prefill GEMM of gemm.cuh is where the expanded weights live: the unpack
// warps write them from registers straight into tensor memory (tcgen05.st),
// and the MMAs read A from there, so no expanded tile is written to or read
// from shared memory.
//
// Measured on B200 and built in:
//   * a tcgen05.mma of M = 128, N = 16, K = 32 keeps the tensor pipe busy
//     for ~10 cycles when a whole warp runs the issue loop and an elected
//     lane issues; a loop run by one lane alone took ~50 cycles per MMA, and
//     ~85 with ALU-bound warps on its SM sub-partition (the unpack warps
//     share it: a warp's tensor-memory lane quarter is fixed by its index);
//     descriptors are built once per stage and the 16 MMAs of a k-group are
//     unrolled with immediate offsets;
//   * DRAM serves 256 contiguous bytes of a row better than 128: a ring stage
//     holds two k-groups (2 x 128 bytes of each of the 128 rows).
//
//   warp 0        TMA producer (an elected lane issues): per stage two boxes of 128 weight rows x 128
//                 packed bytes (128-byte swizzle, one per k-group) and the
//                 stage's activation tiles (BN x 128 int8 per k-block);
//   warps 4-11    unpackers, two groups of four; group g expands k-group g of
//                 every stage.  Warp w owns tensor-memory lanes 32 (w % 4) ..
//                 +31, one weight row per lane: it reads its row's 128 packed
//                 bytes, expands each k-block's 32 bytes to 32 words of codes+1
//                 (four int8 per word, in k order), stores them with one
//                 tcgen05.st per k-block into the k-group's A slot (128
//                 columns), waits once, and hands the slot to the MMA;
//   warp 1        MMA issue warp (an elected lane issues): per k-group 16 x
//                 tcgen05.mma kind::i8 (K = 32),
//                 A from tensor memory, B from the ring, one accumulator per
//                 tile (double-buffered across tiles); a commit per k-group
//                 frees its A slot, one per stage frees the ring stage (the
//                 unpackers have read the packed bytes before they hand over
//                 the slot, so the MMA's completion implies theirs);
//   warps 2,3,12,13  epilogue, one per lane quarter: tcgen05.ld of BN
//                 columns, subtract the token's sum of q (the +1 code offset),
//                 rescale by alpha * amax / 127, store y (lane = row: coalesced).
//
// Tiles (one per 128-row block of every problem of the launch) are spread
// over persistent CTAs by the host's longest-first schedule, as in gemm.cuh.
// Every wait is bounded (GemmParams::wait_ns), and the CTA drains the copies
// and MMAs it has issued before it releases tensor memory.
#pragma once

#include "gemm.cuh"

namespace bl {

constexpr int kSmallUnpackGroups = 2;                              // = k-groups per stage
constexpr int kSmallThreads = (6 + 4 * kSmallUnpackGroups) * 32;   // 14 warps
constexpr int kSmallGroupKb = 4;                                   // k-blocks per k-group
constexpr int kSmallGroupBytes = kSmallGroupKb * kGemmPackedRowBytes;   // 128 per row
constexpr int kSmallStageKb = kSmallUnpackGroups * kSmallGroupKb;  // k-blocks per stage
constexpr uint32_t kSmallTmemCols = 512;
constexpr int kSmallSlotCols = 32 * kSmallGroupKb;                 // one k-group of A
// Tensor memory: two accumulators of BN columns, then the A slots.
__host__ __device__ constexpr int small_acol_base(int bn) { return 2 * bn; }
__host__ __device__ constexpr int small_aslots(int bn) {
  return (static_cast<int>(kSmallTmemCols) - small_acol_base(bn)) / kSmallSlotCols;
}
__host__ __device__ constexpr int small_stages(int bn) { return bn <= 16 ? 4 : 3; }

template <int BN>
struct SmallSmem {
  static constexpr int S = small_stages(BN);
  // each array up to the barriers is a multiple of 1024 bytes
  uint8_t apk[S][kSmallUnpackGroups][kGemmBM * kSmallGroupBytes];   // packed, swizzled
  uint8_t b[S][kSmallStageKb][BN * kGemmBK];                         // 128-byte swizzle
  uint64_t full[S];
  uint64_t empty[S];                      // MMA commit
  uint64_t afull[small_aslots(BN)];       // 4 unpack warps
  uint64_t aempty[small_aslots(BN)];      // MMA commit
  uint64_t tfull[2];
  uint64_t tempty[2];                     // 4 epilogue warps
  uint64_t drain;
  uint32_t tmem_slot;
  int abort;
};
static_assert(small_aslots(16) == 3 && small_aslots(32) == 3, "three A slots");
static_assert(sizeof(SmallSmem<16>) + 1024 <= 232448, "shared memory");
static_assert(sizeof(SmallSmem<32>) + 1024 <= 232448, "shared memory");

// Ring position of a k-group: its stage's k-groups get consecutive sequence
// numbers, and sequence number q uses A slot q % kSlots.
struct SmallSlot {
  uint32_t slot = 0, phase = 0;
  template <int kSlots>
  __device__ __forceinline__ void advance() {
    if (++slot == kSlots) { slot = 0; phase ^= 1u; }
  }
};

template <int BN>
__global__ void __launch_bounds__(kSmallThreads, 1)
gemm_small_kernel(const __grid_constant__ GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  using Smem = SmallSmem<BN>;
  constexpr int S = Smem::S;
  constexpr int kSlots = small_aslots(BN);
  constexpr uint32_t kAColBase = small_acol_base(BN);
  const uint32_t base = smem_u32(smem_raw);
  Smem& s = *reinterpret_cast<Smem*>(smem_raw + ((1024u - (base & 1023u)) & 1023u));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile int* abort = &s.abort;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(&s.afull[i], 4);
      mbar_init(&s.aempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.tfull[i], 1);
      mbar_init(&s.tempty[i], 4);
    }
    mbar_init(&s.drain, 1);
    s.abort = 0;
    fence_mbar_init();
    for (int i = 0; i < p.num_problems; ++i) {
      tma_prefetch_desc(&p.tmA[i]);
      tma_prefetch_desc(&p.tmB[i]);
    }
  }
  if (warp == 1) {
    tmem_alloc(&s.tmem_slot, kSmallTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // The set-up above (barriers, tensor-map prefetch, tensor memory) touches
  // nothing the preceding kernel writes, so it overlaps that kernel's tail.
  pdl_wait_prior_grid();
  pdl_allow_next_grid();
  const uint32_t tmem_base = s.tmem_slot;
  const int ntiles = gemm_my_count(p);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // The whole warp runs the loop; the elected lane issues the copies.
    const bool leader = elect_one_sync();
    uint32_t stage = 0, phase = 0;
    int issued = 0;
    for (int ti = 0; ti < ntiles; ++ti) {
      int pi, m_blk, n_blk;
      gemm_tile_at<BN>(p, ti, pi, m_blk, n_blk);
      const int kblocks = (p.prob[pi].K + kGemmBK - 1) / kGemmBK;
      for (int kb0 = 0; kb0 < kblocks; kb0 += kSmallStageKb) {
        const int nkb = min(kSmallStageKb, kblocks - kb0);
        const int ngroups = (nkb + kSmallGroupKb - 1) / kSmallGroupKb;
        if (!mbar_wait_warp(&s.empty[stage], phase ^ 1u, abort, p.wait_ns)) goto producer_done;
        if (leader) {
          mbar_arrive_expect_tx(&s.full[stage], ngroups * (kGemmBM * kSmallGroupBytes) +
                                                    nkb * (BN * kGemmBK));
          for (int g = 0; g < ngroups; ++g)
            tma_load_2d(s.apk[stage][g], &p.tmA[pi], &s.full[stage],
                        (kb0 + g * kSmallGroupKb) * kGemmPackedRowBytes, m_blk * kGemmBM);
          for (int j = 0; j < nkb; ++j)
            tma_load_2d(s.b[stage][j], &p.tmB[pi], &s.full[stage], (kb0 + j) * kGemmBK,
                        n_blk * BN);
        }
        __syncwarp();
        ++issued;
        if (++stage == S) { stage = 0; phase ^= 1u; }
      }
    }
  producer_done:
    if (leader) gemm_drain_loads<S>(s.full, issued);
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop; the elected lane issues the MMAs and the
    // commits (a commit tracks the MMAs of the thread that issues it).
    const bool leader = elect_one_sync();
    constexpr uint32_t idesc = idesc_i8(kGemmBM, BN);
    uint32_t stage = 0, phase = 0;
    SmallSlot sl;
    const uint64_t b_desc0 = smem_desc_k_sw128(smem_u32(s.b[0][0]));
    for (int ti = 0; ti < ntiles; ++ti) {
      int pi, m_blk, n_blk;
      gemm_tile_at<BN>(p, ti, pi, m_blk, n_blk);
      const int kblocks = (p.prob[pi].K + kGemmBK - 1) / kGemmBK;
      const uint32_t db = ti & 1, dp = (ti >> 1) & 1;
      if (!mbar_wait_warp(&s.tempty[db], dp ^ 1u, abort, p.wait_ns)) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + db * BN;
      bool ok = true;
      for (int kb0 = 0; kb0 < kblocks; kb0 += kSmallStageKb) {
        const int nkb = min(kSmallStageKb, kblocks - kb0);
        if (!mbar_wait_warp(&s.full[stage], phase, abort, p.wait_ns)) {
          ok = false;
          break;
        }
        // descriptor of this stage's first activation tile; the others are
        // immediate offsets from it (start address >> 4 in the low bits)
        const uint64_t bd =
            b_desc0 + static_cast<uint64_t>((stage * (kSmallStageKb * BN * kGemmBK)) >> 4);
        for (int g = 0; g * kSmallGroupKb < nkb; ++g) {
          if (!mbar_wait_warp(&s.afull[sl.slot], sl.phase, abort, p.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_slot = tmem_base + kAColBase + kSmallSlotCols * sl.slot;
          const uint64_t bg =
              bd + static_cast<uint64_t>((g * kSmallGroupKb * BN * kGemmBK) >> 4);
          const int gkb = min(kSmallGroupKb, nkb - g * kSmallGroupKb);
          const uint32_t first = (kb0 == 0 && g == 0) ? 0u : 1u;   // accumulate flag of MMA 0
          if (gkb == kSmallGroupKb) {
#pragma unroll
            for (int j = 0; j < kSmallGroupKb; ++j)
#pragma unroll
              for (int kk = 0; kk < kGemmBK / 32; ++kk) {
                const uint64_t bdesc =
                    bg + static_cast<uint64_t>((j * BN * kGemmBK + 32 * kk) >> 4);
                if (leader)
                  mma_i8_ts(d_tmem, a_slot + 32 * j + 8 * kk, bdesc, idesc,
                            (j | kk) == 0 ? first : 1u);
              }
          } else {
            for (int j = 0; j < gkb; ++j)
#pragma unroll
              for (int kk = 0; kk < kGemmBK / 32; ++kk) {
                const uint64_t bdesc =
                    bg + static_cast<uint64_t>((j * BN * kGemmBK + 32 * kk) >> 4);
                if (leader)
                  mma_i8_ts(d_tmem, a_slot + 32 * j + 8 * kk, bdesc, idesc,
                            (j | kk) == 0 ? first : 1u);
              }
          }
          if (leader) mma_commit(&s.aempty[sl.slot]);
          __syncwarp();
          sl.advance<kSlots>();
        }
        if (!ok) break;
        if (leader) mma_commit(&s.empty[stage]);
        __syncwarp();
        if (++stage == S) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
      if (leader) mma_commit(&s.tfull[db]);
      __syncwarp();
    }
    if (leader) {
      mma_commit(&s.drain);
      mbar_drain(&s.drain, 0);
    }
    __syncwarp();
  } else if (warp >= 4 && warp < 4 + 4 * kSmallUnpackGroups) {
    // ------------------------------------------------------------ unpackers
    const uint32_t quarter = static_cast<uint32_t>(warp & 3);
    const int group = (warp - 4) >> 2;                     // the stage's k-group it expands
    const int u = static_cast<int>(quarter) * 32 + lane;   // weight row within the tile
    const uint32_t sw = static_cast<uint32_t>(u & 7);       // the row's 128-byte swizzle
    const uint32_t lane_addr = (quarter * 32u) << 16;
    uint32_t stage = 0, phase = 0;
    SmallSlot first;   // A slot of the current stage's first k-group
    for (int ti = 0; ti < ntiles; ++ti) {
      int pi, m_blk, n_blk;
      gemm_tile_at<BN>(p, ti, pi, m_blk, n_blk);
      const int kblocks = (p.prob[pi].K + kGemmBK - 1) / kGemmBK;
      for (int kb0 = 0; kb0 < kblocks; kb0 += kSmallStageKb) {
        const int nkb = min(kSmallStageKb, kblocks - kb0);
        const int ngroups = (nkb + kSmallGroupKb - 1) / kSmallGroupKb;
        if (group < ngroups) {
          SmallSlot my = first;
          for (int g = 0; g < group; ++g) my.advance<kSlots>();
          const int gkb = min(kSmallGroupKb, nkb - group * kSmallGroupKb);
          if (!mbar_wait_warp(&s.full[stage], phase, abort, p.wait_ns) ||
              !mbar_wait_warp(&s.aempty[my.slot], my.phase ^ 1u, abort, p.wait_ns))
            goto unpack_done;
          tc_fence_after();
          // the row's 128 bytes: 16-byte chunk c at chunk c ^ (row % 8)
          const uint8_t* row = s.apk[stage][group] + u * kSmallGroupBytes;
          uint4 c[8];
#pragma unroll
          for (int q = 0; q < 8; ++q)
            c[q] = *reinterpret_cast<const uint4*>(row + ((static_cast<uint32_t>(q) ^ sw) << 4));
          const uint32_t a_slot = tmem_base + lane_addr + kAColBase + kSmallSlotCols * my.slot;
#pragma unroll
          for (int j = 0; j < kSmallGroupKb; ++j) {
            if (j < gkb) {
              const uint32_t words[8] = {c[2 * j].x,     c[2 * j].y,     c[2 * j].z,
                                         c[2 * j].w,     c[2 * j + 1].x, c[2 * j + 1].y,
                                         c[2 * j + 1].z, c[2 * j + 1].w};
              uint32_t r[32];
#pragma unroll
              for (int w = 0; w < 8; ++w) {   // column 4w + i holds weights 16w + 4i .. +3
                r[4 * w + 0] = words[w] & 0x03030303u;
                r[4 * w + 1] = (words[w] >> 2) & 0x03030303u;
                r[4 * w + 2] = (words[w] >> 4) & 0x03030303u;
                r[4 * w + 3] = (words[w] >> 6) & 0x03030303u;
              }
              tmem_st_32x32b_x32(a_slot + 32 * j, r);
            }
          }
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&s.afull[my.slot]);
        }
        for (int g = 0; g < ngroups; ++g) first.advance<kSlots>();
        if (++stage == S) { stage = 0; phase ^= 1u; }
      }
    }
  unpack_done:;
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    const uint32_t quarter = static_cast<uint32_t>(warp & 3);   // warps 2, 3, 12, 13
    for (int ti = 0; ti < ntiles; ++ti) {
      int pi, m_blk, n_blk;
      gemm_tile_at<BN>(p, ti, pi, m_blk, n_blk);
      const GemmProblem pr = p.prob[pi];   // by value: registers
      const uint32_t db = ti & 1, dp = (ti >> 1) & 1;
      // lane n holds token n's scale and activation sum
      const int nl = n_blk * BN + lane;
      float sc = 0.0f;
      int xs = 0;
      if (lane < BN && nl < pr.N) {
        sc = __fmul_rn(__ldg(pr.alpha), __fdiv_rn(__ldg(pr.amax + nl), 127.0f));
        xs = __ldg(pr.xsum + nl);
      }
      if (!mbar_wait_warp(&s.tfull[db], dp, abort, p.wait_ns)) break;
      tc_fence_after();
      uint32_t r[BN];
      const uint32_t taddr = tmem_base + ((quarter * 32u) << 16) + db * BN;
      if constexpr (BN == 16) {
        tmem_ld_32x32b_x16(taddr, r);
      } else {
        tmem_ld_32x32b_x32(taddr, r);
      }
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.tempty[db]);
      const int m = m_blk * kGemmBM + static_cast<int>(quarter) * 32 + lane;
#pragma unroll
      for (int j = 0; j < BN; ++j) {
        const float scj = __shfl_sync(0xFFFFFFFFu, sc, j);
        const int xsj = __shfl_sync(0xFFFFFFFFu, xs, j);
        const int n = n_blk * BN + j;
        if (n < pr.N && m < pr.M) {
          const int a = static_cast<int>(r[j]) - xsj;
          const int64_t o = static_cast<int64_t>(n) * pr.M + m;
          pr.y[o] = __fmul_rn(__int2float_rn(a), scj);
          if (pr.acc) pr.acc[o] = a;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, kSmallTmemCols);
  }
}

}  // namespace bl
