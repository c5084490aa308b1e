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
// The ring moves k-groups of four k-blocks (512 weights): per stage one TMA
// box of 128 weight rows x 128 packed bytes (128-byte swizzle, so the row
// reads below are conflict-free) and the group's activation tiles (BN x 128
// int8 each, 128-byte swizzle).  Whole 128-byte rows keep the number of
// memory requests per weight byte low: rows 32 bytes wide (one k-block) left
// DRAM at a seventh of its bandwidth, most of each row's sectors missing L2
// one 32-byte request at a time.
//
//   warp 0        TMA producer;
//   warps 4-11    unpackers, in kSmallUnpackGroups groups of four that take
//                 alternate k-groups: warp w owns tensor-memory lanes
//                 32 (w % 4) .. +31, one weight row per lane; per k-group it
//                 reads its row's 128 packed bytes, expands each k-block's 32
//                 bytes to 32 words of codes+1 (four int8 per word, in k order)
//                 and stores them with one tcgen05.st into one of the four A
//                 buffers (32 columns each) of the group's slot, then waits once
//                 for the group's stores and hands the slot to the MMA;
//   warp 1        MMA issuer: 4 x tcgen05.mma kind::i8 (K = 32) per k-block,
//                 A from tensor memory, B from the ring; one commit per k-group
//                 frees the A slot and one its ring stage (barrier waits and
//                 commits, not the MMAs, took most of this thread's time when
//                 they were per k-block); accumulators double-buffered;
//   warps 2,3,12,13  epilogue, one per lane quarter: tcgen05.ld of BN columns,
//                 subtract the token's sum of q (the +1 code offset), rescale
//                 by alpha * amax / 127, store y (lane = row: coalesced).
//
// Tiles (one per 128-row block of every problem of the launch) are spread
// over persistent CTAs by the host's longest-first schedule, as in gemm.cuh.
// Every wait is bounded (GemmParams::wait_ns), and the CTA drains the copies
// and MMAs it has issued before it releases tensor memory.
#pragma once

#include "gemm.cuh"

namespace bl {

constexpr int kSmallUnpackGroups = 2;
constexpr int kSmallThreads = (6 + 4 * kSmallUnpackGroups) * 32;   // 14 warps
constexpr int kSmallGroupKb = 4;                                   // k-blocks per ring stage
constexpr int kSmallGroupBytes = kSmallGroupKb * kGemmPackedRowBytes;   // 128 per row
// Each tile accumulates into kSmallAcc independent accumulators (MMA kk of every
// k-block into accumulator kk), summed in the epilogue: consecutive MMAs then
// do not wait for each other's result, which short MMAs (N = 16 or 32) would
// otherwise do once per K = 32 step.
constexpr int kSmallAcc = 4;
static_assert(kSmallAcc == kGemmBK / 32, "one accumulator per K = 32 step of a k-block");
constexpr uint32_t kSmallTmemCols = 512;
// Tensor memory: two sets of kSmallAcc accumulators of BN columns, then the A
// buffers (32 columns each) in what is left.
__host__ __device__ constexpr int small_acol_base(int bn) { return 2 * kSmallAcc * bn; }
__host__ __device__ constexpr int small_abufs(int bn) {
  return (static_cast<int>(kSmallTmemCols) - small_acol_base(bn)) / 32;
}
// A slots: the four A buffers of one k-group.
__host__ __device__ constexpr int small_aslots(int bn) { return small_abufs(bn) / kSmallGroupKb; }

__host__ __device__ constexpr int small_stages(int bn) { return bn <= 16 ? 8 : 6; }

template <int BN>
struct SmallSmem {
  static constexpr int S = small_stages(BN);
  // each array up to the barriers is a multiple of 1024 bytes
  uint8_t apk[S][kGemmBM * kSmallGroupBytes];          // packed weights, 16 KB, swizzled
  uint8_t b[S][kSmallGroupKb][BN * kGemmBK];           // activations, 128-byte swizzle
  uint64_t full[S];
  uint64_t empty[S];                                   // MMA commit + 4 unpack warps
  uint64_t afull[small_aslots(BN)];                    // 4 unpack warps
  uint64_t aempty[small_aslots(BN)];                   // MMA commit
  uint64_t tfull[2];
  uint64_t tempty[2];                                  // 4 epilogue warps
  uint64_t drain;
  uint32_t tmem_slot;
  int abort;
};

template <int BN>
__global__ void __launch_bounds__(kSmallThreads, 1)
gemm_small_kernel(const __grid_constant__ GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  using Smem = SmallSmem<BN>;
  constexpr int S = Smem::S;
  constexpr int kSlots = small_aslots(BN);
  constexpr uint32_t kSmallAColBase = small_acol_base(BN);
  pdl_wait_prior_grid();
  pdl_allow_next_grid();
  const uint32_t base = smem_u32(smem_raw);
  Smem& s = *reinterpret_cast<Smem*>(smem_raw + ((1024u - (base & 1023u)) & 1023u));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile int* abort = &s.abort;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1 + 4);
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
  const uint32_t tmem_base = s.tmem_slot;
  const int ntiles = gemm_my_count(p);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      int issued = 0;
      for (int ti = 0; ti < ntiles; ++ti) {
        int pi, m_blk, n_blk;
        gemm_locate<BN>(p, gemm_my_tile(p, ti), pi, m_blk, n_blk);
        const int kblocks = (p.prob[pi].K + kGemmBK - 1) / kGemmBK;
        for (int kb0 = 0; kb0 < kblocks; kb0 += kSmallGroupKb) {
          const int nkb = min(kSmallGroupKb, kblocks - kb0);
          if (!mbar_wait(&s.empty[stage], phase ^ 1u, abort, p.wait_ns)) goto producer_done;
          mbar_arrive_expect_tx(&s.full[stage],
                                kGemmBM * kSmallGroupBytes + nkb * BN * kGemmBK);
          tma_load_2d(s.apk[stage], &p.tmA[pi], &s.full[stage], kb0 * kGemmPackedRowBytes,
                      m_blk * kGemmBM);
          for (int j = 0; j < nkb; ++j)
            tma_load_2d(s.b[stage][j], &p.tmB[pi], &s.full[stage], (kb0 + j) * kGemmBK,
                        n_blk * BN);
          ++issued;
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
      }
    producer_done:
      gemm_drain_loads<S>(s.full, issued);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8(kGemmBM, BN);
      uint32_t stage = 0, phase = 0, slot = 0, sphase = 0;
      for (int ti = 0; ti < ntiles; ++ti) {
        int pi, m_blk, n_blk;
        gemm_locate<BN>(p, gemm_my_tile(p, ti), pi, m_blk, n_blk);
        const int kblocks = (p.prob[pi].K + kGemmBK - 1) / kGemmBK;
        const uint32_t db = ti & 1, dp = (ti >> 1) & 1;
        if (!mbar_wait(&s.tempty[db], dp ^ 1u, abort, p.wait_ns)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + db * kSmallAcc * BN;
        bool ok = true;
        for (int kb0 = 0; kb0 < kblocks; kb0 += kSmallGroupKb) {
          const int nkb = min(kSmallGroupKb, kblocks - kb0);
          if (!mbar_wait(&s.full[stage], phase, abort, p.wait_ns) ||
              !mbar_wait(&s.afull[slot], sphase, abort, p.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_slot = tmem_base + kSmallAColBase + 32 * kSmallGroupKb * slot;
          for (int j = 0; j < nkb; ++j) {
            const uint32_t b_addr = smem_u32(s.b[stage][j]);
#pragma unroll
            for (int kk = 0; kk < kGemmBK / 32; ++kk)   // accumulator kk (kSmallAcc == 4)
              mma_i8_ts(d_tmem + kk * BN, a_slot + 32 * j + 8 * kk,
                        smem_desc_k_sw128(b_addr + 32 * kk), idesc, (kb0 + j) != 0);
          }
          mma_commit(&s.aempty[slot]);
          mma_commit(&s.empty[stage]);
          if (++stage == S) { stage = 0; phase ^= 1u; }
          if (++slot == kSlots) { slot = 0; sphase ^= 1u; }
        }
        if (!ok) break;
        mma_commit(&s.tfull[db]);
      }
      mma_commit(&s.drain);
      mbar_drain(&s.drain, 0);
    }
  } else if (warp >= 4 && warp < 4 + 4 * kSmallUnpackGroups) {
    // ------------------------------------------------------------ unpackers
    const uint32_t quarter = static_cast<uint32_t>(warp & 3);
    const int group = (warp - 4) >> 2;   // takes the k-groups whose sequence number % groups == group
    const int u = static_cast<int>(quarter) * 32 + lane;   // weight row within the tile
    const uint32_t sw = static_cast<uint32_t>(u & 7);       // the row's 128-byte swizzle
    const uint32_t lane_addr = (quarter * 32u) << 16;
    uint32_t stage = 0, phase = 0, slot = 0, sphase = 0;
    int seq = 0;
    for (int ti = 0; ti < ntiles; ++ti) {
      int pi, m_blk, n_blk;
      gemm_locate<BN>(p, gemm_my_tile(p, ti), pi, m_blk, n_blk);
      const int kblocks = (p.prob[pi].K + kGemmBK - 1) / kGemmBK;
      for (int kb0 = 0; kb0 < kblocks; kb0 += kSmallGroupKb, ++seq) {
        const int nkb = min(kSmallGroupKb, kblocks - kb0);
        if (seq % kSmallUnpackGroups == group) {
          if (!mbar_wait(&s.full[stage], phase, abort, p.wait_ns) ||
              !mbar_wait(&s.aempty[slot], sphase ^ 1u, abort, p.wait_ns))
            goto unpack_done;
          tc_fence_after();
          // the row's 128 bytes: 16-byte chunk c at chunk c ^ (row % 8)
          const uint8_t* row = s.apk[stage] + u * kSmallGroupBytes;
          uint4 c[8];
#pragma unroll
          for (int q = 0; q < 8; ++q)
            c[q] = *reinterpret_cast<const uint4*>(row + ((static_cast<uint32_t>(q) ^ sw) << 4));
          const uint32_t a_slot =
              tmem_base + lane_addr + kSmallAColBase + 32 * kSmallGroupKb * slot;
#pragma unroll
          for (int j = 0; j < kSmallGroupKb; ++j) {
            if (j < nkb) {
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
          if (lane == 0) {
            mbar_arrive(&s.afull[slot]);
            mbar_arrive(&s.empty[stage]);   // this warp has read its packed rows
          }
        }
        if (++stage == S) { stage = 0; phase ^= 1u; }
        if (++slot == kSlots) { slot = 0; sphase ^= 1u; }
      }
    }
  unpack_done:;
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    const uint32_t quarter = static_cast<uint32_t>(warp & 3);   // warps 2, 3, 12, 13
    for (int ti = 0; ti < ntiles; ++ti) {
      int pi, m_blk, n_blk;
      gemm_locate<BN>(p, gemm_my_tile(p, ti), pi, m_blk, n_blk);
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
      if (!mbar_wait(&s.tfull[db], dp, abort, p.wait_ns)) break;
      tc_fence_after();
      uint32_t r[BN];
      const uint32_t taddr = tmem_base + ((quarter * 32u) << 16) + db * kSmallAcc * BN;
#pragma unroll
      for (int j = 0; j < BN; ++j) r[j] = 0;
#pragma unroll
      for (int a = 0; a < kSmallAcc; ++a) {   // the accumulators' int32 sums
        uint32_t t[BN];
        if constexpr (BN == 16) {
          tmem_ld_32x32b_x16(taddr + a * BN, t);
        } else {
          tmem_ld_32x32b_x32(taddr + a * BN, t);
        }
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < BN; ++j) r[j] += t[j];
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
