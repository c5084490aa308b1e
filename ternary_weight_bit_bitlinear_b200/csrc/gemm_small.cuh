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
// from shared memory.  Shared memory carries only the TMA ring: 4 KB of packed
// weights and BN x 128 bytes of activations per k-block of 128 weights.
//
//   warp 0        TMA producer: packed weights (128 rows x 32 bytes) and int8
//                 activations (BN x 128, 128-byte swizzle) into a deep ring;
//   warps 4-11    unpackers, in kSmallUnpackGroups groups of four that take
//                 alternate k-blocks: warp w owns tensor-memory lanes
//                 32 (w % 4) .. +31, one weight row per lane; per k-block it
//                 reads its 32 packed bytes, expands them to 32 words of
//                 codes+1 (four int8 per word, in k order) and stores them with
//                 one tcgen05.st into one of kSmallABufs A buffers (32 columns
//                 each).  A store must complete before its buffer is handed to
//                 the MMA, so one group alone would serialise on that latency;
//   warp 1        MMA issuer: 4 x tcgen05.mma kind::i8 (K = 32) per k-block,
//                 A from tensor memory, B from the ring; commits free the ring
//                 stage and the A buffer; accumulators double-buffered;
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
constexpr int kSmallABufs = 14;          // A tiles in tensor memory, 32 columns each
constexpr int kSmallAColBase = 64;       // after two accumulators of up to 32 columns
constexpr uint32_t kSmallTmemCols = 512;

__host__ __device__ constexpr int small_stages(int bn) { return bn <= 16 ? 24 : 20; }

template <int BN>
struct SmallSmem {
  static constexpr int S = small_stages(BN);
  // each array up to the barriers is a multiple of 1024 bytes
  uint8_t b[S][BN * kGemmBK];                          // activations, 128-byte swizzle
  uint8_t apk[S][kGemmBM * kGemmPackedRowBytes];       // packed weights, 4 KB
  uint64_t full[S];
  uint64_t empty[S];                                   // MMA commit + 4 unpack warps
  uint64_t afull[kSmallABufs];                         // 4 unpack warps
  uint64_t aempty[kSmallABufs];                        // MMA commit
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
  pdl_wait_prior_grid();
  pdl_allow_next_grid();
  const uint32_t base = smem_u32(smem_raw);
  Smem& s = *reinterpret_cast<Smem*>(smem_raw + ((1024u - (base & 1023u)) & 1023u));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  constexpr uint32_t kStageTx = kGemmBM * kGemmPackedRowBytes + BN * kGemmBK;
  volatile int* abort = &s.abort;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1 + 4);
    }
    for (int i = 0; i < kSmallABufs; ++i) {
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
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&s.empty[stage], phase ^ 1u, abort, p.wait_ns)) goto producer_done;
          mbar_arrive_expect_tx(&s.full[stage], kStageTx);
          tma_load_2d(s.apk[stage], &p.tmA[pi], &s.full[stage], kb * kGemmPackedRowBytes,
                      m_blk * kGemmBM);
          tma_load_2d(s.b[stage], &p.tmB[pi], &s.full[stage], kb * kGemmBK, n_blk * BN);
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
      uint32_t stage = 0, phase = 0, ab = 0, aphase = 0;
      for (int ti = 0; ti < ntiles; ++ti) {
        int pi, m_blk, n_blk;
        gemm_locate<BN>(p, gemm_my_tile(p, ti), pi, m_blk, n_blk);
        const int kblocks = (p.prob[pi].K + kGemmBK - 1) / kGemmBK;
        const uint32_t db = ti & 1, dp = (ti >> 1) & 1;
        if (!mbar_wait(&s.tempty[db], dp ^ 1u, abort, p.wait_ns)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + db * BN;
        bool ok = true;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&s.full[stage], phase, abort, p.wait_ns) ||
              !mbar_wait(&s.afull[ab], aphase, abort, p.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_tmem = tmem_base + kSmallAColBase + 32 * ab;
          const uint32_t b_addr = smem_u32(s.b[stage]);
#pragma unroll
          for (int kk = 0; kk < kGemmBK / 32; ++kk)
            mma_i8_ts(d_tmem, a_tmem + 8 * kk, smem_desc_k_sw128(b_addr + 32 * kk), idesc,
                      (kb | kk) != 0);
          mma_commit(&s.empty[stage]);
          mma_commit(&s.aempty[ab]);
          if (++stage == S) { stage = 0; phase ^= 1u; }
          if (++ab == kSmallABufs) { ab = 0; aphase ^= 1u; }
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
    const int group = (warp - 4) >> 2;   // takes the k-blocks whose sequence number % groups == group
    const int u = static_cast<int>(quarter) * 32 + lane;   // weight row within the tile
    const int half = (u >> 2) & 1;   // read order of the two 16-byte halves: no bank conflict
    uint32_t stage = 0, phase = 0, ab = 0, aphase = 0;
    int seq = 0;
    for (int ti = 0; ti < ntiles; ++ti) {
      int pi, m_blk, n_blk;
      gemm_locate<BN>(p, gemm_my_tile(p, ti), pi, m_blk, n_blk);
      const int kblocks = (p.prob[pi].K + kGemmBK - 1) / kGemmBK;
      for (int kb = 0; kb < kblocks; ++kb, ++seq) {
        if (seq % kSmallUnpackGroups != group) {   // the other group's k-block
          if (++stage == S) { stage = 0; phase ^= 1u; }
          if (++ab == kSmallABufs) { ab = 0; aphase ^= 1u; }
          continue;
        }
        if (!mbar_wait(&s.full[stage], phase, abort, p.wait_ns) ||
            !mbar_wait(&s.aempty[ab], aphase ^ 1u, abort, p.wait_ns))
          goto unpack_done;
        tc_fence_after();
        const uint4* src = reinterpret_cast<const uint4*>(s.apk[stage] + u * kGemmPackedRowBytes);
        const uint4 h0 = src[half], h1 = src[half ^ 1];
        const uint4 p0 = half ? h1 : h0, p1 = half ? h0 : h1;
        const uint32_t words[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
        uint32_t r[32];
#pragma unroll
        for (int j = 0; j < 8; ++j) {   // column 4j + i holds weights 16j + 4i .. +3
          r[4 * j + 0] = words[j] & 0x03030303u;
          r[4 * j + 1] = (words[j] >> 2) & 0x03030303u;
          r[4 * j + 2] = (words[j] >> 4) & 0x03030303u;
          r[4 * j + 3] = (words[j] >> 6) & 0x03030303u;
        }
        tmem_st_32x32b_x32(tmem_base + ((quarter * 32u) << 16) + kSmallAColBase + 32 * ab, r);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&s.afull[ab]);
          mbar_arrive(&s.empty[stage]);   // this warp has read its packed rows
        }
        if (++stage == S) { stage = 0; phase ^= 1u; }
        if (++ab == kSmallABufs) { ab = 0; aphase ^= 1u; }
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
