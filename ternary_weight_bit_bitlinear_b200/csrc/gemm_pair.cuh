// gemm_pair.cuh -- the prefill GEMM of gemm.cuh on CTA pairs (tcgen05 with
// cta_group::2), for tiles of 256 weight rows x 256 tokens.
//
// The two CTAs of a cluster sit on two SMs.  Each loads its own 128 weight
// rows (packed, then unpacked to int8 as in gemm.cuh) and its own half of the
// tile's activations (128 tokens); an elected lane of the rank-0 CTA's MMA
// warp (the whole warp runs the issue loop, as in gemm.cuh) issues
// tcgen05.mma.cta_group::2 with M = 256 and N = 256, which reads A and B from
// both shared memories and writes each CTA's 128 rows of D into that CTA's
// tensor memory.  Per SM this halves the activation bytes that TMA brings in
// and that the MMAs read from shared memory, compared with one CTA per
// 128 x 256 tile, so the same shared memory holds a deeper ring.
//
// Synchronisation (barriers at the same offsets in both CTAs):
//   afull[s]   local: this CTA's packed weight rows of stage s landed
//   bfull[s]   rank 0: both halves of the activations of stage s landed
//              (the rank-1 TMA counts its bytes on rank 0's barrier)
//   ufull[u]   rank 0: all 8 unpack warps of the pair are done
//   empty[s], uempty[u], tfull[a], drain
//              local in both: tcgen05.commit multicast to the pair
//   tempty[a]  rank 0: all 16 epilogue warps of the pair have read D
// Unpacked tiles are made visible to the MMAs with fence.proxy.async before
// the arrival; tensor-memory reads are ordered with tcgen05 fences.  Every
// wait is bounded, and both CTAs meet at a cluster barrier before either
// releases tensor memory or exits.
#pragma once

#include "gemm.cuh"

namespace bl {

constexpr int kPairBN = 256;           // tokens per pair tile
constexpr int kPairHalfN = 128;        // tokens whose activations each CTA loads
constexpr int kPairBM = 2 * kGemmBM;   // weight rows per pair tile
// Unpacked tiles in flight: the MMA of a k-block waits for both CTAs'
// unpackers, whose buffer is freed by the pair's commit, so every k-block
// crosses between the SMs twice; four buffers keep that round trip off the
// MMA's critical path.
constexpr int kPairUnpackBufs = 4;

template <int STAGES>
struct GemmPairSmem {
  // every array below up to ep_out is a multiple of 1024 bytes
  uint8_t b[STAGES][kPairHalfN * kGemmBK];                  // this CTA's activations, 16 KB
  uint8_t apk[STAGES][kGemmBM * kGemmPackedRowBytes];       // this CTA's packed rows, 4 KB
  uint8_t a[kPairUnpackBufs][kGemmBM * kGemmBK];            // unpacked codes+1
  float ep_out[kGemmEpiWarps][32 * 32];
  uint64_t afull[STAGES];
  uint64_t bfull[STAGES];
  uint64_t empty[STAGES];
  uint64_t ufull[kPairUnpackBufs];
  uint64_t uempty[kPairUnpackBufs];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  float ep_scale[kGemmEpiWarps][kPairBN / 2];
  int ep_xsum[kGemmEpiWarps][kPairBN / 2];
  uint32_t tmem_slot;
  int abort;
};

template <int STAGES>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
gemm_i8_pair_kernel(const __grid_constant__ GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  using Smem = GemmPairSmem<STAGES>;
  const uint32_t base = smem_u32(smem_raw);
  Smem& s = *reinterpret_cast<Smem*>(smem_raw + ((1024u - (base & 1023u)) & 1023u));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int npairs = static_cast<int>(gridDim.x >> 1);
  constexpr uint32_t kTmemCols = 2 * kPairBN;
  constexpr uint32_t kATx = kGemmBM * kGemmPackedRowBytes;
  constexpr uint32_t kBTx = 2 * kPairHalfN * kGemmBK;   // both halves, counted on rank 0
  volatile int* abort = &s.abort;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&s.afull[i], 1);
      mbar_init(&s.bfull[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    for (int i = 0; i < kPairUnpackBufs; ++i) {
      mbar_init(&s.ufull[i], 2 * 4);                   // one arrival per unpack warp
      mbar_init(&s.uempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.tfull[i], 1);
      mbar_init(&s.tempty[i], 2 * kGemmEpiWarps);      // one arrival per epilogue warp
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
    tmem_alloc_pair(&s.tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();   // both CTAs' barriers exist before either CTA touches the other's
  tc_fence_after();
  // The set-up above (barriers, tensor-map prefetch, tensor memory) touches
  // nothing the preceding kernel writes, so it overlaps that kernel's tail.
  pdl_wait_prior_grid();
  pdl_allow_next_grid();
  const uint32_t tmem_base = s.tmem_slot;
  const int ntiles = gemm_my_count(p, pair, npairs);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // The whole warp runs the loop; the elected lane issues the copies.
    // The two producers must issue the same number of loads: rank 1's
    // activation loads complete on rank 0's barriers, and rank 0 drains them
    // before the pair exits.  So they do not follow the CTA's abort flag
    // (which is per CTA) and wait on `empty` (committed to both CTAs alike)
    // with the drain limit: both stop at the same stage when the commits stop.
    const bool leader = elect_one_sync();
    volatile int no_abort = 0;
    uint32_t stage = 0, phase = 0;
    int issued = 0;
    for (int ti = 0; ti < ntiles; ++ti) {
      int pi, m_blk, n_blk;
      gemm_tile_at<kPairBN>(p, pair, npairs, ti, pi, m_blk, n_blk);
      const int kblocks = (p.prob[pi].K + kGemmBK - 1) / kGemmBK;
      for (int kb = 0; kb < kblocks; ++kb) {
        if (!mbar_wait_cluster_warp(&s.empty[stage], phase ^ 1u, &no_abort, kDrainLimitNs))
          goto producer_done;
        if (leader) {
          mbar_arrive_expect_tx(&s.afull[stage], kATx);
          tma_load_2d(s.apk[stage], &p.tmA[pi], &s.afull[stage], kb * kGemmPackedRowBytes,
                      m_blk * kPairBM + static_cast<int>(rank) * kGemmBM);
          if (rank == 0) mbar_arrive_expect_tx(&s.bfull[stage], kBTx);
          tma_load_2d_pair(s.b[stage], &p.tmB[pi], &s.bfull[stage], kb * kGemmBK,
                           n_blk * kPairBN + static_cast<int>(rank) * kPairHalfN);
        }
        __syncwarp();
        ++issued;
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
  producer_done:
    // This CTA's weight loads land on its own afull barriers; both CTAs'
    // activation loads count on rank 0's bfull barriers, so rank 0 waits for
    // those of the pair (the two producers issue the same sequence).
    if (leader) {
      gemm_drain_loads<STAGES>(s.afull, issued);
      if (rank == 0) gemm_drain_loads<STAGES>(s.bfull, issued);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (rank 0)
    // The whole warp of rank 0 runs the loop; the elected lane issues.
    if (rank == 0) {
      const bool leader = elect_one_sync();
      constexpr uint32_t idesc = idesc_i8(kPairBM, kPairBN);
      const uint64_t a_desc0 = smem_desc_k_sw128(smem_u32(s.a[0]));
      const uint64_t b_desc0 = smem_desc_k_sw128(smem_u32(s.b[0]));
      uint32_t stage = 0, phase = 0, ub = 0, uphase = 0;
      int it = 0;
      for (int ti = 0; ti < ntiles; ++ti, ++it) {
        int pi, m_blk, n_blk;
        gemm_tile_at<kPairBN>(p, pair, npairs, ti, pi, m_blk, n_blk);
        const int kblocks = (p.prob[pi].K + kGemmBK - 1) / kGemmBK;
        const uint32_t ab = it & 1, ap = (it >> 1) & 1;
        if (!mbar_wait_cluster_warp(&s.tempty[ab], ap ^ 1u, abort, p.wait_ns)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + ab * kPairBN;
        bool ok = true;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait_cluster_warp(&s.bfull[stage], phase, abort, p.wait_ns) ||
              !mbar_wait_cluster_warp(&s.ufull[ub], uphase, abort, p.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // descriptors: start address >> 4 in the low bits, so offsets add
          const uint64_t ad =
              a_desc0 + static_cast<uint64_t>((ub * static_cast<int>(sizeof(s.a[0]))) >> 4);
          const uint64_t bd =
              b_desc0 + static_cast<uint64_t>((stage * static_cast<int>(sizeof(s.b[0]))) >> 4);
#pragma unroll
          for (int kk = 0; kk < kGemmBK / 32; ++kk) {
            if (leader)
              mma_i8_ss_pair(d_tmem, ad + static_cast<uint64_t>(2 * kk),
                             bd + static_cast<uint64_t>(2 * kk), idesc, (kb | kk) != 0);
          }
          if (leader) {
            mma_commit_pair(&s.empty[stage]);
            mma_commit_pair(&s.uempty[ub]);
          }
          __syncwarp();
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
          if (++ub == kPairUnpackBufs) { ub = 0; uphase ^= 1u; }
        }
        if (!ok) break;
        if (leader) mma_commit_pair(&s.tfull[ab]);
        __syncwarp();
      }
      // Both CTAs learn through `drain` when the pair's last MMAs are done.
      if (leader) mma_commit_pair(&s.drain);
      __syncwarp();
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ unpackers
    const int u = threadIdx.x - 64;   // weight row within this CTA's 128
    const uint32_t sw = static_cast<uint32_t>(u & 7);
    const int half = (u >> 2) & 1;   // read order of the two 16-byte halves: no bank conflict
    uint32_t stage = 0, phase = 0, ub = 0, uphase = 0;
    for (int ti = 0; ti < ntiles; ++ti) {
      int pi, m_blk, n_blk;
      gemm_tile_at<kPairBN>(p, pair, npairs, ti, pi, m_blk, n_blk);
      const int kblocks = (p.prob[pi].K + kGemmBK - 1) / kGemmBK;
      for (int kb = 0; kb < kblocks; ++kb) {
        if (!mbar_wait_warp(&s.afull[stage], phase, abort, p.wait_ns) ||
            !mbar_wait_cluster_warp(&s.uempty[ub], uphase ^ 1u, abort, p.wait_ns))
          goto unpack_done;
        const uint4* src = reinterpret_cast<const uint4*>(s.apk[stage] + u * kGemmPackedRowBytes);
        const uint4 h0 = src[half], h1 = src[half ^ 1];
        const uint4 p0 = half ? h1 : h0, p1 = half ? h0 : h1;
        const uint32_t words[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
        uint8_t* row = s.a[ub] + (u >> 3) * 1024 + (u & 7) * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint32_t w = words[j];
          uint4 v;
          v.x = w & 0x03030303u;
          v.y = (w >> 2) & 0x03030303u;
          v.z = (w >> 4) & 0x03030303u;
          v.w = (w >> 6) & 0x03030303u;
          *reinterpret_cast<uint4*>(row + ((static_cast<uint32_t>(j) ^ sw) << 4)) = v;
        }
        fence_proxy_async_smem();   // each thread's stores, before the warp's one arrival
        __syncwarp();
        if (lane == 0) mbar_arrive_leader(&s.ufull[ub]);
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        if (++ub == kPairUnpackBufs) { ub = 0; uphase ^= 1u; }
      }
    }
  unpack_done:;
  } else {
    // ------------------------------------------------------------ epilogue
    const int e = warp - 6;                 // 0..7
    const int half = e >> 2;                // which alternate 32-column blocks
    const uint32_t quarter = warp & 3;      // TMEM lane quarter this warp may read
    const int r_in_tile = static_cast<int>(quarter) * 32 + lane;
    int it = 0;
    for (int ti = 0; ti < ntiles; ++ti, ++it) {
      int pi, m_blk, n_blk;
      gemm_tile_at<kPairBN>(p, pair, npairs, ti, pi, m_blk, n_blk);
      const GemmProblem pr = p.prob[pi];   // by value: registers, not parameter-space reloads
      const uint32_t ab = it & 1, ap = (it >> 1) & 1;
      if (!mbar_wait_cluster_warp(&s.tfull[ab], ap, abort, p.wait_ns)) break;
      tc_fence_after();
      const int m_base = m_blk * kPairBM + static_cast<int>(rank) * kGemmBM;
      const int m = m_base + r_in_tile;
      float* sc = s.ep_scale[e];
      int* xs = s.ep_xsum[e];
      {
        const float alpha = __ldg(pr.alpha);
        float am[kPairBN / 64];
        int xv[kPairBN / 64];
#pragma unroll
        for (int k = 0; k < kPairBN / 64; ++k) {
          const int n = n_blk * kPairBN + (2 * k + half) * 32 + lane;
          am[k] = n < pr.N ? __ldg(pr.amax + n) : 0.0f;
          xv[k] = n < pr.N ? __ldg(pr.xsum + n) : 0;
        }
        __syncwarp();
#pragma unroll
        for (int k = 0; k < kPairBN / 64; ++k) {
          sc[k * 32 + lane] = __fmul_rn(alpha, __fdiv_rn(am[k], 127.0f));
          xs[k * 32 + lane] = xv[k];
        }
        __syncwarp();
      }
#pragma unroll 1
      for (int cc = half; cc < kPairBN / 32; cc += 2) {
        uint32_t r[32];
        __syncwarp();
        tmem_ld_32x32b_x32(tmem_base + ((quarter * 32u) << 16) + ab * kPairBN + cc * 32, r);
        tmem_ld_wait();
        const int n0 = n_blk * kPairBN + cc * 32;
        if (n0 >= pr.N) continue;          // tokens past N: nothing to store
        if (pr.direct_store) {   // rows past M and tokens past N are not stored
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int a = static_cast<int>(r[j]) - xs[(cc >> 1) * 32 + j];
            if (m < pr.M && n0 + j < pr.N) {
              const int64_t o = static_cast<int64_t>(n0 + j) * pr.M + m;
              pr.y[o] = __fmul_rn(__int2float_rn(a), sc[(cc >> 1) * 32 + j]);
              if (pr.acc) pr.acc[o] = a;
            }
          }
          continue;
        }
        if (m_base + static_cast<int>(quarter) * 32 >= pr.M) continue;   // rows past M
        float* blk = s.ep_out[e];
        if (lane == 0) bulk_wait_group_read<0>();   // the previous store has read the block
        __syncwarp();
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int a = static_cast<int>(r[j]) - xs[(cc >> 1) * 32 + j];
          blk[j * 32 + lane] = __fmul_rn(__int2float_rn(a), sc[(cc >> 1) * 32 + j]);
          if (pr.acc && n0 + j < pr.N && m < pr.M)
            pr.acc[static_cast<int64_t>(n0 + j) * pr.M + m] = a;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&p.tmY[pi], blk, m_base + static_cast<int>(quarter) * 32, n0);
          bulk_commit_group();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_leader(&s.tempty[ab]);
    }
    if (lane == 0) bulk_wait_group<0>();   // outputs written before the CTA retires
  }

  // The pair's last MMAs write both CTAs' tensor memory and read both shared
  // memories: each CTA waits for them, then both meet before anything is freed.
  if (warp == 1 && lane == 0) mbar_drain(&s.drain, 0);
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

}  // namespace bl
