// gemm.cuh -- prefill mpGEMM on the 5th-generation tensor cores.
//
// For many tokens the ternary x int8 product is a dense contraction (the
// reading notes, section 4.4, note that prefill turns compute-bound and is
// left unoptimised by the CPU kernels).  Each CTA owns a 128-row weight block
// and a BN-token block, accumulating D[128 x BN] (int32) in tensor memory:
//
//   warp 0      TMA producer (elected lane): packed weight tile (128 rows x 32 bytes = 128
//               weights per row) and int8 activation tile (BN x 128, 128-byte
//               swizzle) into a STAGES-deep shared-memory ring;
//   warps 2-5   unpackers: one weight row per thread, 2-bit fields -> int8
//               codes+1 written in the 128-byte-swizzled K-major layout the
//               MMA reads (a double buffer of its own, so the TMA ring only
//               holds what is in flight from memory), then a proxy fence and an
//               mbarrier arrive;
//   warp 1      MMA issue warp, an elected lane issuing (a loop run by one
//               lane alone costs ~50 cycles per MMA in instruction overhead):
//               4 x tcgen05.mma kind::i8 (K = 32 each) per stage,
//               tcgen05.commit frees the stage; accumulators double-buffered
//               in tensor memory so the epilogue of tile i overlaps tile i+1;
//   warps 6-13  epilogue, two warps per TMEM lane quarter, alternate 32-column
//               chunks: tcgen05.ld, acc - xsum (removes the +1 code offset),
//               rescale by alpha * amax/127, staged in shared memory per 32 x 32
//               block and written by bulk tensor stores.
//
// Several independent problems (e.g. the projections of a layer) can share one
// persistent launch: tiles are numbered across problems.
#pragma once

#include "ptx.cuh"

namespace bl {

constexpr int kGemmBM = 128;
constexpr int kGemmBK = 128;                       // int8 elements per k-block
constexpr int kGemmPackedRowBytes = kGemmBK / 4;   // 32 bytes of 2-bit fields
constexpr int kGemmEpiWarps = 8;                   // two per TMEM lane quarter
constexpr int kGemmThreads = (6 + kGemmEpiWarps) * 32;   // 14 warps
constexpr int kGemmMaxProblems = 8;
constexpr int kGemmUnpackBufs = 2;    // unpacked A tiles live only from unpack to MMA
constexpr int kGemmMaxGrid = 160;      // CTAs a host-built schedule can describe
constexpr int kGemmMaxSched = 4096;    // tiles a host-built schedule can describe

struct GemmProblem {
  const float* alpha;
  const float* amax;
  const int32_t* xsum;
  float* y;
  int32_t* acc;
  int M, K, N;
  int n_tiles;      // ceil(N / BN)
  int tile_begin;   // first global tile of this problem
  int direct_store; // 1: y is written with plain stores (its row pitch is not a TMA stride)
};

struct GemmParams {
  CUtensorMap tmA[kGemmMaxProblems];   // packed weights as uint8 [M][row bytes], box 32 x 128
  CUtensorMap tmB[kGemmMaxProblems];   // xq as uint8 [N][K], box 128 x BN, 128B swizzle
  CUtensorMap tmY[kGemmMaxProblems];   // y as fp32 [N][M], box 32 x 32
  GemmProblem prob[kGemmMaxProblems];
  int num_problems;
  int total_tiles;
  // Tile schedule: with use_sched, CTA b runs sched[sched_begin[b] ..
  // sched_begin[b+1]) in that order (built on the host, longest tiles first,
  // each to the least-loaded CTA); otherwise tiles b, b + grid, b + 2 grid...
  int use_sched;
  unsigned long long wait_ns;   // limit of every bounded wait of the launch
  uint16_t sched_begin[kGemmMaxGrid + 1];
  uint32_t sched[kGemmMaxSched];   // gemm_sched_entry(problem, m_blk, n_blk)
};
static_assert(sizeof(GemmParams) <= 32764, "kernel parameter space");

// A schedule entry packs a tile's problem, row block and token block, so a
// CTA finds its tile with two parameter loads (begin, entry) instead of a
// search over the problem table.  Schedules exist only for launches of at
// most kGemmMaxSched tiles, so both blocks fit in their fields.
__host__ __device__ constexpr uint32_t gemm_sched_entry(int pi, int m_blk, int n_blk) {
  return (static_cast<uint32_t>(pi) << 29) | (static_cast<uint32_t>(m_blk) << 12) |
         static_cast<uint32_t>(n_blk);
}
static_assert(kGemmMaxProblems <= 8 && kGemmMaxSched <= 4096, "schedule entry fields");

// Tiles of worker `who` out of `nwho` (a CTA, or a CTA pair).
__device__ __forceinline__ int gemm_my_count(const GemmParams& p, int who, int nwho) {
  if (p.use_sched) return p.sched_begin[who + 1] - p.sched_begin[who];
  return who < p.total_tiles ? (p.total_tiles - 1 - who) / nwho + 1 : 0;
}


__device__ __forceinline__ int gemm_my_count(const GemmParams& p) {
  return gemm_my_count(p, static_cast<int>(blockIdx.x), static_cast<int>(gridDim.x));
}


// Per epilogue warp: the 32-token chunks it handles (alternate ones: half 0
// takes chunks 0, 2, ..., half 1 takes 1, 3, ...), 32 table entries each.
__host__ __device__ constexpr int gemm_ep_chunks(int BN) { return (BN / 32 + 1) / 2; }

template <int BN, int STAGES>
struct GemmSmem {
  // every array below up to ep_out is a multiple of 1024 bytes, so all of
  // them start 1024-byte aligned
  uint8_t b[STAGES][BN * kGemmBK];                          // TMA ring: activations
  uint8_t apk[STAGES][kGemmBM * kGemmPackedRowBytes];       // TMA ring: packed weights
  uint8_t a[kGemmUnpackBufs][kGemmBM * kGemmBK];            // unpacked codes+1
  float ep_out[kGemmEpiWarps][32 * 32];   // per epilogue warp: one 32 (n) x 32 (m) block
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t ufull[kGemmUnpackBufs];    // unpacked tile ready (one arrival per unpack warp)
  uint64_t uempty[kGemmUnpackBufs];   // unpacked tile consumed by the MMAs (commit)
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  float ep_scale[kGemmEpiWarps][32 * gemm_ep_chunks(BN)];   // per epilogue warp: alpha * amax/127
  int ep_xsum[kGemmEpiWarps][32 * gemm_ep_chunks(BN)];      // per epilogue warp: activation sums
  uint32_t tmem_slot;
  int abort;
};

// Before the CTA releases its shared memory: wait for the TMA loads still in
// flight.  Only the last STAGES loads issued can be (the producer waited for
// each stage to be consumed before refilling it); load i completes phase
// (i / STAGES) & 1 of full[i % STAGES], and nothing re-arms those barriers
// after the producer stops.  On the normal path every one of them has been
// consumed already and the waits return at once.
template <int STAGES>
__device__ __forceinline__ void gemm_drain_loads(uint64_t* full, int issued) {
  for (int i = issued - 1; i >= 0 && i >= issued - STAGES; --i)
    mbar_drain(&full[i % STAGES], static_cast<uint32_t>((i / STAGES) & 1));
}

template <int BN>
__device__ __forceinline__ void gemm_locate(const GemmParams& p, int tile, int& pi, int& m_blk,
                                            int& n_blk) {
  pi = 0;
  while (pi + 1 < p.num_problems && tile >= p.prob[pi + 1].tile_begin) ++pi;
  const int lt = tile - p.prob[pi].tile_begin;
  m_blk = lt / p.prob[pi].n_tiles;
  n_blk = lt - m_blk * p.prob[pi].n_tiles;
}

// Tile i of worker `who` (a CTA, or a CTA pair) out of `nwho`: its problem,
// row block and token block.
template <int BN>
__device__ __forceinline__ void gemm_tile_at(const GemmParams& p, int who, int nwho, int i,
                                             int& pi, int& m_blk, int& n_blk) {
  if (p.use_sched) {
    const uint32_t e = p.sched[p.sched_begin[who] + i];
    pi = static_cast<int>(e >> 29);
    m_blk = static_cast<int>((e >> 12) & 0x1FFFFu);
    n_blk = static_cast<int>(e & 0xFFFu);
    return;
  }
  gemm_locate<BN>(p, who + i * nwho, pi, m_blk, n_blk);
}

template <int BN>
__device__ __forceinline__ void gemm_tile_at(const GemmParams& p, int i, int& pi, int& m_blk,
                                             int& n_blk) {
  gemm_tile_at<BN>(p, static_cast<int>(blockIdx.x), static_cast<int>(gridDim.x), i, pi, m_blk,
                   n_blk);
}

template <int BN, int STAGES>
__global__ void __launch_bounds__(kGemmThreads, 1)
gemm_i8_tcgen05_kernel(const __grid_constant__ GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  using Smem = GemmSmem<BN, STAGES>;
  const uint32_t base = smem_u32(smem_raw);
  Smem& s = *reinterpret_cast<Smem*>(smem_raw + ((1024u - (base & 1023u)) & 1023u));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  constexpr uint32_t kTmemCols = 2 * BN;
  constexpr uint32_t kStageTx = kGemmBM * kGemmPackedRowBytes + BN * kGemmBK;
  volatile int* abort = &s.abort;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    for (int i = 0; i < kGemmUnpackBufs; ++i) {
      mbar_init(&s.ufull[i], 4);                   // one arrival per unpack warp
      mbar_init(&s.uempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.tfull[i], 1);
      mbar_init(&s.tempty[i], kGemmEpiWarps);      // one arrival per epilogue warp
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
    tmem_alloc(&s.tmem_slot, kTmemCols);
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

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // The whole warp runs the loop; the elected lane issues the copies.
    const bool leader = elect_one_sync();
    uint32_t stage = 0, phase = 0;
    int issued = 0;
    for (int ti = 0, tn = gemm_my_count(p); ti < tn; ++ti) {
      int pi, m_blk, n_blk;
      gemm_tile_at<BN>(p, ti, pi, m_blk, n_blk);
      const int kblocks = (p.prob[pi].K + kGemmBK - 1) / kGemmBK;
      for (int kb = 0; kb < kblocks; ++kb) {
        if (!mbar_wait_warp(&s.empty[stage], phase ^ 1u, abort, p.wait_ns)) goto producer_done;
        if (leader) {
          mbar_arrive_expect_tx(&s.full[stage], kStageTx);
          tma_load_2d(s.apk[stage], &p.tmA[pi], &s.full[stage], kb * kGemmPackedRowBytes,
                      m_blk * kGemmBM);
          tma_load_2d(s.b[stage], &p.tmB[pi], &s.full[stage], kb * kGemmBK, n_blk * BN);
        }
        __syncwarp();
        ++issued;
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
  producer_done:
    if (leader) gemm_drain_loads<STAGES>(s.full, issued);
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop (warp-uniform control and descriptors);
    // the elected lane issues the MMAs and the commits.
    const bool leader = elect_one_sync();
    constexpr uint32_t idesc = idesc_i8(kGemmBM, BN);
    const uint64_t a_desc0 = smem_desc_k_sw128(smem_u32(s.a[0]));
    const uint64_t b_desc0 = smem_desc_k_sw128(smem_u32(s.b[0]));
    uint32_t stage = 0, phase = 0, ub = 0, uphase = 0;
    int it = 0;
    for (int ti = 0, tn = gemm_my_count(p); ti < tn; ++ti, ++it) {
      int pi, m_blk, n_blk;
      gemm_tile_at<BN>(p, ti, pi, m_blk, n_blk);
      const int kblocks = (p.prob[pi].K + kGemmBK - 1) / kGemmBK;
      const uint32_t ab = it & 1, ap = (it >> 1) & 1;
      if (!mbar_wait_warp(&s.tempty[ab], ap ^ 1u, abort, p.wait_ns)) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + ab * BN;
      bool ok = true;
      for (int kb = 0; kb < kblocks; ++kb) {
        if (!mbar_wait_warp(&s.full[stage], phase, abort, p.wait_ns) ||
            !mbar_wait_warp(&s.ufull[ub], uphase, abort, p.wait_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // descriptors: start address >> 4 in the low bits, so offsets add
        const uint64_t ad = a_desc0 + static_cast<uint64_t>((ub * (kGemmBM * kGemmBK)) >> 4);
        const uint64_t bd = b_desc0 + static_cast<uint64_t>((stage * (BN * kGemmBK)) >> 4);
#pragma unroll
        for (int kk = 0; kk < kGemmBK / 32; ++kk) {
          if (leader)
            mma_i8_ss(d_tmem, ad + static_cast<uint64_t>(2 * kk),
                      bd + static_cast<uint64_t>(2 * kk), idesc, (kb | kk) != 0);
        }
        if (leader) {
          mma_commit(&s.empty[stage]);
          mma_commit(&s.uempty[ub]);
        }
        __syncwarp();
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        if (++ub == kGemmUnpackBufs) { ub = 0; uphase ^= 1u; }
      }
      if (!ok) break;
      if (leader) mma_commit(&s.tfull[ab]);
      __syncwarp();
    }
    // Everything issued must finish before tensor memory is released.
    if (leader) {
      mma_commit(&s.drain);
      mbar_drain(&s.drain, 0);
    }
    __syncwarp();
  } else if (warp < 6) {
    // ------------------------------------------------------------ unpackers
    const int u = threadIdx.x - 64;   // weight row within the tile
    const uint32_t sw = static_cast<uint32_t>(u & 7);
    const int half = (u >> 2) & 1;   // read order of the two 16-byte halves: no bank conflict
    uint32_t stage = 0, phase = 0, ub = 0, uphase = 0;
    for (int ti = 0, tn = gemm_my_count(p); ti < tn; ++ti) {
        int pi, m_blk, n_blk;
        gemm_tile_at<BN>(p, ti, pi, m_blk, n_blk);
      const int kblocks = (p.prob[pi].K + kGemmBK - 1) / kGemmBK;
      for (int kb = 0; kb < kblocks; ++kb) {
        if (!mbar_wait_warp(&s.full[stage], phase, abort, p.wait_ns) ||
            !mbar_wait_warp(&s.uempty[ub], uphase ^ 1u, abort, p.wait_ns))
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
        if (lane == 0) mbar_arrive(&s.ufull[ub]);
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        if (++ub == kGemmUnpackBufs) { ub = 0; uphase ^= 1u; }
      }
    }
  unpack_done:;
  } else {
    // ------------------------------------------------------------ epilogue
    const uint32_t quarter = static_cast<uint32_t>(warp & 3);   // TMEM lanes 32q .. 32q+31
    const int r_in_tile = static_cast<int>(quarter) * 32 + lane;
    const int e = warp - 6;                 // epilogue warp 0..7
    const int half = e >> 2;                // this warp stores column chunks cc = half, half+2, ...
    int it = 0;
    for (int ti = 0, tn = gemm_my_count(p); ti < tn; ++ti, ++it) {
        int pi, m_blk, n_blk;
        gemm_tile_at<BN>(p, ti, pi, m_blk, n_blk);
      // by value: registers, not re-read from parameter space after each store
      const GemmProblem pr = p.prob[pi];
      const uint32_t ab = it & 1, ap = (it >> 1) & 1;
      if (!mbar_wait_warp(&s.tfull[ab], ap, abort, p.wait_ns)) break;
      tc_fence_after();
      const int m = m_blk * kGemmBM + r_in_tile;
      // this warp's copy of the tile's per-token scale and sum
      float* sc = s.ep_scale[e];
      int* xs = s.ep_xsum[e];
      {
        // all loads in flight at once, then the divisions
        const float alpha = __ldg(pr.alpha);
        constexpr int kChunks = gemm_ep_chunks(BN);
        float am[kChunks];
        int xv[kChunks];
#pragma unroll
        for (int k = 0; k < kChunks; ++k) {
          const int n = n_blk * BN + (2 * k + half) * 32 + lane;
          const bool in = 2 * k + half < BN / 32 && n < pr.N;
          am[k] = in ? __ldg(pr.amax + n) : 0.0f;
          xv[k] = in ? __ldg(pr.xsum + n) : 0;
        }
        __syncwarp();
#pragma unroll
        for (int k = 0; k < kChunks; ++k) {
          sc[k * 32 + lane] = __fmul_rn(alpha, __fdiv_rn(am[k], 127.0f));
          xs[k * 32 + lane] = xv[k];
        }
        __syncwarp();
      }
      // Each 32 (token) x 32 (row) block is staged in shared memory, [n][m],
      // and written with one bulk tensor store (one staging buffer per warp).
#pragma unroll 1
      for (int cc = half; cc < BN / 32; cc += 2) {
        uint32_t r[32];
        __syncwarp();
        tmem_ld_32x32b_x32(tmem_base + ((quarter * 32u) << 16) + ab * BN + cc * 32, r);
        tmem_ld_wait();
        const int n0 = n_blk * BN + cc * 32;
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
        if (m_blk * kGemmBM + static_cast<int>(quarter) * 32 >= pr.M) continue;   // rows past M
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
          tma_store_2d(&p.tmY[pi], blk, m_blk * kGemmBM + static_cast<int>(quarter) * 32, n0);
          bulk_commit_group();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.tempty[ab]);
    }
    if (lane == 0) bulk_wait_group<0>();   // outputs written before the CTA retires
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace bl
