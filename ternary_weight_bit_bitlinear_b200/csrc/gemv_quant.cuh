// gemv_quant.cuh -- decode GEMV with the per-token activation quantiser fused
// into it: fp32 activations in, fp32 outputs out, no int8 round trip through
// global memory and no second launch.
//
// The fusion follows the FairyFuse "fused kernel design" (activation handling,
// unpacking and accumulation in one kernel, no intermediate writes) and keeps
// the I2_S arithmetic of the "Bitnet.cpp" reading notes (section 2.3, section
// 4.1): per-token absmax int8 activations, ternary weights, int32 sums, one
// fp32 rescale.  The quantised values are the ones quant.cuh produces:
//   amax = max_k |x[k]|,  s = 127 / amax,  q = clamp(rint(x * s), -128, 127).
//
// Work.  A launch's problems (layers) form segments: runs of consecutive
// problems that read the same input (pointer and K -- q, k and v, or gate and
// up, given side by side).  A unit is 32 rows of one problem over all of its K,
// and a pair is one unit and one k-chunk of 512 weights (128 bytes per row), so
// a segment holds units x ceil(K / 512) pairs.  The launch's units are cut
// into one contiguous range per CTA with about the same number of pairs each:
// CTA c starts at the unit nearest to pair (total pairs) x c / (CTAs), which
// every CTA computes from the segment table.  The host launches exactly the
// CTAs that fit on the GPU at once (one per resident slot, at most one per
// unit): with the two-stage rings and 256-byte L2 fills below, later waves of
// CTAs only add start-up work (each CTA quantises its inputs), and the 70B-
// shaped stream ran 2 to 3 % slower with two or four CTAs per slot.  A CTA's
// range meets one or more segments; each such meeting is an item, and the
// CTA takes its items in order:
//   1. all its threads quantise the item's input, once, into the CTA's int8
//      copy in shared memory (amax and the sum of q per token reduced across
//      the CTA);
//   2. its warps split the item's pairs evenly (warp w takes pairs
//      [P w / WC, P (w + 1) / WC) in unit-major order), each streaming the
//      weights through its own ring of 4 KB stages (16-byte cp.async copies,
//      the swizzled layout and dp4a arithmetic of gemv.cuh), with activations
//      read as broadcasts from the int8 copy;
//   3. a unit that one warp covers whole is written by it; a unit split
//      between warps is finished by the warp that holds its first k-chunk,
//      which adds the other warps' int32 partial sums (left in shared memory)
//      after a CTA barrier.  Integer sums: the order does not matter.
// The copy side of every warp runs ahead through its whole sequence of pairs,
// across units and items, so weights keep arriving while the CTA quantises
// the next item's input.  Before the dependent-launch wait, each warp
// prefetches its first stages' weights into L2 (a hint: the weights are not
// written by the preceding kernel, and nothing is read before the wait).
//
// Shared memory of a CTA (dynamic): the int8 copy [NT][xstride], the partial
// sums [WC][NT][4][32] int32, then WC rings of kGqStages x 4 KB.
#pragma once

#include "gemv.cuh"
#include "quant_math.cuh"

namespace bl {

// Two stages per warp: one computed while the next arrives.  The copies ask
// L2 for 256 bytes each (cp_async16_l2_256), so a row's following k-chunk is
// already on its way; the small ring leaves registers and shared memory for
// more warps per SM, and more warps hide more of the arithmetic's latency.
// (Four stages with the same copies stream about 7 % slower on the 70B-shaped
// launch, four stages with plain copies 12 to 14 % slower.)
constexpr int kGqStages = 2;                                          // power of two
constexpr int kGqStageBytes = kGemvTileRows * kGemvChunkBytes;        // 4 KB of weights
constexpr int kGqRingBytes = kGqStages * kGqStageBytes;
constexpr int kGqMaxProblems = 256;
constexpr int kGqMaxWarps = 12;          // 12 x 16 KB of rings already fill shared memory
constexpr int kGqMaxXBytes = 65536;   // tokens x K (rounded up to 512) held per CTA
constexpr int kGqRegF4 = 16;          // float4s per thread kept in registers while quantising

struct GqProblem {
  const uint32_t* packed;
  const float* alpha;
  float* y;                // fp32 [NT][M]
  int32_t* acc;            // int32 [NT][M] or null
  int M, W;                // W = words per packed row
  int unit_begin;          // first unit of this problem
};

// A run of problems that read one input.  Its units all have the same K.
struct GqSegment {
  const float* x;          // fp32 [NT][K]
  int K;
  int chunks;              // k-chunks per unit: ceil(K / 512)
  int unit_begin, units;   // the segment's units, numbered across the launch
  int prob_begin;          // first problem of the segment
  long long pair_begin;    // (unit, k-chunk) pairs of the segments before this one
};

struct GqParams {
  GqProblem prob[kGqMaxProblems];
  GqSegment seg[kGqMaxProblems];
  long long total_pairs;
  int total_units;
  int num_problems;
  int num_segments;
  int xstride;             // bytes per token of the int8 copy: 512 x the launch's largest chunks
  int area;                // dynamic shared memory bytes (gq_smem_bytes)
};

__host__ __device__ constexpr int gq_partial_bytes(int nt, int warps) {
  return warps * nt * 4 * 32 * 4;
}

__host__ __device__ constexpr int gq_smem_bytes(int nt, int warps, int xstride) {
  return nt * xstride + gq_partial_bytes(nt, warps) + warps * kGqRingBytes;
}

// Last index i in [0, n) with begin(i) <= v (begin nondecreasing, begin(0) <= v).
template <class F>
__device__ __forceinline__ int gq_last_le(int n, int v, F begin) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (begin(mid) <= v) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// First unit of CTA c's range (c in [0, ctas]): the unit boundary nearest to
// pair total_pairs * c / ctas.  Nondecreasing in c; 0 at c = 0 and every unit
// at c = ctas.  The host sizes the grid with the same rule in mind (a CTA
// whose range comes out empty returns at once).
__device__ __forceinline__ int gq_unit_bound(const GqParams& p, int c, int ctas) {
  if (c <= 0) return 0;
  if (c >= ctas) return p.total_units;
  const long long t = p.total_pairs * c / ctas;
  const int sg = gq_last_le(p.num_segments, 0, [&](int i) {
    return p.seg[i].pair_begin <= t ? 0 : 1;   // segments whose pairs start at or before t
  });
  const long long C = p.seg[sg].chunks;
  const long long u = p.seg[sg].unit_begin + (t - p.seg[sg].pair_begin + C / 2) / C;
  return static_cast<int>(u < p.total_units ? u : p.total_units);
}

// One item of a CTA: the units [ub, ue) of segment `seg`, `chunks` k-chunks
// each, and this warp's share [qb, qe) of its (ue - ub) * chunks pairs.
struct GqItem {
  int seg, ub, ue, chunks, qb, qe;
};

__device__ __forceinline__ GqItem gq_item(const GqParams& p, int seg, int u0, int u1, int warp,
                                          int nwarps) {
  const GqSegment& sg = p.seg[seg];
  GqItem it;
  it.seg = seg;
  it.ub = max(u0, sg.unit_begin);
  it.ue = min(u1, sg.unit_begin + sg.units);
  it.chunks = sg.chunks;
  const int P = (it.ue - it.ub) * it.chunks;
  it.qb = static_cast<int>(static_cast<int64_t>(P) * warp / nwarps);
  it.qe = static_cast<int>(static_cast<int64_t>(P) * (warp + 1) / nwarps);
  return it;
}

// Index i (< K4, or past it: left alone) moved by rot (0 <= rot < K4) modulo K4.
__device__ __forceinline__ int gq_rot(int i, int rot, int K4) {
  if (i >= K4) return i;
  const int r = i + rot;
  return r >= K4 ? r - K4 : r;
}

// Quantise segment sg's input x [NT][K] into xs [NT][xstride] (zero from K up
// to chunks * 512); amax / 127 and the sum of q per token go to s_a127 and
// s_xsum.  Run by every thread of the CTA; starts and ends with a barrier's
// worth of ordering (callers sync before reusing xs).  Thread tid takes the
// float4s (tid + rot + j n) mod K/4: CTAs that quantise one input at the same
// moment pass different `rot` and so read different lines of it at any time
// (the max and the integer sum do not depend on the order).
template <int NT>
__device__ __forceinline__ void gq_quantise_cta(const GqSegment& sg, uint8_t* xs, int xstride,
                                                float (*red_f)[NT], int (*red_i)[NT],
                                                float* s_a127, int* s_xsum, int tid,
                                                int nthreads, int rot) {
  const int warp = tid >> 5, lane = tid & 31, nwarps = nthreads >> 5;
  const int K4 = sg.K / 4, P4 = sg.chunks * (kGemvChunkK / 4);
  constexpr int R = kGqRegF4 / NT > 0 ? kGqRegF4 / NT : 1;   // float4s per thread and token
  constexpr int RB = R > 8 ? 8 : R;   // loads per thread in flight when reading in batches
  const bool in_regs = K4 <= R * nthreads;
  float4 v[NT][R];
  float m[NT];
#pragma unroll
  for (int t = 0; t < NT; ++t) m[t] = 0.0f;
  if (in_regs) {
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const float4* x4 = reinterpret_cast<const float4*>(sg.x + static_cast<int64_t>(t) * sg.K);
#pragma unroll
      for (int j = 0; j < R; ++j) {
        const int i = gq_rot(tid + j * nthreads, rot, K4);
        v[t][j] = i < K4 ? x4[i] : make_float4(0.f, 0.f, 0.f, 0.f);
        m[t] = fmaxf(m[t], absmax4(v[t][j]));
      }
    }
  } else {
    // longer rows: batches of RB loads per thread in flight, read again below
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const float4* x4 = reinterpret_cast<const float4*>(sg.x + static_cast<int64_t>(t) * sg.K);
#pragma unroll 1
      for (int b = tid; b < K4; b += RB * nthreads) {
        float4 w[RB];
#pragma unroll
        for (int j = 0; j < RB; ++j) {
          const int i = gq_rot(b + j * nthreads, rot, K4);
          w[j] = i < K4 ? x4[i] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int j = 0; j < RB; ++j) m[t] = fmaxf(m[t], absmax4(w[j]));
      }
    }
  }
#pragma unroll
  for (int t = 0; t < NT; ++t) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m[t] = fmaxf(m[t], __shfl_xor_sync(0xFFFFFFFFu, m[t], o));
    if (lane == 0) red_f[warp][t] = m[t];
  }
  __syncthreads();
  int sum[NT];
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    float mt = 0.0f;
    for (int w = 0; w < nwarps; ++w) mt = fmaxf(mt, red_f[w][t]);
    m[t] = mt;
    sum[t] = 0;
    const float s = mt == 0.0f ? 0.0f : __fdiv_rn(127.0f, mt);
    uint32_t* out = reinterpret_cast<uint32_t*>(xs + t * xstride);
    if (in_regs) {
#pragma unroll
      for (int j = 0; j < R; ++j) {
        const int i = gq_rot(tid + j * nthreads, rot, K4);
        if (i < K4) out[i] = mt == 0.0f ? 0u : quant_pack4(v[t][j], s, sum[t]);
      }
    } else {
      const float4* x4 = reinterpret_cast<const float4*>(sg.x + static_cast<int64_t>(t) * sg.K);
#pragma unroll 1
      for (int b = tid; b < K4; b += RB * nthreads) {
        float4 w[RB];
#pragma unroll
        for (int j = 0; j < RB; ++j) {
          const int i = gq_rot(b + j * nthreads, rot, K4);
          w[j] = i < K4 ? x4[i] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int j = 0; j < RB; ++j) {
          const int i = gq_rot(b + j * nthreads, rot, K4);
          if (i < K4) out[i] = mt == 0.0f ? 0u : quant_pack4(w[j], s, sum[t]);
        }
      }
    }
    for (int i = K4 + tid; i < P4; i += nthreads) out[i] = 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum[t] += __shfl_xor_sync(0xFFFFFFFFu, sum[t], o);
    if (lane == 0) red_i[warp][t] = sum[t];
  }
  __syncthreads();
  if (tid < NT) {
    int st = 0;
    for (int w = 0; w < nwarps; ++w) st += red_i[w][tid];
    s_a127[tid] = __fdiv_rn(m[tid], 127.0f);
    s_xsum[tid] = st;
  }
  __syncthreads();
}

// y (and acc) of one unit's rows: lane = row.
template <int NT>
__device__ __forceinline__ void gq_epilogue(const GqProblem& pr, int row, const int (&acc)[NT][4],
                                            const float* s_a127, const int* s_xsum) {
  if (row >= pr.M) return;
  const float alpha = *pr.alpha;
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    const int a = acc[t][0] + (acc[t][1] >> 2) + (acc[t][2] >> 4) + (acc[t][3] >> 6) - s_xsum[t];
    const float scale = __fmul_rn(alpha, s_a127[t]);
    const int64_t o = static_cast<int64_t>(t) * pr.M + row;
    pr.y[o] = __fmul_rn(__int2float_rn(a), scale);
    if (pr.acc) pr.acc[o] = a;
  }
}

// Warps a CTA may have: up to 12 for 1..4 tokens; 4 beyond, where each
// thread's accumulators take most of its registers.
__host__ __device__ constexpr int gq_max_warps(int nt) { return nt <= 4 ? kGqMaxWarps : 4; }

template <int NT>
__global__ void __launch_bounds__(32 * gq_max_warps(NT))
gemv_quant_kernel(const __grid_constant__ GqParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ float red_f[kGqMaxWarps][NT];
  __shared__ int red_i[kGqMaxWarps][NT];
  __shared__ float s_a127[NT];
  __shared__ int s_xsum[NT];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nwarps = blockDim.x >> 5;
  const uint32_t sw = static_cast<uint32_t>(lane & 7);
  uint8_t* xs = smem;
  int* part_all = reinterpret_cast<int*>(smem + NT * p.xstride);
  uint8_t* ring = smem + NT * p.xstride + gq_partial_bytes(NT, nwarps) + warp * kGqRingBytes;

  const int u0 = gq_unit_bound(p, blockIdx.x, gridDim.x);
  const int u1 = gq_unit_bound(p, blockIdx.x + 1, gridDim.x);
  const int seg0 = u0 < u1 ? gq_last_le(p.num_segments, u0,
                                        [&](int i) { return p.seg[i].unit_begin; })
                           : 0;

  // ---- copy side: this warp's pairs, item after item, kGqStages - 1 ahead.
  // (iu, ikc) is the unit and k-chunk of pair iq of the current item, kept
  // incrementally: one division per item, none per pair.
  int iseg = seg0;
  GqItem ii = gq_item(p, iseg, u0, u1, warp, nwarps);
  int iq = ii.qb;
  int iu = ii.ub + ii.qb / ii.chunks, ikc = ii.qb % ii.chunks;
  int ipi = p.seg[iseg].prob_begin;
  int iunit = -1;
  GqProblem ipr;
  GemvCopyPlan icp;
  // Moves the copy cursor to a pair that exists (skipping empty shares), or
  // past the CTA's last item; returns whether one exists.
  auto copy_valid = [&]() -> bool {
    while (u0 < u1 && iq >= ii.qe) {
      if (ii.ue >= u1 || iseg + 1 >= p.num_segments) return false;
      ii = gq_item(p, ++iseg, u0, u1, warp, nwarps);
      iq = ii.qb;
      iu = ii.ub + ii.qb / ii.chunks;
      ikc = ii.qb % ii.chunks;
    }
    return u0 < u1;
  };
  auto copy_plan_for = [&](int unit) {
    if (unit == iunit) return;
    iunit = unit;
    while (ipi + 1 < p.num_problems && p.prob[ipi + 1].unit_begin <= unit) ++ipi;
    ipr = p.prob[ipi];
    icp = gemv_plan(ipr, (unit - ipr.unit_begin) * kGemvTileRows, lane);
  };

  // L2 prefetch of the first stages (before the wait on the preceding kernel).
  // The problem cursor only moves forward, so it is put back afterwards: the
  // prefetched pairs may already reach the next problem.
  if (copy_valid()) {
    const int save_pi = ipi;
    int pq = iq, pu = iu, pkc = ikc;
#pragma unroll 1
    for (int st = 0; st < kGqStages - 1 && pq < ii.qe; ++st, ++pq) {
      copy_plan_for(pu);
      if (pkc * (kGemvChunkBytes / 4) + icp.wword < ipr.W) {
        const uint8_t* src = icp.wsrc + pkc * kGemvChunkBytes;
#pragma unroll 1
        for (int i = 0; i < icp.vrows; ++i)
          asm volatile("prefetch.global.L2 [%0];" ::"l"(src + i * icp.wstep) : "memory");
      }
      if (++pkc == ii.chunks) { pkc = 0; ++pu; }
    }
    ipi = save_pi;
    iunit = -1;
  }
  pdl_wait_prior_grid();
  pdl_allow_next_grid();
  if (u0 >= u1) return;   // the whole CTA: u0, u1 are uniform

  int slot = 0;
  auto issue_next = [&]() {
    if (copy_valid()) {
      copy_plan_for(iu);
      gemv_issue_weights(ipr.W, icp, ikc, ring + slot * kGqStageBytes);
      ++iq;
      if (++ikc == ii.chunks) { ikc = 0; ++iu; }
    }
    cp_async_commit();   // one group per stage, empty once the sequence is done
    slot = (slot + 1) & (kGqStages - 1);
  };
#pragma unroll 1
  for (int st = 0; st < kGqStages - 1; ++st) issue_next();

  // ---- consume side, item by item
  int cslot = 0;
  int cpi = p.seg[seg0].prob_begin;
  int* my_part = part_all + warp * (NT * 4 * 32);
#pragma unroll 1
  for (int cseg = seg0;; ++cseg) {
    const GqItem it = gq_item(p, cseg, u0, u1, warp, nwarps);
    __syncthreads();   // every warp is done with the previous item's int8 copy and partials
    // CTAs that start together read their common input from different offsets
    gq_quantise_cta<NT>(p.seg[cseg], xs, p.xstride, red_f, red_i, s_a127, s_xsum, tid,
                        32 * nwarps,
                        static_cast<int>(static_cast<int64_t>(blockIdx.x) *
                                         (p.seg[cseg].K / 4) / gridDim.x));

    int acc[NT][4];
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[t][j] = 0;
    const int C = it.chunks;
    int own_unit = -1;   // a unit this warp started at chunk 0 and left unfinished
    int q = it.qb;
#pragma unroll 1
    while (q < it.qe) {
      const int ul = q / C;                    // unit within the item
      const int c0 = q - ul * C;               // first chunk this warp takes of it
      const int c1 = min(C, it.qe - ul * C);   // one past the last
#pragma unroll 1
      for (int kc = c0; kc < c1; ++kc) {
        issue_next();
        cp_async_wait<kGqStages - 1>();
        __syncwarp();
        const uint8_t* st = ring + cslot * kGqStageBytes;
        cslot = (cslot + 1) & (kGqStages - 1);
        gemv_chunk_dot<NT>(st + lane * kGemvChunkBytes, sw, xs + kc * kGemvChunkK, p.xstride,
                           acc);
        __syncwarp();   // every lane is done with this stage before it is refilled
      }
      const int unit = it.ub + ul;
      if (c0 == 0 && c1 == C) {                // the whole unit: finish it here
        while (cpi + 1 < p.num_problems && p.prob[cpi + 1].unit_begin <= unit) ++cpi;
        const GqProblem pr = p.prob[cpi];
        gq_epilogue<NT>(pr, (unit - pr.unit_begin) * kGemvTileRows + lane, acc, s_a127,
                        s_xsum);
      } else if (c0 != 0) {                    // started mid-unit: leave the partial sums
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
          for (int j = 0; j < 4; ++j) my_part[(t * 4 + j) * 32 + lane] = acc[t][j];
      } else {                                 // holds chunk 0, ends early: finish it later
        own_unit = unit;
        break;                                 // (always this warp's last unit of the item)
      }
#pragma unroll
      for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[t][j] = 0;
      q = (ul + 1) * C;
    }
    __syncthreads();   // partial sums of split units are in shared memory
    if (own_unit >= 0) {
      // The warps after this one that start inside own_unit hold its other
      // k-chunks (every one of them started mid-unit and left its partial).
      const int ul = own_unit - it.ub;
      const int P = (it.ue - it.ub) * C;
#pragma unroll 1
      for (int w2 = warp + 1; w2 < nwarps; ++w2) {
        const int qb2 = static_cast<int>(static_cast<int64_t>(P) * w2 / nwarps);
        const int qe2 = static_cast<int>(static_cast<int64_t>(P) * (w2 + 1) / nwarps);
        if (qb2 >= (ul + 1) * C) break;
        if (qe2 > qb2) {
          const int* o = part_all + w2 * (NT * 4 * 32);
#pragma unroll
          for (int t = 0; t < NT; ++t)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[t][j] += o[(t * 4 + j) * 32 + lane];
        }
      }
      while (cpi + 1 < p.num_problems && p.prob[cpi + 1].unit_begin <= own_unit) ++cpi;
      const GqProblem pr = p.prob[cpi];
      gq_epilogue<NT>(pr, (own_unit - pr.unit_begin) * kGemvTileRows + lane, acc, s_a127,
                      s_xsum);
    }
    if (it.ue >= u1 || cseg + 1 >= p.num_segments) break;
  }
  cp_async_wait<0>();
}

}  // namespace bl
