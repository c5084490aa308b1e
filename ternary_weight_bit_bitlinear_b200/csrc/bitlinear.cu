// bitlinear.cu -- the C ABI of libbitlinear.so (declared in include/bitlinear.h):
// argument checks, problem tables, launch configuration and TMA descriptor
// set-up around the sm_100a kernels.  The weight-packing and quantiser kernels
// (pack.cuh, quant.cuh) are launched from here; the GEMV, fused decode, GEMM
// and TL2 kernels from their own units (launch_*.cu, see internal.h).
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <climits>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

#include "internal.h"
#include "gemm_small.cuh"
#include "pack.cuh"
#include "quant.cuh"

namespace blh {

namespace {
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mutex;
std::atomic<unsigned long long> g_wait_limit_ns{bl::kWaitLimitNs};
}  // namespace

bitlinear_status device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return BITLINEAR_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  DeviceInfo& d = g_dev[dev];
  if (d.sms == 0) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return BITLINEAR_ERR_CUDA;
    d.sms = sms;
  }
  *out = &d;
  return BITLINEAR_OK;
}

unsigned long long wait_limit_ns() { return g_wait_limit_ns.load(std::memory_order_relaxed); }

}  // namespace blh

namespace {

using blh::DeviceInfo;
using blh::device_info;
using blh::launch_pdl;
using blh::launch_status;
using blh::kMaxDevices;

constexpr int64_t kMaxK = 131072;
constexpr int64_t kMaxElems = int64_t(1) << 40;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// Words per packed row: K/16 rounded up to a multiple of 4 (16 bytes).
int64_t packed_row_words(int64_t K) { return 4 * ((K + 63) / 64); }

bitlinear_status check_mk(int64_t M, int64_t K) {
  if (M < 0 || K < 0) return BITLINEAR_ERR_INVALID_ARG;
  if (M == 0 || K == 0 || K % 16 != 0 || K > kMaxK) return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
  if (M > INT_MAX / 2 || M * K > kMaxElems) return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
  return BITLINEAR_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

// 2-D uint8 tensor [rows][cols] with row pitch `cols` bytes, box {box_cols, box_rows}.
bool encode_u8_2d(CUtensorMap* map, const void* ptr, uint64_t cols, uint64_t rows,
                  uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swizzle) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Decode GEMV over problems that share N (all validated): one launch
// per kGemvMaxProblems problems, units of 32 rows numbered across problems.
bitlinear_status gemv_group(const bitlinear_problem* probs, int64_t count, int64_t N,
                            cudaStream_t s) {
  DeviceInfo* dev = nullptr;
  bitlinear_status st = device_info(&dev);
  if (st != BITLINEAR_OK) return st;
  for (int64_t base = 0; base < count; base += bl::kGemvMaxProblems) {
    const int n = static_cast<int>(count - base < bl::kGemvMaxProblems
                                       ? count - base : bl::kGemvMaxProblems);
    bl::GemvParams p;
    memset(&p, 0, sizeof p);
    int64_t units = 0;
    for (int i = 0; i < n; ++i) {
      const bitlinear_problem& q = probs[base + i];
      bl::GemvProblem& g = p.prob[i];
      g.packed = q.packed;
      g.alpha = q.alpha;
      g.xq = q.xq;
      g.amax = q.amax;
      g.xsum = q.xsum;
      g.y = q.y;
      g.acc = q.acc;
      g.M = static_cast<int>(q.M);
      g.K = static_cast<int>(q.K);
      g.W = static_cast<int>(packed_row_words(q.K));
      g.unit_begin = static_cast<int>(units);
      units += (q.M + bl::kGemvTileRows - 1) / bl::kGemvTileRows;
    }
    if (units > INT_MAX) return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
    p.num_problems = n;
    p.total_units = static_cast<int>(units);
    st = blh::launch_gemv(static_cast<int>(N), p, dev, s);
    if (st != BITLINEAR_OK) return st;
  }
  return BITLINEAR_OK;
}

// 2-D fp32 tensor [rows][cols], box {box_cols, box_rows}, no swizzle.
bool encode_f32_2d(CUtensorMap* map, const void* ptr, uint64_t cols, uint64_t rows,
                   uint32_t box_cols, uint32_t box_rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 4};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(ptr), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bitlinear_status check_matmul_args(const uint32_t* packed, const float* alpha, int64_t M,
                                   int64_t K, const int8_t* xq, const float* amax,
                                   const int32_t* xsum, int64_t N, float* y, int32_t* acc) {
  bitlinear_status st = check_mk(M, K);
  if (st != BITLINEAR_OK) return st;
  if (N < 0) return BITLINEAR_ERR_INVALID_ARG;
  if (N == 0) return BITLINEAR_OK;
  if (N > INT_MAX / 2) return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
  if (!packed || !alpha || !xq || !amax || !xsum || !y) return BITLINEAR_ERR_INVALID_ARG;
  if (!aligned16(packed) || !aligned16(xq) || !aligned16(y) || (acc && !aligned16(acc)))
    return BITLINEAR_ERR_MISALIGNED;
  if (!aligned4(alpha) || !aligned4(amax) || !aligned4(xsum)) return BITLINEAR_ERR_MISALIGNED;
  return BITLINEAR_OK;
}

bitlinear_status check_problem(const bitlinear_problem& q, int64_t N) {
  return check_matmul_args(q.packed, q.alpha, q.M, q.K, q.xq, q.amax, q.xsum, N, q.y, q.acc);
}

// Longest-processing-time-first schedule: tiles (already ordered by K,
// descending) go one by one to the CTA with the least work so far (cost = K,
// the tile's main-loop length).  Skipped when the grid or the tile count does
// not fit the parameter tables; the kernel then takes tiles round-robin.
void build_gemm_schedule(bl::GemmParams& p, int sms) {
  const int grid = p.total_tiles < sms ? p.total_tiles : sms;
  p.use_sched = 0;
  if (grid > bl::kGemmMaxGrid || p.total_tiles > bl::kGemmMaxSched || p.num_problems < 2) return;
  std::vector<std::pair<int64_t, int>> heap;   // (load, cta), min-heap
  heap.reserve(grid);
  for (int c = 0; c < grid; ++c) heap.push_back({0, c});
  std::vector<int> owner(p.total_tiles);
  std::vector<int> count(grid, 0);
  auto cmp = [](const std::pair<int64_t, int>& a, const std::pair<int64_t, int>& b) {
    return a.first != b.first ? a.first > b.first : a.second > b.second;
  };
  std::make_heap(heap.begin(), heap.end(), cmp);
  for (int pi = 0; pi < p.num_problems; ++pi) {
    const bl::GemmProblem& g = p.prob[pi];
    const int end = pi + 1 < p.num_problems ? p.prob[pi + 1].tile_begin : p.total_tiles;
    for (int t = g.tile_begin; t < end; ++t) {
      std::pop_heap(heap.begin(), heap.end(), cmp);
      auto& least = heap.back();
      owner[t] = least.second;
      count[least.second] += 1;
      least.first += g.K;
      std::push_heap(heap.begin(), heap.end(), cmp);
    }
  }
  p.sched_begin[0] = 0;
  for (int c = 0; c < grid; ++c)
    p.sched_begin[c + 1] = static_cast<uint16_t>(p.sched_begin[c] + count[c]);
  std::vector<int> fill(p.sched_begin, p.sched_begin + grid);
  for (int pi = 0; pi < p.num_problems; ++pi) {
    const bl::GemmProblem& g = p.prob[pi];
    const int end = pi + 1 < p.num_problems ? p.prob[pi + 1].tile_begin : p.total_tiles;
    for (int t = g.tile_begin; t < end; ++t) {
      const int lt = t - g.tile_begin;
      p.sched[fill[owner[t]]++] = bl::gemm_sched_entry(pi, lt / g.n_tiles, lt % g.n_tiles);
    }
  }
  p.use_sched = 1;
}

// Tensor-core GEMM over problems that share N (all validated): one
// persistent launch per kGemmMaxProblems problems, tiles numbered across
// problems with the largest K first so the longest tiles start in the first
// wave.  Ragged edges come from the tensor maps: loads past M, K or N read
// zeros, and stores past M or N are dropped.  A y whose row pitch (4M bytes)
// is not a multiple of 16 cannot be a TMA tensor; its epilogue stores directly.
bitlinear_status gemm_group(const bitlinear_problem* probs, int64_t count, int64_t N,
                            cudaStream_t s) {
  DeviceInfo* dev = nullptr;
  bitlinear_status st = device_info(&dev);
  if (st != BITLINEAR_OK) return st;
  // Up to 32 tokens: one 128-row tile of all tokens per CTA, the expanded
  // weights in tensor memory (gemm_small.cuh), 16 or 32 tokens wide.  Wide
  // token blocks: 256-token tiles on CTA pairs.  In between: one CTA per
  // 128-row tile, 64 or 128 tokens wide -- the narrower the tile, the smaller
  // its activation stage and the deeper the ring of weight stages the same
  // shared memory holds.
  const bool small = N <= 32;
  const bool wide = N > 128;
  const int BN = small ? (N <= 16 ? 16 : 32) : wide ? bl::kPairBN : N <= 64 ? 64 : 128;
  const int BMt = wide ? bl::kPairBM : bl::kGemmBM;
  const int64_t n_tiles = (N + BN - 1) / BN;
  for (int64_t base = 0; base < count; base += bl::kGemmMaxProblems) {
    const int n = static_cast<int>(count - base < bl::kGemmMaxProblems
                                       ? count - base : bl::kGemmMaxProblems);
    int order[bl::kGemmMaxProblems];
    for (int i = 0; i < n; ++i) order[i] = i;
    for (int i = 1; i < n; ++i)   // insertion sort by K, descending (stable)
      for (int j = i; j > 0 && probs[base + order[j]].K > probs[base + order[j - 1]].K; --j) {
        const int t = order[j];
        order[j] = order[j - 1];
        order[j - 1] = t;
      }
    bl::GemmParams p;
    memset(&p, 0, sizeof p);
    int64_t tiles = 0;
    for (int i = 0; i < n; ++i) {
      const bitlinear_problem& q = probs[base + order[i]];
      const bool direct = small || q.M % 4 != 0;   // the small kernel stores directly
      // packed weights: one k-block (32 bytes) per row, or for the small kernel
      // four k-blocks (128 bytes, swizzled) per row
      if (!encode_u8_2d(&p.tmA[i], q.packed, static_cast<uint64_t>(packed_row_words(q.K) * 4),
                        static_cast<uint64_t>(q.M),
                        small ? bl::kSmallGroupBytes : bl::kGemmPackedRowBytes, bl::kGemmBM,
                        small ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE) ||
          !encode_u8_2d(&p.tmB[i], q.xq, static_cast<uint64_t>(q.K), static_cast<uint64_t>(N),
                        bl::kGemmBK, wide ? bl::kPairHalfN : BN,
                        CU_TENSOR_MAP_SWIZZLE_128B) ||
          (!direct && !encode_f32_2d(&p.tmY[i], q.y, static_cast<uint64_t>(q.M),
                                     static_cast<uint64_t>(N), 32, 32)))
        return BITLINEAR_ERR_CUDA;
      bl::GemmProblem& g = p.prob[i];
      g.alpha = q.alpha;
      g.amax = q.amax;
      g.xsum = q.xsum;
      g.y = q.y;
      g.acc = q.acc;
      g.M = static_cast<int>(q.M);
      g.K = static_cast<int>(q.K);
      g.N = static_cast<int>(N);
      g.n_tiles = static_cast<int>(n_tiles);
      g.tile_begin = static_cast<int>(tiles);
      g.direct_store = direct ? 1 : 0;
      tiles += (q.M + BMt - 1) / BMt * n_tiles;
    }
    if (tiles > INT_MAX) return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
    p.num_problems = n;
    p.total_tiles = static_cast<int>(tiles);
    p.wait_ns = blh::wait_limit_ns();
    build_gemm_schedule(p, wide ? dev->sms / 2 : dev->sms);
    st = blh::launch_gemm(small ? (BN == 16 ? 4 : 5) : wide ? 1 : BN == 64 ? 3 : 0, p, dev, s);
    if (st != BITLINEAR_OK) return st;
  }
  return BITLINEAR_OK;
}

// ---- decode GEMV with the quantiser fused in

bitlinear_status check_fused_problem(const bitlinear_fused_problem& q, int64_t N) {
  bitlinear_status st = check_mk(q.M, q.K);
  if (st != BITLINEAR_OK) return st;
  if (!q.packed || !q.alpha || !q.x || !q.y) return BITLINEAR_ERR_INVALID_ARG;
  if (!aligned16(q.packed) || !aligned16(q.x) || !aligned16(q.y) || (q.acc && !aligned16(q.acc)))
    return BITLINEAR_ERR_MISALIGNED;
  if (!aligned4(q.alpha)) return BITLINEAR_ERR_MISALIGNED;
  const int64_t kpad = (q.K + bl::kGemvChunkK - 1) / bl::kGemvChunkK * bl::kGemvChunkK;
  if (N * kpad > bl::kGqMaxXBytes) return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
  return BITLINEAR_OK;
}

// Plan of one fused launch: its problems and segments (runs of consecutive
// problems on one input), the CTA size with the most warps resident per SM
// (fewest warps per CTA on a tie: more CTAs to share the work), and each CTA's
// range of units, cut so that every range holds about the same number of
// (unit, k-chunk) pairs.
bitlinear_status gemv_quant_plan(const bitlinear_fused_problem* probs, int n, int nt,
                                 DeviceInfo* dev, bl::GqParams& p, int* grid, int* warps) {
  memset(&p, 0, sizeof p);
  int64_t units = 0, kmax = 0;
  int segs = 0;
  std::vector<int64_t> seg_pairs;
  for (int i = 0; i < n; ++i) {
    const bitlinear_fused_problem& q = probs[i];
    bl::GqProblem& g = p.prob[i];
    g.packed = q.packed;
    g.alpha = q.alpha;
    g.y = q.y;
    g.acc = q.acc;
    g.M = static_cast<int>(q.M);
    g.W = static_cast<int>(packed_row_words(q.K));
    g.unit_begin = static_cast<int>(units);
    const int64_t u = (q.M + bl::kGemvTileRows - 1) / bl::kGemvTileRows;
    const bool same = segs > 0 && p.seg[segs - 1].x == q.x && p.seg[segs - 1].K == q.K;
    if (!same) {
      bl::GqSegment& sg = p.seg[segs++];
      sg.x = q.x;
      sg.K = static_cast<int>(q.K);
      sg.chunks = static_cast<int>((q.K + bl::kGemvChunkK - 1) / bl::kGemvChunkK);
      sg.unit_begin = static_cast<int>(units);
      sg.prob_begin = i;
      seg_pairs.push_back(0);
    }
    p.seg[segs - 1].units += static_cast<int>(u);
    seg_pairs.back() += u * p.seg[segs - 1].chunks;
    units += u;
    kmax = std::max<int64_t>(kmax, q.K);
    if (units > INT_MAX / 2) return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
  }
  p.num_problems = n;
  p.num_segments = segs;
  p.xstride = static_cast<int>((kmax + bl::kGemvChunkK - 1) / bl::kGemvChunkK * bl::kGemvChunkK);
  // CTA size: the most warps resident per SM, among sizes that fit at least
  // two CTAs per SM when there are any (a CTA that starts on an SM quantises
  // its input while the other one streams weights); on a tie, the most warps
  // per CTA (fewer CTAs quantise each input, and each CTA's range is longer).
  // The 70B-shaped stream then runs 2 CTAs of 6 warps per SM rather than 3 of
  // 4 (6635-6644 against 6624 GB/s; the 2B-shaped stream 5617-5633 against
  // 5570-5590, on one box).
  int best_w = 0, best_per_sm = 0, best_score = 0;
  for (int w = 4; w <= bl::gq_max_warps(nt); ++w) {
    int per_sm = 0;
    bitlinear_status st =
        blh::gemv_quant_occupancy(nt, w, bl::gq_smem_bytes(nt, w, p.xstride), dev, &per_sm);
    if (st != BITLINEAR_OK) return st;
    const int score = per_sm * w + (per_sm >= 2 ? 1000 : 0);
    if (per_sm > 0 && score >= best_score) {
      best_score = score;
      best_w = w;
      best_per_sm = per_sm;
    }
  }
  if (best_w == 0) return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
  p.area = bl::gq_smem_bytes(nt, best_w, p.xstride);
  // One CTA per resident slot, at most one per unit.
  p.total_units = static_cast<int>(units);
  int64_t total = 0;
  for (int g = 0; g < segs; ++g) {
    p.seg[g].pair_begin = total;
    total += seg_pairs[g];
  }
  p.total_pairs = total;
  const int64_t slots = static_cast<int64_t>(dev->sms) * best_per_sm;
  *grid = static_cast<int>(std::min<int64_t>(std::min<int64_t>(slots, units), INT_MAX / 2));
  *warps = best_w;
  return BITLINEAR_OK;
}

// Fused decode over validated problems sharing N: one launch per at most
// kGqMaxProblems problems.
bitlinear_status gemv_quant_group(const bitlinear_fused_problem* probs, int64_t count,
                                  int64_t N, cudaStream_t s) {
  DeviceInfo* dev = nullptr;
  bitlinear_status st = device_info(&dev);
  if (st != BITLINEAR_OK) return st;
  const int nt = static_cast<int>(N);
  bl::GqParams p;
  for (int64_t base = 0; base < count; base += bl::kGqMaxProblems) {
    const int n = static_cast<int>(std::min<int64_t>(count - base, bl::kGqMaxProblems));
    int grid = 0, warps = 0;
    st = gemv_quant_plan(probs + base, n, nt, dev, p, &grid, &warps);
    if (st != BITLINEAR_OK) return st;
    st = blh::gemv_quant_launch(nt, grid, warps, p, s);
    if (st != BITLINEAR_OK) return st;
  }
  return BITLINEAR_OK;
}

// ---- TL2-style storage

bitlinear_status check_tl2_problem(const bitlinear_tl2_problem& q, int64_t N) {
  bitlinear_status st = check_mk(q.M, q.K);
  if (st != BITLINEAR_OK) return st;
  if (!q.tl2 || !q.alpha || !q.xq || !q.amax || !q.y) return BITLINEAR_ERR_INVALID_ARG;
  if (!aligned16(q.tl2) || !aligned16(q.xq) || !aligned16(q.y) || (q.acc && !aligned16(q.acc)))
    return BITLINEAR_ERR_MISALIGNED;
  if (!aligned4(q.alpha) || !aligned4(q.amax)) return BITLINEAR_ERR_MISALIGNED;
  (void)N;
  return BITLINEAR_OK;
}

bitlinear_status gemv_tl2_group(const bitlinear_tl2_problem* probs, int64_t count, int64_t N,
                                cudaStream_t s) {
  DeviceInfo* dev = nullptr;
  bitlinear_status st = device_info(&dev);
  if (st != BITLINEAR_OK) return st;
  for (int64_t base = 0; base < count; base += bl::kTl2MaxProblems) {
    const int n = static_cast<int>(count - base < bl::kTl2MaxProblems
                                       ? count - base : bl::kTl2MaxProblems);
    bl::Tl2Params p;
    memset(&p, 0, sizeof p);
    int64_t units = 0;
    for (int i = 0; i < n; ++i) {
      const bitlinear_tl2_problem& q = probs[base + i];
      bl::Tl2Problem& g = p.prob[i];
      g.tl2 = q.tl2;
      g.alpha = q.alpha;
      g.xq = q.xq;
      g.amax = q.amax;
      g.y = q.y;
      g.acc = q.acc;
      g.M = static_cast<int>(q.M);
      g.K = static_cast<int>(q.K);
      g.nb = static_cast<int>(bl::tl2_blocks(q.K));
      g.row_bytes = static_cast<int>(bl::tl2_row_bytes(q.K));
      g.sign_off = static_cast<int>(bl::tl2_sign_offset(q.K));
      g.tail_off = static_cast<int>(bl::tl2_tail_offset(q.K));
      g.unit_begin = static_cast<int>(units);
      units += (q.M + bl::kGemvTileRows - 1) / bl::kGemvTileRows;
    }
    if (units > INT_MAX) return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
    p.num_problems = n;
    p.total_units = static_cast<int>(units);
    st = blh::launch_gemv_tl2(static_cast<int>(N), p, dev, s);
    if (st != BITLINEAR_OK) return st;
  }
  return BITLINEAR_OK;
}

}  // namespace

extern "C" {

const char* bitlinear_status_string(int status) {
  switch (status) {
    case BITLINEAR_OK: return "ok";
    case BITLINEAR_ERR_INVALID_ARG: return "invalid argument";
    case BITLINEAR_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case BITLINEAR_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case BITLINEAR_ERR_WORKSPACE: return "workspace missing or too small";
    case BITLINEAR_ERR_CUDA: return "CUDA error";
    case BITLINEAR_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case BITLINEAR_ERR_NONFINITE: return "non-finite weights (inf or NaN)";
    default: return "unknown status";
  }
}

int bitlinear_version(void) { return 101; }

size_t bitlinear_pack_workspace_bytes(int64_t M, int64_t K) {
  (void)M;
  (void)K;
  return bl::kPackWorkspaceBytes;
}

bitlinear_status bitlinear_pack_weights(const float* W, int64_t M, int64_t K, uint32_t* packed,
                                        float* alpha, void* workspace, size_t workspace_bytes,
                                        bitlinear_stream_t stream) {
  bitlinear_status st = check_mk(M, K);
  if (st != BITLINEAR_OK) return st;
  if (!W || !packed || !alpha) return BITLINEAR_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < bl::kPackWorkspaceBytes) return BITLINEAR_ERR_WORKSPACE;
  if (!aligned16(W) || !aligned16(packed) || !aligned16(workspace) || !aligned4(alpha))
    return BITLINEAR_ERR_MISALIGNED;
  DeviceInfo* dev = nullptr;
  if ((st = device_info(&dev)) != BITLINEAR_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  auto* bins = static_cast<unsigned long long*>(workspace);
  auto* flag = reinterpret_cast<unsigned int*>(bins + bl::kBins);
  if (cudaMemsetAsync(workspace, 0, bl::kPackWorkspaceBytes, s) != cudaSuccess)
    return BITLINEAR_ERR_CUDA;
  const int64_t n4 = M * K / 4;
  int grid = dev->sms * 4;
  bl::abs_bins_kernel<<<grid, bl::kBinsThreads, 0, s>>>(reinterpret_cast<const float4*>(W), n4,
                                                         bins, flag);
  bl::alpha_finalize_kernel<<<1, 32, 0, s>>>(bins, flag, static_cast<uint64_t>(M * K), alpha);
  const int64_t wp = packed_row_words(K);
  const int64_t words = M * wp;
  int64_t g = (words + 255) / 256;
  if (g > dev->sms * 16) g = dev->sms * 16;
  bl::ternarize_pack_kernel<<<static_cast<int>(g), 256, 0, s>>>(
      reinterpret_cast<const float4*>(W), M, static_cast<int>(K / 16), static_cast<int>(wp),
      alpha, packed);
  return launch_status();
}

bitlinear_status bitlinear_quant_act(const float* x, int64_t N, int64_t K, int8_t* xq,
                                     float* amax, int32_t* xsum, bitlinear_stream_t stream) {
  const bitlinear_act a = {x, N, K, xq, amax, xsum};
  return bitlinear_quant_act_grouped(&a, 1, stream);
}

// The row quantiser over `rows` rows, the widest kmax wide: when the rows do
// not fill the SMs (each row's latency is then the launch's), CTAs wide
// enough to hold the row in registers; 256-thread CTAs otherwise.
static cudaError_t launch_quant_rows(int rows, int64_t kmax, const DeviceInfo* dev,
                                     cudaStream_t s, const bl::QuantParams& p) {
  const int threads = rows < dev->sms ? bl::quant_wide_threads(kmax) : bl::kQuantThreads;
  if (threads == 1024)
    return launch_pdl(bl::quant_rows_kernel<1024>, rows, 1024, 0, s, p);
  if (threads == 512) return launch_pdl(bl::quant_rows_kernel<512>, rows, 512, 0, s, p);
  return launch_pdl(bl::quant_rows_kernel<256>, rows, 256, 0, s, p);
}

bitlinear_status bitlinear_quant_act_grouped(const bitlinear_act* acts, int64_t count,
                                             bitlinear_stream_t stream) {
  if (count < 0 || (count > 0 && !acts)) return BITLINEAR_ERR_INVALID_ARG;
  for (int64_t i = 0; i < count; ++i) {
    const bitlinear_act& a = acts[i];
    if (a.N < 0 || a.K < 0) return BITLINEAR_ERR_INVALID_ARG;
    if (a.K == 0 || a.K % 16 != 0 || a.K > kMaxK || a.N > INT_MAX)
      return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
    if (a.N == 0) continue;
    if (!a.x || !a.xq || !a.amax) return BITLINEAR_ERR_INVALID_ARG;
    if (!aligned16(a.x) || !aligned16(a.xq) || !aligned4(a.amax) || (a.xsum && !aligned4(a.xsum)))
      return BITLINEAR_ERR_MISALIGNED;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  bl::QuantParams p;
  memset(&p, 0, sizeof p);
  int64_t rows = 0, kmax = 0;
  DeviceInfo* dev = nullptr;
  auto flush = [&]() -> bitlinear_status {
    if (p.count == 0) return BITLINEAR_OK;
    if (!dev) {
      const bitlinear_status dst = device_info(&dev);
      if (dst != BITLINEAR_OK) return dst;
    }
    const cudaError_t e = launch_quant_rows(static_cast<int>(rows), kmax, dev, s, p);
    memset(&p, 0, sizeof p);
    rows = 0;
    kmax = 0;
    return e == cudaSuccess ? launch_status() : BITLINEAR_ERR_CUDA;
  };
  for (int64_t i = 0; i < count; ++i) {
    const bitlinear_act& a = acts[i];
    if (a.N == 0) continue;
    if (p.count == bl::kQuantMaxMatrices || rows + a.N > INT_MAX) {
      bitlinear_status st = flush();
      if (st != BITLINEAR_OK) return st;
    }
    bl::QuantMatrix& m = p.m[p.count++];
    m.x = a.x;
    m.xq = a.xq;
    m.amax = a.amax;
    m.xsum = a.xsum;
    m.K = static_cast<int>(a.K);
    m.row_begin = static_cast<int>(rows);
    rows += a.N;
    kmax = std::max<int64_t>(kmax, a.K);
  }
  return flush();
}

size_t bitlinear_quant_act_per_tensor_workspace_bytes(void) { return 16; }

bitlinear_status bitlinear_quant_act_per_tensor(const float* x, int64_t N, int64_t K, int8_t* xq,
                                                float* amax, int32_t* xsum, void* workspace,
                                                size_t workspace_bytes,
                                                bitlinear_stream_t stream) {
  if (N < 0 || K < 0) return BITLINEAR_ERR_INVALID_ARG;
  if (K == 0 || K % 16 != 0 || K > kMaxK || N > INT_MAX) return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
  if (N == 0) return BITLINEAR_OK;
  if (!x || !xq || !amax) return BITLINEAR_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < 16) return BITLINEAR_ERR_WORKSPACE;
  if (!aligned16(x) || !aligned16(xq) || !aligned4(amax) || (xsum && !aligned4(xsum)) ||
      !aligned16(workspace))
    return BITLINEAR_ERR_MISALIGNED;
  DeviceInfo* dev = nullptr;
  bitlinear_status st = device_info(&dev);
  if (st != BITLINEAR_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  auto* word = static_cast<unsigned int*>(workspace);
  if (cudaMemsetAsync(word, 0, 4, s) != cudaSuccess) return BITLINEAR_ERR_CUDA;
  const int64_t n4 = N * K / 4;
  int64_t g = (n4 + bl::kQuantThreads - 1) / bl::kQuantThreads;
  if (g > dev->sms * 8) g = dev->sms * 8;
  if (launch_pdl(bl::tensor_absmax_kernel, static_cast<int>(g), bl::kQuantThreads, 0, s,
                 reinterpret_cast<const float4*>(x), n4, word) != cudaSuccess)
    return BITLINEAR_ERR_CUDA;
  bl::QuantParams p;
  memset(&p, 0, sizeof p);
  p.count = 1;
  p.m[0].x = x;
  p.m[0].xq = xq;
  p.m[0].amax = amax;
  p.m[0].xsum = xsum;
  p.m[0].tensor_amax = word;
  p.m[0].K = static_cast<int>(K);
  p.m[0].row_begin = 0;
  if (launch_quant_rows(static_cast<int>(N), K, dev, s, p) != cudaSuccess)
    return BITLINEAR_ERR_CUDA;
  return launch_status();
}

bitlinear_status bitlinear_gemv(const uint32_t* packed, const float* alpha, int64_t M, int64_t K,
                                const int8_t* xq, const float* amax, const int32_t* xsum,
                                int64_t N, float* y, int32_t* acc, bitlinear_stream_t stream) {
  bitlinear_status st = check_matmul_args(packed, alpha, M, K, xq, amax, xsum, N, y, acc);
  if (st != BITLINEAR_OK || N == 0) return st;
  if (N > bl::kGemvMaxTokens) return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
  const bitlinear_problem q = {packed, alpha, M, K, xq, amax, xsum, y, acc};
  return gemv_group(&q, 1, N, reinterpret_cast<cudaStream_t>(stream));
}

bitlinear_status bitlinear_gemv_grouped(const bitlinear_problem* problems, int64_t count,
                                        int64_t N, bitlinear_stream_t stream) {
  if (count < 0 || N < 0 || (count > 0 && !problems)) return BITLINEAR_ERR_INVALID_ARG;
  if (count == 0 || N == 0) return BITLINEAR_OK;
  if (N > bl::kGemvMaxTokens) return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
  for (int64_t i = 0; i < count; ++i) {
    bitlinear_status st = check_problem(problems[i], N);
    if (st != BITLINEAR_OK) return st;
  }
  return gemv_group(problems, count, N, reinterpret_cast<cudaStream_t>(stream));
}

bitlinear_status bitlinear_gemm(const uint32_t* packed, const float* alpha, int64_t M, int64_t K,
                                const int8_t* xq, const float* amax, const int32_t* xsum,
                                int64_t N, float* y, int32_t* acc, bitlinear_stream_t stream) {
  bitlinear_status st = check_matmul_args(packed, alpha, M, K, xq, amax, xsum, N, y, acc);
  if (st != BITLINEAR_OK || N == 0) return st;
  const bitlinear_problem q = {packed, alpha, M, K, xq, amax, xsum, y, acc};
  return gemm_group(&q, 1, N, reinterpret_cast<cudaStream_t>(stream));
}

bitlinear_status bitlinear_gemm_grouped(const bitlinear_problem* problems, int64_t count,
                                        int64_t N, bitlinear_stream_t stream) {
  if (count < 0 || N < 0 || (count > 0 && !problems)) return BITLINEAR_ERR_INVALID_ARG;
  if (count == 0 || N == 0) return BITLINEAR_OK;
  for (int64_t i = 0; i < count; ++i) {
    bitlinear_status st = check_problem(problems[i], N);
    if (st != BITLINEAR_OK) return st;
  }
  return gemm_group(problems, count, N, reinterpret_cast<cudaStream_t>(stream));
}

bitlinear_status bitlinear_gemv_quant(const uint32_t* packed, const float* alpha, int64_t M,
                                      int64_t K, const float* x, int64_t N, float* y,
                                      int32_t* acc, bitlinear_stream_t stream) {
  if (N < 0) return BITLINEAR_ERR_INVALID_ARG;
  if (N > bl::kGemvMaxTokens) return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
  const bitlinear_fused_problem q = {packed, alpha, M, K, x, y, acc};
  if (N == 0) return check_mk(M, K);
  bitlinear_status st = check_fused_problem(q, N);
  if (st != BITLINEAR_OK) return st;
  return gemv_quant_group(&q, 1, N, reinterpret_cast<cudaStream_t>(stream));
}

bitlinear_status bitlinear_gemv_quant_grouped(const bitlinear_fused_problem* problems,
                                              int64_t count, int64_t N,
                                              bitlinear_stream_t stream) {
  if (count < 0 || N < 0 || (count > 0 && !problems)) return BITLINEAR_ERR_INVALID_ARG;
  if (count == 0 || N == 0) return BITLINEAR_OK;
  if (N > bl::kGemvMaxTokens) return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
  for (int64_t i = 0; i < count; ++i) {
    bitlinear_status st = check_fused_problem(problems[i], N);
    if (st != BITLINEAR_OK) return st;
  }
  return gemv_quant_group(problems, count, N, reinterpret_cast<cudaStream_t>(stream));
}

size_t bitlinear_tl2_row_bytes(int64_t K) {
  if (K <= 0 || K % 16 != 0 || K > kMaxK) return 0;
  return static_cast<size_t>(bl::tl2_row_bytes(K));
}

bitlinear_status bitlinear_tl2_from_packed(const uint32_t* packed, int64_t M, int64_t K,
                                           uint8_t* tl2, bitlinear_stream_t stream) {
  bitlinear_status st = check_mk(M, K);
  if (st != BITLINEAR_OK) return st;
  if (!packed || !tl2) return BITLINEAR_ERR_INVALID_ARG;
  if (!aligned16(packed) || !aligned16(tl2)) return BITLINEAR_ERR_MISALIGNED;
  DeviceInfo* dev = nullptr;
  if ((st = device_info(&dev)) != BITLINEAR_OK) return st;
  const int64_t nb = bl::tl2_blocks(K);
  const int64_t total = M * (nb + (K - bl::kTl2Block * nb + 63) / 64);
  int64_t g = (total + 255) / 256;
  if (g > dev->sms * 16) g = dev->sms * 16;
  return blh::launch_tl2_convert(packed, M, K, static_cast<int>(packed_row_words(K)), tl2,
                                 static_cast<int>(g), reinterpret_cast<cudaStream_t>(stream));
}

bitlinear_status bitlinear_gemv_tl2(const uint8_t* tl2, const float* alpha, int64_t M, int64_t K,
                                    const int8_t* xq, const float* amax, int64_t N, float* y,
                                    int32_t* acc, bitlinear_stream_t stream) {
  if (N < 0) return BITLINEAR_ERR_INVALID_ARG;
  if (N > bl::kGemvMaxTokens) return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
  const bitlinear_tl2_problem q = {tl2, alpha, M, K, xq, amax, y, acc};
  if (N == 0) return check_mk(M, K);
  bitlinear_status st = check_tl2_problem(q, N);
  if (st != BITLINEAR_OK) return st;
  return gemv_tl2_group(&q, 1, N, reinterpret_cast<cudaStream_t>(stream));
}

bitlinear_status bitlinear_gemv_tl2_grouped(const bitlinear_tl2_problem* problems, int64_t count,
                                            int64_t N, bitlinear_stream_t stream) {
  if (count < 0 || N < 0 || (count > 0 && !problems)) return BITLINEAR_ERR_INVALID_ARG;
  if (count == 0 || N == 0) return BITLINEAR_OK;
  if (N > bl::kGemvMaxTokens) return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
  for (int64_t i = 0; i < count; ++i) {
    bitlinear_status st = check_tl2_problem(problems[i], N);
    if (st != BITLINEAR_OK) return st;
  }
  return gemv_tl2_group(problems, count, N, reinterpret_cast<cudaStream_t>(stream));
}

bitlinear_status bitlinear_device_error(int* status_out, int clear) {
  if (!status_out) return BITLINEAR_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return BITLINEAR_ERR_CUDA;
  // One error word per unit of the library; this unit's holds the pack step's.
  unsigned int v = 0, w = 0;
  if (blh::read_error_word(bl::g_device_error, &w, clear != 0) != cudaSuccess)
    return BITLINEAR_ERR_CUDA;
  v |= w;
  cudaError_t (*const readers[])(unsigned int*, bool) = {
      blh::device_error_gemv, blh::device_error_gemv_quant, blh::device_error_gemm,
      blh::device_error_tl2};
  for (auto rd : readers) {
    w = 0;
    if (rd(&w, clear != 0) != cudaSuccess) return BITLINEAR_ERR_CUDA;
    v |= w;
  }
  *status_out = (v & bl::kDeviceTimeout)     ? BITLINEAR_ERR_DEVICE_TIMEOUT
                : (v & bl::kDeviceNonFinite) ? BITLINEAR_ERR_NONFINITE
                                             : BITLINEAR_OK;
  return BITLINEAR_OK;
}

unsigned long long bitlinear_set_wait_limit(unsigned long long limit_ns) {
  const unsigned long long v = limit_ns ? limit_ns : bl::kWaitLimitNs;
  return blh::g_wait_limit_ns.exchange(v);
}

}  // extern "C"
// ---------------------------------------------------------------- no-alloc pack
// Scratch of bitlinear_pack_weights_noalloc: the exponent bins and flag word
// that bitlinear_pack_weights otherwise takes as workspace.  One copy per
// device, shared by every call on that device.
static __device__ __align__(256) unsigned char g_noalloc_pack_scratch[bl::kPackWorkspaceBytes];

namespace {
// Device address of the scratch array for the current device.  Host code may
// not pass the symbol itself to a kernel: on the host it names a stand-in,
// not device memory.  Looked up on every call, with the caller's device
// current, so a device reset or a new primary context never leaves a stale
// address behind (the lookup is a host-side table read once the module is
// loaded).
bitlinear_status noalloc_pack_scratch(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_pack_scratch) != cudaSuccess || !p)
    return BITLINEAR_ERR_CUDA;
  *out = p;
  return BITLINEAR_OK;
}
}  // namespace

extern "C" bitlinear_status bitlinear_pack_weights_noalloc(const float* W, int64_t M, int64_t K,
                                                           uint32_t* packed, float* alpha,
                                                           bitlinear_stream_t stream) {
  // Argument checks first, so a bad call touches no CUDA state.  check_mk
  // rejects M*K > 2^40, beyond which the fixed bins could overflow.
  bitlinear_status st = check_mk(M, K);
  if (st != BITLINEAR_OK) return st;
  if (!W || !packed || !alpha) return BITLINEAR_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(packed) || !aligned4(alpha)) return BITLINEAR_ERR_MISALIGNED;
  void* scratch = nullptr;
  if ((st = noalloc_pack_scratch(&scratch)) != BITLINEAR_OK) return st;
  return bitlinear_pack_weights(W, M, K, packed, alpha, scratch, sizeof(g_noalloc_pack_scratch),
                                stream);
}
