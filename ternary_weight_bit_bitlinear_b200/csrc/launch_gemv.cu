// launch_gemv.cu -- launchers of the decode GEMV on int8 activations
// (gemv.cuh: one warp per 32-row unit; gemv_split.cuh: one 4-warp CTA per
// unit for launches that would leave resident warps idle).
#include "internal.h"
#include "gemv_split.cuh"

namespace blh {
namespace {

template <int NT>
bitlinear_status launch_gemv_tile(const bl::GemvParams& p, DeviceInfo* dev, cudaStream_t s) {
  auto kernel = bl::gemv_tile_kernel<NT>;
  constexpr int smem = bl::GemvCfg<NT>::kSmemBytes;
  int& per_sm = dev->gemv_blocks_per_sm[NT];
  if (per_sm == 0) {
    int nb = 0;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
            cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kernel, bl::kGemvThreads, smem) !=
            cudaSuccess ||
        nb < 1)
      return BITLINEAR_ERR_CUDA;
    per_sm = nb;
  }
  // Every warp resident at once, with the same number of units (give or take
  // one) per warp: units per warp first, then just enough warps.  A launch
  // with fewer units than resident warps, or one where that would leave more
  // than a quarter of them idle (a little over a whole multiple: 1792 units on
  // 1776 warps would run 896 warps of two units each), takes the split-unit
  // kernel instead: one CTA per unit, its k-chunks split over the CTA's warps,
  // CTAs handed to SMs as they free up.
  const int64_t cap = static_cast<int64_t>(dev->sms) * per_sm * bl::kGemvWarps;
  const int64_t upw = (p.total_units + cap - 1) / cap;
  if (p.total_units < cap || p.total_units * 4 < upw * cap * 3) {
    auto split = bl::gemv_split_kernel<NT>;
    if (!dev->gemv_split_attr_set[NT]) {
      if (cudaFuncSetAttribute(split, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
          cudaSuccess)
        return BITLINEAR_ERR_CUDA;
      dev->gemv_split_attr_set[NT] = true;
    }
    if (launch_pdl(split, p.total_units, bl::kGemvThreads, smem, s, p) != cudaSuccess)
      return BITLINEAR_ERR_CUDA;
    return launch_status();
  }
  const int64_t warps = (p.total_units + upw - 1) / upw;
  const int grid = static_cast<int>((warps + bl::kGemvWarps - 1) / bl::kGemvWarps);
  if (launch_pdl(kernel, grid, bl::kGemvThreads, smem, s, p) != cudaSuccess)
    return BITLINEAR_ERR_CUDA;
  return launch_status();
}

}  // namespace

bitlinear_status launch_gemv(int N, const bl::GemvParams& p, DeviceInfo* dev, cudaStream_t s) {
  switch (N) {
#define BL_GEMV_CASE(n) \
  case n: return launch_gemv_tile<n>(p, dev, s);
    BL_GEMV_CASE(1) BL_GEMV_CASE(2) BL_GEMV_CASE(3) BL_GEMV_CASE(4)
    BL_GEMV_CASE(5) BL_GEMV_CASE(6) BL_GEMV_CASE(7) BL_GEMV_CASE(8)
    BL_GEMV_CASE(9) BL_GEMV_CASE(10) BL_GEMV_CASE(11) BL_GEMV_CASE(12)
    BL_GEMV_CASE(13) BL_GEMV_CASE(14) BL_GEMV_CASE(15) BL_GEMV_CASE(16)
#undef BL_GEMV_CASE
    default: return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
  }
}

cudaError_t device_error_gemv(unsigned int* v, bool clear) {
  return read_error_word(bl::g_device_error, v, clear);
}

}  // namespace blh
