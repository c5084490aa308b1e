// launch_gemm.cu -- launchers of the tensor-core GEMMs (gemm.cuh: one CTA per
// 128-row tile; gemm_pair.cuh: CTA pairs per 256 x 256 tile; gemm_small.cuh:
// A in tensor memory for up to 32 tokens).
#include "internal.h"
#include "gemm_small.cuh"

namespace blh {
namespace {

template <int BN, int STAGES>
bitlinear_status launch_single(const bl::GemmParams& p, DeviceInfo* dev, int slot,
                               cudaStream_t s) {
  auto kernel = bl::gemm_i8_tcgen05_kernel<BN, STAGES>;
  const int smem = static_cast<int>(sizeof(bl::GemmSmem<BN, STAGES>)) + 1024;
  if (!dev->gemm_attr_set[slot]) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
      return BITLINEAR_ERR_CUDA;
    dev->gemm_attr_set[slot] = true;
  }
  const int grid = p.total_tiles < dev->sms ? p.total_tiles : dev->sms;
  if (launch_pdl(kernel, grid, bl::kGemmThreads, smem, s, p) != cudaSuccess)
    return BITLINEAR_ERR_CUDA;
  return launch_status();
}

// CTA-pair GEMM for wide token blocks: two CTAs (a compile-time cluster) per
// 256 x 256 tile, one pair per two SMs.
template <int STAGES>
bitlinear_status launch_pair(const bl::GemmParams& p, DeviceInfo* dev, cudaStream_t s) {
  auto kernel = bl::gemm_i8_pair_kernel<STAGES>;
  const int smem = static_cast<int>(sizeof(bl::GemmPairSmem<STAGES>)) + 1024;
  if (!dev->gemm_attr_set[1]) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
      return BITLINEAR_ERR_CUDA;
    dev->gemm_attr_set[1] = true;
  }
  const int pairs = p.total_tiles < dev->sms / 2 ? p.total_tiles : dev->sms / 2;
  if (launch_pdl(kernel, 2 * pairs, bl::kGemmThreads, smem, s, p) != cudaSuccess)
    return BITLINEAR_ERR_CUDA;
  return launch_status();
}

template <int BN>
bitlinear_status launch_small(const bl::GemmParams& p, DeviceInfo* dev, int slot,
                              cudaStream_t s) {
  auto kernel = bl::gemm_small_kernel<BN>;
  const int smem = static_cast<int>(sizeof(bl::SmallSmem<BN>)) + 1024;
  if (!dev->gemm_attr_set[slot]) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
      return BITLINEAR_ERR_CUDA;
    dev->gemm_attr_set[slot] = true;
  }
  const int grid = p.total_tiles < dev->sms ? p.total_tiles : dev->sms;
  if (launch_pdl(kernel, grid, bl::kSmallThreads, smem, s, p) != cudaSuccess)
    return BITLINEAR_ERR_CUDA;
  return launch_status();
}

}  // namespace

bitlinear_status launch_gemm(int variant, const bl::GemmParams& p, DeviceInfo* dev,
                             cudaStream_t s) {
  switch (variant) {
    case 0: return launch_single<128, 7>(p, dev, 0, s);
    case 1: return launch_pair<5>(p, dev, s);
    case 3: return launch_single<64, 12>(p, dev, 3, s);
    case 4: return launch_small<16>(p, dev, 4, s);
    case 5: return launch_small<32>(p, dev, 5, s);
    default: return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
  }
}

cudaError_t device_error_gemm(unsigned int* v, bool clear) {
  return read_error_word(bl::g_device_error, v, clear);
}

}  // namespace blh
