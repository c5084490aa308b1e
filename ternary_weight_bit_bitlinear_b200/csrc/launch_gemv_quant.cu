// launch_gemv_quant.cu -- launchers of the fused quantise + GEMV decode
// kernels (gemv_quant.cuh).
#include "internal.h"

namespace blh {
namespace {

template <int NT>
bitlinear_status gemv_quant_blocks_per_sm(int area, DeviceInfo* dev, int* out) {
  auto kernel = bl::gemv_quant_kernel<NT>;
  if (!dev->gq_attr_set[NT]) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             bl::kGqMaxXBytes + bl::kGqRingBytes) != cudaSuccess)
      return BITLINEAR_ERR_CUDA;
    dev->gq_attr_set[NT] = true;
  }
  if (dev->gq_smem[NT] != area) {
    int nb = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kernel, 32, area) != cudaSuccess ||
        nb < 1)
      return BITLINEAR_ERR_CUDA;
    dev->gq_smem[NT] = area;
    dev->gq_blocks_per_sm[NT] = nb;
  }
  *out = dev->gq_blocks_per_sm[NT];
  return BITLINEAR_OK;
}

template <int NT>
bitlinear_status launch_split(int grid, const bl::GqParams& p, DeviceInfo* dev, cudaStream_t s) {
  auto kernel = bl::gemv_quant_split_kernel<NT>;
  if (!dev->gqs_attr_set[NT]) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             bl::kGqMaxXBytes + bl::kGqsWarps * bl::kGqRingBytes) != cudaSuccess)
      return BITLINEAR_ERR_CUDA;
    dev->gqs_attr_set[NT] = true;
  }
  if (launch_pdl(kernel, grid, bl::kGqsThreads,
                 static_cast<size_t>(bl::gqs_smem_bytes(NT, p.xstride)), s, p) != cudaSuccess)
    return BITLINEAR_ERR_CUDA;
  return launch_status();
}

}  // namespace

bitlinear_status gemv_quant_occupancy(int N, int area, DeviceInfo* dev, int* out) {
  switch (N) {
#define BL_GQ_CASE(n) \
  case n: return gemv_quant_blocks_per_sm<n>(area, dev, out);
    BL_GQ_CASE(1) BL_GQ_CASE(2) BL_GQ_CASE(3) BL_GQ_CASE(4)
    BL_GQ_CASE(5) BL_GQ_CASE(6) BL_GQ_CASE(7) BL_GQ_CASE(8)
    BL_GQ_CASE(9) BL_GQ_CASE(10) BL_GQ_CASE(11) BL_GQ_CASE(12)
    BL_GQ_CASE(13) BL_GQ_CASE(14) BL_GQ_CASE(15) BL_GQ_CASE(16)
#undef BL_GQ_CASE
    default: return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
  }
}

bitlinear_status gemv_quant_launch(int N, int grid, const bl::GqParams& p, cudaStream_t s) {
  cudaError_t e = cudaErrorInvalidValue;
  switch (N) {
#define BL_GQ_CASE(n) \
  case n: e = launch_pdl(bl::gemv_quant_kernel<n>, grid, 32, static_cast<size_t>(p.area), s, p); \
    break;
    BL_GQ_CASE(1) BL_GQ_CASE(2) BL_GQ_CASE(3) BL_GQ_CASE(4)
    BL_GQ_CASE(5) BL_GQ_CASE(6) BL_GQ_CASE(7) BL_GQ_CASE(8)
    BL_GQ_CASE(9) BL_GQ_CASE(10) BL_GQ_CASE(11) BL_GQ_CASE(12)
    BL_GQ_CASE(13) BL_GQ_CASE(14) BL_GQ_CASE(15) BL_GQ_CASE(16)
#undef BL_GQ_CASE
    default: return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
  }
  if (e != cudaSuccess) return BITLINEAR_ERR_CUDA;
  return launch_status();
}

bitlinear_status gemv_quant_split_launch(int N, int grid, const bl::GqParams& p,
                                         DeviceInfo* dev, cudaStream_t s) {
  switch (N) {
    case 1: return launch_split<1>(grid, p, dev, s);
    case 2: return launch_split<2>(grid, p, dev, s);
    case 3: return launch_split<3>(grid, p, dev, s);
    case 4: return launch_split<4>(grid, p, dev, s);
    default: return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
  }
}

cudaError_t device_error_gemv_quant(unsigned int* v, bool clear) {
  return read_error_word(bl::g_device_error, v, clear);
}

}  // namespace blh
