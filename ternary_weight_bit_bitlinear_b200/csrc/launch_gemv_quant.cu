// launch_gemv_quant.cu -- launchers of the fused quantise + GEMV decode
// kernel (gemv_quant.cuh).
#include "internal.h"

namespace blh {
namespace {

// Dynamic shared memory a CTA of this kernel may use: the device's opt-in
// maximum per block less the kernel's static shared memory.
template <int NT>
bitlinear_status max_dyn_smem(DeviceInfo* dev, int* out) {
  auto kernel = bl::gemv_quant_kernel<NT>;
  if (!dev->gq_attr_set[NT]) {
    int dev_id = 0, optin = 0;
    cudaFuncAttributes fa;
    if (cudaGetDevice(&dev_id) != cudaSuccess ||
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev_id) !=
            cudaSuccess ||
        cudaFuncGetAttributes(&fa, kernel) != cudaSuccess)
      return BITLINEAR_ERR_CUDA;
    const int dyn = optin - static_cast<int>(fa.sharedSizeBytes);
    if (dyn <= 0 ||
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn) !=
            cudaSuccess)
      return BITLINEAR_ERR_CUDA;
    dev->gq_max_dyn[NT] = dyn;
    dev->gq_attr_set[NT] = true;
  }
  *out = dev->gq_max_dyn[NT];
  return BITLINEAR_OK;
}

template <int NT>
bitlinear_status occupancy_nt(int warps, int area, DeviceInfo* dev, int* out) {
  auto kernel = bl::gemv_quant_kernel<NT>;
  int dyn = 0;
  bitlinear_status st = max_dyn_smem<NT>(dev, &dyn);
  if (st != BITLINEAR_OK) return st;
  if (area > dyn) {
    *out = 0;
    return BITLINEAR_OK;
  }
  if (dev->gq_area[NT][warps] != area) {
    int nb = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kernel, 32 * warps, area) !=
        cudaSuccess)
      return BITLINEAR_ERR_CUDA;
    dev->gq_area[NT][warps] = area;
    dev->gq_occ[NT][warps] = nb;
  }
  *out = dev->gq_occ[NT][warps];
  return BITLINEAR_OK;
}

}  // namespace

bitlinear_status gemv_quant_occupancy(int N, int warps, int area, DeviceInfo* dev, int* out) {
  if (warps < 1 || warps > bl::gq_max_warps(N)) {
    *out = 0;
    return BITLINEAR_OK;
  }
  switch (N) {
#define BL_GQ_CASE(n) \
  case n: return occupancy_nt<n>(warps, area, dev, out);
    BL_GQ_CASE(1) BL_GQ_CASE(2) BL_GQ_CASE(3) BL_GQ_CASE(4)
    BL_GQ_CASE(5) BL_GQ_CASE(6) BL_GQ_CASE(7) BL_GQ_CASE(8)
    BL_GQ_CASE(9) BL_GQ_CASE(10) BL_GQ_CASE(11) BL_GQ_CASE(12)
    BL_GQ_CASE(13) BL_GQ_CASE(14) BL_GQ_CASE(15) BL_GQ_CASE(16)
#undef BL_GQ_CASE
    default: return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
  }
}

bitlinear_status gemv_quant_launch(int N, int grid, int warps, const bl::GqParams& p,
                                   cudaStream_t s) {
  cudaError_t e = cudaErrorInvalidValue;
  switch (N) {
#define BL_GQ_CASE(n) \
  case n: e = launch_pdl(bl::gemv_quant_kernel<n>, grid, 32 * warps, \
                         static_cast<size_t>(p.area), s, p); \
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

cudaError_t device_error_gemv_quant(unsigned int* v, bool clear) {
  return read_error_word(bl::g_device_error, v, clear);
}

}  // namespace blh
