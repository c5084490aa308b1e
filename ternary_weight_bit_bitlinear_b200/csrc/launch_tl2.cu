// launch_tl2.cu -- launchers of the TL2-style storage kernels (tl2.cuh): the
// conversion from 2-bit rows and the decode GEMV over TL2 rows.
#include "internal.h"

namespace blh {
namespace {

template <int NT>
bitlinear_status launch_gemv_tl2_nt(const bl::Tl2Params& p, DeviceInfo* dev, cudaStream_t s) {
  auto kernel = bl::gemv_tl2_kernel<NT>;
  constexpr int smem = bl::Tl2Cfg<NT>::kSmemBytes;
  int& per_sm = dev->tl2_blocks_per_sm[NT];
  if (per_sm == 0) {
    int nb = 0;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
            cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kernel, bl::kTl2Threads, smem) !=
            cudaSuccess ||
        nb < 1)
      return BITLINEAR_ERR_CUDA;
    per_sm = nb;
  }
  const int64_t cap = static_cast<int64_t>(dev->sms) * per_sm * bl::kTl2Warps;
  const int64_t upw = (p.total_units + cap - 1) / cap;
  const int64_t warps = (p.total_units + upw - 1) / upw;
  const int grid = static_cast<int>((warps + bl::kTl2Warps - 1) / bl::kTl2Warps);
  if (launch_pdl(kernel, grid, bl::kTl2Threads, smem, s, p) != cudaSuccess)
    return BITLINEAR_ERR_CUDA;
  return launch_status();
}

}  // namespace

bitlinear_status launch_gemv_tl2(int N, const bl::Tl2Params& p, DeviceInfo* dev,
                                 cudaStream_t s) {
  switch (N) {
#define BL_TL2_CASE(n) \
  case n: return launch_gemv_tl2_nt<n>(p, dev, s);
    BL_TL2_CASE(1) BL_TL2_CASE(2) BL_TL2_CASE(3) BL_TL2_CASE(4)
    BL_TL2_CASE(5) BL_TL2_CASE(6) BL_TL2_CASE(7) BL_TL2_CASE(8)
    BL_TL2_CASE(9) BL_TL2_CASE(10) BL_TL2_CASE(11) BL_TL2_CASE(12)
    BL_TL2_CASE(13) BL_TL2_CASE(14) BL_TL2_CASE(15) BL_TL2_CASE(16)
#undef BL_TL2_CASE
    default: return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
  }
}

bitlinear_status launch_tl2_convert(const uint32_t* packed, int64_t M, int64_t K, int wp,
                                    uint8_t* tl2, int grid, cudaStream_t s) {
  bl::tl2_convert_kernel<<<grid, 256, 0, s>>>(packed, M, K, wp, tl2);
  return launch_status();
}

cudaError_t device_error_tl2(unsigned int* v, bool clear) {
  return read_error_word(bl::g_device_error, v, clear);
}

}  // namespace blh
