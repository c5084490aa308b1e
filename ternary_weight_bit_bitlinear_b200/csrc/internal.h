// internal.h -- host-side pieces shared by the translation units of
// libbitlinear.so: per-device facts, the launch helper, and the launchers that
// each kernel family's unit (launch_*.cu) defines for the C ABI in
// bitlinear.cu.  Not part of the public interface.
//
// Each unit is compiled on its own (whole-program device code per unit), so
// the kernels of a family, their template instantiations and their device
// error word live in that unit only.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>
#include <utility>

#include "bitlinear.h"
#include "gemm.cuh"
#include "gemm_pair.cuh"
#include "gemv.cuh"
#include "gemv_quant.cuh"
#include "tl2.cuh"

namespace blh {

constexpr int kMaxDevices = 64;

// Per-device facts and one-time set-up flags, looked up once per device.
struct DeviceInfo {
  int sms = 0;
  bool gemm_attr_set[8] = {};
  int gemv_blocks_per_sm[bl::kGemvMaxTokens + 1] = {};   // 0: not set up yet
  int tl2_blocks_per_sm[bl::kGemvMaxTokens + 1] = {};    // 0: not set up yet
  bool gq_attr_set[bl::kGemvMaxTokens + 1] = {};
  int gq_max_dyn[bl::kGemvMaxTokens + 1] = {};            // dynamic shared memory limit
  int gq_area[bl::kGemvMaxTokens + 1][bl::kGqMaxWarps + 1] = {};   // last shared-memory size
  int gq_occ[bl::kGemvMaxTokens + 1][bl::kGqMaxWarps + 1] = {};    // and its CTAs per SM
  bool gemv_split_attr_set[bl::kGemvMaxTokens + 1] = {};
};

// The calling thread's current device.
bitlinear_status device_info(DeviceInfo** out);

// Wall-time limit every bounded wait of a launch uses (bitlinear_set_wait_limit).
unsigned long long wait_limit_ns();

// Launch with programmatic stream serialisation (see pdl_wait_prior_grid).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), int grid, int block, size_t smem,
                       cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(static_cast<unsigned>(block));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

inline bitlinear_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? BITLINEAR_OK : BITLINEAR_ERR_CUDA;
}

// ---- launchers, one unit per kernel family

// launch_gemv.cu: decode GEMV on int8 activations (tile or split-unit kernel).
bitlinear_status launch_gemv(int N, const bl::GemvParams& p, DeviceInfo* dev, cudaStream_t s);

// launch_gemv_quant.cu: the fused quantise + GEMV decode kernel.  CTAs of
// `warps` warps with `area` bytes of dynamic shared memory each.
bitlinear_status gemv_quant_occupancy(int N, int warps, int area, DeviceInfo* dev, int* out);
bitlinear_status gemv_quant_launch(int N, int grid, int warps, const bl::GqParams& p,
                                   cudaStream_t s);

// launch_gemm.cu: tensor-core GEMMs.  variant: 0 = 128-token tiles, 1 = CTA
// pairs, 3 = 64-token tiles (A unpacked into shared memory); 4 = 16 tokens,
// 5 = 32 tokens (A in tensor memory).
bitlinear_status launch_gemm(int variant, const bl::GemmParams& p, DeviceInfo* dev,
                             cudaStream_t s);

// launch_tl2.cu: TL2-style storage.
bitlinear_status launch_gemv_tl2(int N, const bl::Tl2Params& p, DeviceInfo* dev,
                                 cudaStream_t s);
bitlinear_status launch_tl2_convert(const uint32_t* packed, int64_t M, int64_t K, int wp,
                                    uint8_t* tl2, int grid, cudaStream_t s);

// Device error words, one per unit: read (and, with clear, reset) into *v.
cudaError_t device_error_gemv(unsigned int* v, bool clear);
cudaError_t device_error_gemv_quant(unsigned int* v, bool clear);
cudaError_t device_error_gemm(unsigned int* v, bool clear);
cudaError_t device_error_tl2(unsigned int* v, bool clear);

// Shared body of the device_error_* readers (each unit passes its own symbol).
template <typename Sym>
cudaError_t read_error_word(const Sym& sym, unsigned int* v, bool clear) {
  cudaError_t e = cudaMemcpyFromSymbol(v, sym, sizeof(unsigned int));
  if (e != cudaSuccess || !clear || *v == 0) return e;
  const unsigned int zero = 0;
  return cudaMemcpyToSymbol(sym, &zero, sizeof zero);
}

}  // namespace blh
