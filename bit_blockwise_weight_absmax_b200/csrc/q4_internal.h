// q4_internal.h -- host-side launcher entry points shared by the translation
// units of libq4.so (not part of the public C ABI).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <utility>

#include "q4_common.cuh"
#include "quantize.cuh"
#include "dequantize.cuh"
#include "gemv_small.cuh"
#include "gemm.cuh"
#include "quantize_grouped.cuh"

namespace q4 {
// Launch with programmatic stream serialization (the kernel calls
// pdl_launch_then_wait() before any global memory access).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Raise a kernel's dynamic shared-memory limit (and, optionally, its
// shared-memory carveout) once per device: the attribute is per device, and
// the first calls on a device may come from several threads at once.
constexpr int kMaxDevices = 64;
template <auto Kern>
int set_smem_attr_once(int bytes, bool max_carveout) {
  static std::once_flag once[kMaxDevices];
  static int rc[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return Q4_ERR_CUDA;
  }
  std::call_once(once[dev], [&] {
    bool ok = cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess;
    if (ok && max_carveout)
      ok = cudaFuncSetAttribute(Kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                cudaSharedmemCarveoutMaxShared) == cudaSuccess;
    if (!ok) cudaGetLastError();
    rc[dev] = ok ? Q4_OK : Q4_ERR_CUDA;
  });
  return rc[dev];
}

int run_quantize(int dt, int qt, int bs, bool dq, const QuantParams &p, int grid, cudaStream_t st);
int run_double_quant(const float *absmax, int64_t nb, const float *mean, int8_t *absmax_q,
                     float *absmax_scale, cudaStream_t st);
int run_quantize_grouped(int dt, int qt, int bs, bool dq, const QuantGroupParams &p, int grid, cudaStream_t st);
int run_double_quant_grouped(const DqGroupParams &p, cudaStream_t st);
int run_dequantize(int qt, int dout, int bs, bool dq, const DequantGroupParams &p, int sms, cudaStream_t st);
// the instance set follows split and p.tile_m (tall or half-height tiles)
int run_gemm(int da, int mode, bool split, const GemmParams &p, cudaStream_t st);
template <bool SPLIT, bool TALL>
int run_gemm_t(int da, int mode, const GemmParams &p, cudaStream_t st);
int run_gemv_small(int da, int bs, int M, bool asym, const GsParams &p, int sms, cudaStream_t st);
template <bool AZ>
int run_gemv_small_t(int da, int bs, int M, const GsParams &p, int sms, cudaStream_t st);
}  // namespace q4
