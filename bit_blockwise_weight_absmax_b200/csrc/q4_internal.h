// q4_internal.h -- host-side launcher entry points shared by the translation
// units of libq4.so (not part of the public C ABI).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "q4_common.cuh"
#include "quantize.cuh"
#include "dequantize.cuh"
#include "gemv_small.cuh"
#include "gemm.cuh"

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

int run_quantize(int dt, int qt, int bs, bool dq, const QuantParams &p, int grid, cudaStream_t st);
int run_double_quant(const float *absmax, int64_t nb, const float *mean, int8_t *absmax_q,
                     float *absmax_scale, cudaStream_t st);
int run_dequantize(int qt, int dout, int bs, bool dq, const DequantParams &p, int sms,
                   cudaStream_t st);
int run_gemv_small(int da, int bs, int M, const GsParams &p, int sms, cudaStream_t st);
int run_gemm(int da, const GemmParams &p, int sms, cudaStream_t st);
}  // namespace q4
