// k_gemm_impl.cuh -- launch templates of the tcgen05 W4A16 GEMM
// (gemm.cuh), one instance set per tile height and split mode:
// k_gemm.cu (tall tiles, whole), k_gemm_low.cu (half-height tiles, whole),
// k_gemm_split.cu and k_gemm_split_low.cu (tiles cut in k).
#pragma once
#include "q4_internal.h"

namespace q4 {
namespace gemm_launch {

template <int DA, int MODE, bool SPLIT, bool TALL>
int go(const GemmParams &p, cudaStream_t st) {
  constexpr auto kern = gemm_kernel<DA, MODE, SPLIT, TALL>;
  if (set_smem_attr_once<kern>(kGemmSmem, false) != Q4_OK) return Q4_ERR_CUDA;
  launch_pdl(kern, dim3(p.grid), dim3(kGemmThreads), kGemmSmem, st, p);  // the host planned the grid
  return cudaGetLastError() == cudaSuccess ? Q4_OK : Q4_ERR_CUDA;
}
template <int DA, bool SPLIT, bool TALL>
int by_mode(int mode, const GemmParams &p, cudaStream_t st) {
  if (mode == kGemmDq) return go<DA, kGemmDq, SPLIT, TALL>(p, st);
  if (mode == kGemmAsym) return go<DA, kGemmAsym, SPLIT, TALL>(p, st);
  return go<DA, kGemmPlain, SPLIT, TALL>(p, st);
}

}  // namespace gemm_launch

template <bool SPLIT, bool TALL>
int run_gemm_t(int da, int mode, const GemmParams &p, cudaStream_t st) {
  return da == Q4_F16 ? gemm_launch::by_mode<Q4_F16, SPLIT, TALL>(mode, p, st)
                      : gemm_launch::by_mode<Q4_BF16, SPLIT, TALL>(mode, p, st);
}

}  // namespace q4
