// k_gemm.cu -- launcher of the tcgen05 W4A16 GEMM kernel.
#include <algorithm>

#include "q4_internal.h"

namespace q4 {
namespace {
template <int DA, int MODE>
int go(const GemmParams &p, int sms, cudaStream_t st) {
  if (set_smem_attr_once<gemm_kernel<DA, MODE>>(kGemmSmem, false) != Q4_OK) return Q4_ERR_CUDA;
  const int grid = (int)std::min<int64_t>(p.total_tiles, (int64_t)sms);
  launch_pdl(gemm_kernel<DA, MODE>, dim3(grid), dim3(kGemmThreads), kGemmSmem, st, p);
  return cudaGetLastError() == cudaSuccess ? Q4_OK : Q4_ERR_CUDA;
}
template <int DA>
int by_mode(int mode, const GemmParams &p, int sms, cudaStream_t st) {
  if (mode == kGemmDq) return go<DA, kGemmDq>(p, sms, st);
  if (mode == kGemmAsym) return go<DA, kGemmAsym>(p, sms, st);
  return go<DA, kGemmPlain>(p, sms, st);
}
}  // namespace

int run_gemm(int da, int mode, const GemmParams &p, int sms, cudaStream_t st) {
  return da == Q4_F16 ? by_mode<Q4_F16>(mode, p, sms, st) : by_mode<Q4_BF16>(mode, p, sms, st);
}
}  // namespace q4
