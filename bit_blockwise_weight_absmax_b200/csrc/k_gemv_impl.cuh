// k_gemv_impl.cuh -- launchers of the decode GEMV (gemv.cuh), instantiated
// per (activation dtype, scale mode) in the k_gemv_*.cu translation units so
// that they compile in parallel.
#pragma once
#include "q4_internal.h"

namespace q4 {

template <int DA, int MODE, int NT, int B>
int gemv_go(const GvParams &p, int grid, cudaStream_t st) {
  constexpr auto kern = gemv_kernel<DA, MODE, NT, B>;
  if (set_smem_attr_once<kern>(kGvSmemBytes, true) != Q4_OK) return Q4_ERR_CUDA;
  launch_pdl(kern, dim3(grid), dim3((GvShape<NT>::WARPS + 1) * 32), kGvSmemBytes, st, p);
  return cudaGetLastError() == cudaSuccess ? Q4_OK : Q4_ERR_CUDA;
}

template <int DA, int MODE, int NT>
int gemv_by_bs(int bs, const GvParams &p, int grid, cudaStream_t st) {
  switch (bs) {
    case 32: return gemv_go<DA, MODE, NT, 32>(p, grid, st);
    case 64: return gemv_go<DA, MODE, NT, 64>(p, grid, st);
    case 128: return gemv_go<DA, MODE, NT, 128>(p, grid, st);
    case 256: return gemv_go<DA, MODE, NT, 256>(p, grid, st);
  }
  return Q4_ERR_ARG;
}

template <int DA, int MODE>
int run_gemv_dm(int nt, int bs, const GvParams &p, int grid, cudaStream_t st) {
  if (nt == 1) return gemv_by_bs<DA, MODE, 1>(bs, p, grid, st);
  if (nt == 2) return gemv_by_bs<DA, MODE, 2>(bs, p, grid, st);
  return gemv_by_bs<DA, MODE, 4>(bs, p, grid, st);
}

}  // namespace q4
