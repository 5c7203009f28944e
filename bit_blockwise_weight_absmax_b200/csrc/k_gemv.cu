// k_gemv.cu -- dispatch of the one-pass decode GEMV (gemv.cuh), which runs
// INT4 asymmetric states; its instantiations live in k_gemv_{f16,bf16}_asym.cu.
#include "q4_internal.h"

namespace q4 {

int gv_tile_rows(int nt) {
  return nt == 1 ? 16 * GvShape<1>::R * GvShape<1>::WARPS
                 : nt == 2 ? 16 * GvShape<2>::R * GvShape<2>::WARPS : 16 * GvShape<4>::R * GvShape<4>::WARPS;
}

int run_gemv(int da, int mode, int nt, int bs, const GvParams &p, int grid, cudaStream_t st) {
  if (mode != kGvAsym) return Q4_ERR_ARG;
  return da == Q4_F16 ? run_gemv_dm<Q4_F16, kGvAsym>(nt, bs, p, grid, st)
                      : run_gemv_dm<Q4_BF16, kGvAsym>(nt, bs, p, grid, st);
}

}  // namespace q4
