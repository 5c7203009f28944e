// k_gemm_low.cu -- launchers of the tcgen05 W4A16 GEMM for launches of
// whole half-height tiles.
#include "k_gemm_impl.cuh"

namespace q4 {

template int run_gemm_t<false, false>(int da, int mode, const GemmParams &p, cudaStream_t st);

}  // namespace q4
