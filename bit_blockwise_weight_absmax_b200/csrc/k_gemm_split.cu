// k_gemm_split.cu -- launchers of the tcgen05 W4A16 GEMM for launches of
// tall tiles whose plan cuts tiles in halves of their k range (split-K).
#include "k_gemm_impl.cuh"

namespace q4 {

template int run_gemm_t<true, true>(int da, int mode, const GemmParams &p, cudaStream_t st);

}  // namespace q4
