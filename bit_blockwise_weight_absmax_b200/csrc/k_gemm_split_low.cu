// k_gemm_split_low.cu -- launchers of the tcgen05 W4A16 GEMM for launches
// of half-height tiles whose plan cuts tiles in k (split-K).
#include "k_gemm_impl.cuh"

namespace q4 {

template int run_gemm_t<true, false>(int da, int mode, const GemmParams &p, cudaStream_t st);

}  // namespace q4
