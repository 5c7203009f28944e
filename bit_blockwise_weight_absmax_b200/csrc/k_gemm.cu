// k_gemm.cu -- launchers of the tcgen05 W4A16 GEMM for launches of whole
// tiles, and the entry that picks the instance set.
#include "k_gemm_impl.cuh"

namespace q4 {

template int run_gemm_t<false>(int da, int mode, const GemmParams &p, cudaStream_t st);

int run_gemm(int da, int mode, bool split, const GemmParams &p, cudaStream_t st) {
  return split ? run_gemm_t<true>(da, mode, p, st) : run_gemm_t<false>(da, mode, p, st);
}

}  // namespace q4
