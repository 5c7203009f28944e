// k_gemm.cu -- launchers of the tcgen05 W4A16 GEMM for launches of whole
// tall tiles, and the entry that picks the instance set.
#include "k_gemm_impl.cuh"

namespace q4 {

template int run_gemm_t<false, true>(int da, int mode, const GemmParams &p, cudaStream_t st);
// the other instance sets are compiled in their own units
extern template int run_gemm_t<false, false>(int da, int mode, const GemmParams &p, cudaStream_t st);
extern template int run_gemm_t<true, true>(int da, int mode, const GemmParams &p, cudaStream_t st);
extern template int run_gemm_t<true, false>(int da, int mode, const GemmParams &p, cudaStream_t st);

int run_gemm(int da, int mode, bool split, const GemmParams &p, cudaStream_t st) {
  const bool tall = p.tile_m == kGemmBM;
  if (split) return tall ? run_gemm_t<true, true>(da, mode, p, st) : run_gemm_t<true, false>(da, mode, p, st);
  return tall ? run_gemm_t<false, true>(da, mode, p, st) : run_gemm_t<false, false>(da, mode, p, st);
}

}  // namespace q4
