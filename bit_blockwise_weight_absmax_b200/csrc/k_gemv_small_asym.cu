// k_gemv_small_asym.cu -- launchers of the decode GEMV (gemv_small.cuh) for
// INT4 asymmetric states (codes 0..15 with a zero-point per block).
#include "k_gemv_small_impl.cuh"

namespace q4 {

template int run_gemv_small_t<true>(int da, int bs, int M, const GsParams &p, int sms, cudaStream_t st);

}  // namespace q4
