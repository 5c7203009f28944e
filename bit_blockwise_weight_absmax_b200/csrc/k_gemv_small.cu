// k_gemv_small.cu -- launchers of the decode GEMV (gemv_small.cuh) for NF4
// and INT4 symmetric states, and the entry that picks the instance set.
#include "k_gemv_small_impl.cuh"

namespace q4 {

template int run_gemv_small_t<false>(int da, int bs, int M, const GsParams &p, int sms, cudaStream_t st);

int run_gemv_small(int da, int bs, int M, bool asym, const GsParams &p, int sms, cudaStream_t st) {
  return asym ? run_gemv_small_t<true>(da, bs, M, p, sms, st) : run_gemv_small_t<false>(da, bs, M, p, sms, st);
}

}  // namespace q4
