// k_gemv_f16_asym.cu -- decode GEMV launchers for f16 activations, asym block scales.
#include "k_gemv_impl.cuh"

namespace q4 {
template int run_gemv_dm<Q4_F16, kGvAsym>(int, int, const GvParams &, int, cudaStream_t);
}  // namespace q4
