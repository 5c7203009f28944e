// k_gemv_bf16_asym.cu -- decode GEMV launchers for bf16 activations, asym block scales.
#include "k_gemv_impl.cuh"

namespace q4 {
template int run_gemv_dm<Q4_BF16, kGvAsym>(int, int, const GvParams &, int, cudaStream_t);
}  // namespace q4
