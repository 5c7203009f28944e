// k_quantize.cu -- launchers of the quantize and double-quant kernels.
#include "q4_internal.h"

namespace q4 {
namespace {
template <int DT, int QT, int B, bool DQ>
void go(const QuantParams &p, int grid, cudaStream_t st) {
  launch_pdl(quantize_kernel<DT, QT, B, DQ>, dim3(grid), dim3(kQThreads), 0, st, p);
}
template <int DT, int QT, bool DQ>
int by_bs(int bs, const QuantParams &p, int grid, cudaStream_t st) {
  switch (bs) {
    case 32: go<DT, QT, 32, DQ>(p, grid, st); return 0;
    case 64: go<DT, QT, 64, DQ>(p, grid, st); return 0;
    case 128: go<DT, QT, 128, DQ>(p, grid, st); return 0;
    case 256: go<DT, QT, 256, DQ>(p, grid, st); return 0;
  }
  return Q4_ERR_ARG;
}
template <int DT>
int by_qt(int qt, int bs, bool dq, const QuantParams &p, int grid, cudaStream_t st) {
  if (qt == Q4_NF4) return dq ? by_bs<DT, Q4_NF4, true>(bs, p, grid, st) : by_bs<DT, Q4_NF4, false>(bs, p, grid, st);
  if (qt == Q4_INT4_SYM) return by_bs<DT, Q4_INT4_SYM, false>(bs, p, grid, st);
  return by_bs<DT, Q4_INT4_ASYM, false>(bs, p, grid, st);
}
}  // namespace

int run_quantize(int dt, int qt, int bs, bool dq, const QuantParams &p, int grid, cudaStream_t st) {
  if (dq && qt != Q4_NF4) return Q4_ERR_ARG;
  int rc = dt == Q4_F16 ? by_qt<Q4_F16>(qt, bs, dq, p, grid, st) : by_qt<Q4_BF16>(qt, bs, dq, p, grid, st);
  if (rc) return rc;
  return cudaGetLastError() == cudaSuccess ? Q4_OK : Q4_ERR_CUDA;
}

int run_double_quant(const float *absmax, int64_t nb, const float *mean, int8_t *absmax_q,
                     float *absmax_scale, cudaStream_t st) {
  const int64_t ng = (nb + Q4_DQ_GROUP - 1) / Q4_DQ_GROUP;
  launch_pdl(double_quant_kernel, dim3((unsigned)((ng + 7) / 8)), dim3(256), 0, st, absmax, nb, mean, absmax_q,
             absmax_scale);
  return cudaGetLastError() == cudaSuccess ? Q4_OK : Q4_ERR_CUDA;
}
}  // namespace q4
