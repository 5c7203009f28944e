// k_quantize.cu -- launchers of the quantize and double-quant kernels.
#include "q4_internal.h"
#include "quantize_grouped.cuh"

namespace q4 {
namespace {
template <int DT, int QT, int B, bool DQ>
int go(const QuantParams &p, int grid, cudaStream_t st) {
  launch_pdl(quantize_kernel<DT, QT, B, DQ>, dim3(grid), dim3(kQThreads), 0, st, p);
  return 0;
}
template <int DT, int QT, int B, bool DQ>
int gog(const QuantGroupParams &p, int grid, cudaStream_t st) {
  constexpr auto kern = quantize_grouped_kernel<DT, QT, B, DQ>;
  const int rc = set_smem_attr_once<kern>(kQgSmem, true);
  if (rc != Q4_OK) return rc;
  launch_pdl(kern, dim3(grid), dim3(kQgThreads), kQgSmem, st, p);
  return 0;
}
template <bool GROUPED, int DT, int QT, int B, bool DQ, typename P>
int launch(const P &p, int grid, cudaStream_t st) {
  if constexpr (GROUPED) return gog<DT, QT, B, DQ>(p, grid, st);
  else return go<DT, QT, B, DQ>(p, grid, st);
}
template <bool GROUPED, int DT, int QT, bool DQ, typename P>
int by_bs(int bs, const P &p, int grid, cudaStream_t st) {
  switch (bs) {
    case 32: return launch<GROUPED, DT, QT, 32, DQ>(p, grid, st);
    case 64: return launch<GROUPED, DT, QT, 64, DQ>(p, grid, st);
    case 128: return launch<GROUPED, DT, QT, 128, DQ>(p, grid, st);
    case 256: return launch<GROUPED, DT, QT, 256, DQ>(p, grid, st);
  }
  return Q4_ERR_ARG;
}
template <bool GROUPED, int DT, typename P>
int by_qt(int qt, int bs, bool dq, const P &p, int grid, cudaStream_t st) {
  if (qt == Q4_NF4)
    return dq ? by_bs<GROUPED, DT, Q4_NF4, true>(bs, p, grid, st) : by_bs<GROUPED, DT, Q4_NF4, false>(bs, p, grid, st);
  if (qt == Q4_INT4_SYM) return by_bs<GROUPED, DT, Q4_INT4_SYM, false>(bs, p, grid, st);
  return by_bs<GROUPED, DT, Q4_INT4_ASYM, false>(bs, p, grid, st);
}
template <bool GROUPED, typename P>
int dispatch(int dt, int qt, int bs, bool dq, const P &p, int grid, cudaStream_t st) {
  if (dq && qt != Q4_NF4) return Q4_ERR_ARG;
  const int rc = dt == Q4_F16 ? by_qt<GROUPED, Q4_F16>(qt, bs, dq, p, grid, st)
                              : by_qt<GROUPED, Q4_BF16>(qt, bs, dq, p, grid, st);
  if (rc) return rc;
  return cudaGetLastError() == cudaSuccess ? Q4_OK : Q4_ERR_CUDA;
}
}  // namespace

int run_quantize(int dt, int qt, int bs, bool dq, const QuantParams &p, int grid, cudaStream_t st) {
  return dispatch<false>(dt, qt, bs, dq, p, grid, st);
}

// grid: at most one CTA per SM (the kernel is persistent over the chunks)
int run_quantize_grouped(int dt, int qt, int bs, bool dq, const QuantGroupParams &p, int grid, cudaStream_t st) {
  return dispatch<true>(dt, qt, bs, dq, p, grid, st);
}

int run_double_quant(const float *absmax, int64_t nb, const float *mean, int8_t *absmax_q,
                     float *absmax_scale, cudaStream_t st) {
  const int64_t ng = (nb + Q4_DQ_GROUP - 1) / Q4_DQ_GROUP;
  launch_pdl(double_quant_kernel, dim3((unsigned)((ng + 7) / 8)), dim3(256), 0, st, absmax, nb, mean, absmax_q,
             absmax_scale);
  return cudaGetLastError() == cudaSuccess ? Q4_OK : Q4_ERR_CUDA;
}

int run_double_quant_grouped(const DqGroupParams &p, cudaStream_t st) {
  launch_pdl(double_quant_grouped_kernel, dim3((unsigned)((p.total_groups + 7) / 8)), dim3(256), 0, st, p);
  return cudaGetLastError() == cudaSuccess ? Q4_OK : Q4_ERR_CUDA;
}
}  // namespace q4
