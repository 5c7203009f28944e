// k_dequantize.cu -- launcher of the dequantize kernel.
#include <algorithm>

#include "q4_internal.h"

namespace q4 {
namespace {
template <int QT, int DO, int B, bool DQ>
int go(const DequantGroupParams &p, int grid, cudaStream_t st) {
  constexpr auto kern = dequantize_kernel<QT, DO, B, DQ>;
  const int rc = set_smem_attr_once<kern>(kDqSmem, true);
  if (rc != Q4_OK) return rc;
  launch_pdl(kern, dim3(grid), dim3(kDqThreads), kDqSmem, st, p);
  return 0;
}
template <int QT, int DO, bool DQ>
int by_bs(int bs, const DequantGroupParams &p, int grid, cudaStream_t st) {
  switch (bs) {
    case 32: return go<QT, DO, 32, DQ>(p, grid, st);
    case 64: return go<QT, DO, 64, DQ>(p, grid, st);
    case 128: return go<QT, DO, 128, DQ>(p, grid, st);
    case 256: return go<QT, DO, 256, DQ>(p, grid, st);
  }
  return Q4_ERR_ARG;
}
template <int QT, bool DQ>
int by_do(int dout, int bs, const DequantGroupParams &p, int grid, cudaStream_t st) {
  return dout == Q4_F16 ? by_bs<QT, Q4_F16, DQ>(bs, p, grid, st) : by_bs<QT, Q4_BF16, DQ>(bs, p, grid, st);
}
}  // namespace

// One CTA per SM (at most one per 32 spans), persistent over the spans.
int run_dequantize(int qt, int dout, int bs, bool dq, const DequantGroupParams &p, int sms, cudaStream_t st) {
  const int grid = (int)std::max<int64_t>(
      1, std::min<int64_t>((p.total_spans + kDqThreads / 32 - 1) / (kDqThreads / 32), (int64_t)sms));
  int rc;
  if (qt == Q4_NF4) rc = dq ? by_do<Q4_NF4, true>(dout, bs, p, grid, st) : by_do<Q4_NF4, false>(dout, bs, p, grid, st);
  else if (qt == Q4_INT4_SYM) rc = by_do<Q4_INT4_SYM, false>(dout, bs, p, grid, st);
  else rc = by_do<Q4_INT4_ASYM, false>(dout, bs, p, grid, st);
  if (rc) return rc;
  return cudaGetLastError() == cudaSuccess ? Q4_OK : Q4_ERR_CUDA;
}
}  // namespace q4
