// k_dequantize.cu -- launchers of the dequantize kernel.
#include <algorithm>

#include "q4_internal.h"

namespace q4 {
namespace {
template <int QT, int DO, int B, bool DQ>
void go(const DequantParams &p, int grid, cudaStream_t st) {
  launch_pdl(dequantize_kernel<QT, DO, B, DQ>, dim3(grid), dim3(kDqThreads), 0, st, p);
}
template <int QT, int DO, bool DQ>
int by_bs(int bs, const DequantParams &p, int grid, cudaStream_t st) {
  switch (bs) {
    case 32: go<QT, DO, 32, DQ>(p, grid, st); return 0;
    case 64: go<QT, DO, 64, DQ>(p, grid, st); return 0;
    case 128: go<QT, DO, 128, DQ>(p, grid, st); return 0;
    case 256: go<QT, DO, 256, DQ>(p, grid, st); return 0;
  }
  return Q4_ERR_ARG;
}
template <int QT, bool DQ>
int by_do(int dout, int bs, const DequantParams &p, int grid, cudaStream_t st) {
  return dout == Q4_F16 ? by_bs<QT, Q4_F16, DQ>(bs, p, grid, st) : by_bs<QT, Q4_BF16, DQ>(bs, p, grid, st);
}
template <int QT, int DO, int B, bool DQ>
void gog(const DequantGroupParams &p, int grid, cudaStream_t st) {
  launch_pdl(dequantize_grouped_kernel<QT, DO, B, DQ>, dim3(grid), dim3(kDqThreads), 0, st, p);
}
template <int QT, int DO, bool DQ>
int gby_bs(int bs, const DequantGroupParams &p, int grid, cudaStream_t st) {
  switch (bs) {
    case 32: gog<QT, DO, 32, DQ>(p, grid, st); return 0;
    case 64: gog<QT, DO, 64, DQ>(p, grid, st); return 0;
    case 128: gog<QT, DO, 128, DQ>(p, grid, st); return 0;
    case 256: gog<QT, DO, 256, DQ>(p, grid, st); return 0;
  }
  return Q4_ERR_ARG;
}
template <int QT, bool DQ>
int gby_do(int dout, int bs, const DequantGroupParams &p, int grid, cudaStream_t st) {
  return dout == Q4_F16 ? gby_bs<QT, Q4_F16, DQ>(bs, p, grid, st) : gby_bs<QT, Q4_BF16, DQ>(bs, p, grid, st);
}
}  // namespace

int run_dequantize_grouped(int qt, int dout, int bs, bool dq, const DequantGroupParams &p, int sms,
                           cudaStream_t st) {
  const int occ = qt == Q4_INT4_ASYM ? dq_ctas_per_sm<Q4_INT4_ASYM>() : dq_ctas_per_sm<Q4_NF4>();
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>((p.total_spans + kDqThreads / 32 - 1) / (kDqThreads / 32),
                                                                 (int64_t)sms * occ));
  int rc;
  if (qt == Q4_NF4) rc = dq ? gby_do<Q4_NF4, true>(dout, bs, p, grid, st) : gby_do<Q4_NF4, false>(dout, bs, p, grid, st);
  else if (qt == Q4_INT4_SYM) rc = gby_do<Q4_INT4_SYM, false>(dout, bs, p, grid, st);
  else rc = gby_do<Q4_INT4_ASYM, false>(dout, bs, p, grid, st);
  if (rc) return rc;
  return cudaGetLastError() == cudaSuccess ? Q4_OK : Q4_ERR_CUDA;
}

int run_dequantize(int qt, int dout, int bs, bool dq, const DequantParams &p, int sms,
                   cudaStream_t st) {
  // one warp per span at a time, as many CTAs as are resident at once
  const int64_t spans = (p.n + kDqSpan - 1) / kDqSpan;
  const int occ = qt == Q4_INT4_ASYM ? dq_ctas_per_sm<Q4_INT4_ASYM>() : dq_ctas_per_sm<Q4_NF4>();
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>((spans + kDqThreads / 32 - 1) / (kDqThreads / 32),
                                                                 (int64_t)sms * occ));
  int rc;
  if (qt == Q4_NF4) rc = dq ? by_do<Q4_NF4, true>(dout, bs, p, grid, st) : by_do<Q4_NF4, false>(dout, bs, p, grid, st);
  else if (qt == Q4_INT4_SYM) rc = by_do<Q4_INT4_SYM, false>(dout, bs, p, grid, st);
  else rc = by_do<Q4_INT4_ASYM, false>(dout, bs, p, grid, st);
  if (rc) return rc;
  return cudaGetLastError() == cudaSuccess ? Q4_OK : Q4_ERR_CUDA;
}
}  // namespace q4
