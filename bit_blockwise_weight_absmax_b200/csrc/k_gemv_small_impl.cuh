// k_gemv_small_impl.cuh -- launch templates of the decode GEMV
// (gemv_small.cuh); k_gemv_small.cu instantiates them for NF4 and INT4
// symmetric states, k_gemv_small_asym.cu for INT4 asymmetric ones.
#pragma once
#include <algorithm>

#include "q4_internal.h"

namespace q4 {
namespace gs_launch {

// The mma.sync kernel: one CTA per SM with all of its shared memory (the
// kernel lays out its table, buffers and ring itself).
template <int DA, int NT, int B, bool AZ>
int go_small(const GsParams &p, int sms, cudaStream_t st) {
  // 16-row groups per compute warp: one, so 16 compute warps (+ the
  // producer), wherever that fits the 96 registers 17 warps leave a thread
  // (per-scheduler register file) without spilling: binary16 up to M = 16
  // and bf16 up to M = 8 (at M = 16, 8 warps of 32 rows were 9% slower for
  // binary16).  bf16 at 9 <= M <= 16 and every M > 16 (four column tiles)
  // use 8 warps of 32 rows.
  constexpr int R = (NT == 4 || (DA == Q4_BF16 && NT == 2)) ? 2 : 1;
  constexpr auto kern = gemv_small_kernel<DA, NT, B, R, AZ>;
  if (set_smem_attr_once<kern>(kGsSmemBytes, true) != Q4_OK) return Q4_ERR_CUDA;
  const int grid = (int)std::min<int64_t>(p.total_stages, (int64_t)std::min(sms, kGsMaxCtas));
  launch_pdl(kern, dim3(grid), dim3(GsShape<R>::kThreads), kGsSmemBytes, st, p);
  return cudaGetLastError() == cudaSuccess ? Q4_OK : Q4_ERR_CUDA;
}
template <int DA, int NT, bool AZ>
int small_bs(int bs, const GsParams &p, int sms, cudaStream_t st) {
  switch (bs) {
    case 32: return go_small<DA, NT, 32, AZ>(p, sms, st);
    case 64: return go_small<DA, NT, 64, AZ>(p, sms, st);
    case 128: return go_small<DA, NT, 128, AZ>(p, sms, st);
    case 256: return go_small<DA, NT, 256, AZ>(p, sms, st);
  }
  return Q4_ERR_ARG;
}
template <int DA, bool AZ>
int small_m(int M, int bs, const GsParams &p, int sms, cudaStream_t st) {
  if (M <= 8) return small_bs<DA, 1, AZ>(bs, p, sms, st);
  if (M <= 16) return small_bs<DA, 2, AZ>(bs, p, sms, st);
  return small_bs<DA, 4, AZ>(bs, p, sms, st);
}

}  // namespace gs_launch

template <bool AZ>
int run_gemv_small_t(int da, int bs, int M, const GsParams &p, int sms, cudaStream_t st) {
  return da == Q4_F16 ? gs_launch::small_m<Q4_F16, AZ>(M, bs, p, sms, st)
                      : gs_launch::small_m<Q4_BF16, AZ>(M, bs, p, sms, st);
}

}  // namespace q4
