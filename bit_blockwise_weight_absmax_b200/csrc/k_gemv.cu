// k_gemv.cu -- launchers of the tcgen05 fused dequant-GEMV kernel.
#include <algorithm>

#include "q4_internal.h"

namespace q4 {
namespace {

template <int DA, int B, int MP>
int go(const GvParams &p, int sms, cudaStream_t st) {
  constexpr int NB = MP <= 16 ? 16 : 32;
  constexpr int STAGE = NB * kGvStageK * 2 + kGvWTile;
  constexpr int S = (DA == Q4_BF16) ? 4 : (NB == 16 ? 8 : 6);
  constexpr int LUTB = (DA == Q4_BF16) ? 256 * 32 * 8 : 256 * 32 * 4;
  constexpr int SCALES = 2 * kGvRows * (kGvUnitK / B + 1) * 4;
  constexpr int SMEM = S * STAGE + LUTB + SCALES + 3 * S * 8 + 128 + 1024;
  auto kern = gemv_tc_kernel<DA, B, MP, NB, S>;
  static bool attr = false;
  if (!attr) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM) != cudaSuccess ||
        cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared) != cudaSuccess)
      return Q4_ERR_CUDA;
    attr = true;
  }
  // CTAs per SM: two when their shared memory fits (228 KB per SM, 1 KB
  // reserved per CTA) and the kernel was compiled for two (registers); their
  // 2 x 256 tensor-memory columns always fit.
  constexpr int OCC = (MP < 32 && 2 * (SMEM + 1024) <= 228 * 1024) ? 2 : 1;
  const int grid = (int)std::min<int64_t>(p.total_units, (int64_t)sms * OCC);
  kern<<<grid, kGvThreads, SMEM, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? Q4_OK : Q4_ERR_CUDA;
}

template <int DA, int B>
int by_mp(int mp, const GvParams &p, int sms, cudaStream_t st) {
  switch (mp) {
    case 1: return go<DA, B, 1>(p, sms, st);
    case 2: return go<DA, B, 2>(p, sms, st);
    case 4: return go<DA, B, 4>(p, sms, st);
    case 8: return go<DA, B, 8>(p, sms, st);
    case 16: return go<DA, B, 16>(p, sms, st);
    case 32: return go<DA, B, 32>(p, sms, st);
  }
  return Q4_ERR_ARG;
}

template <int DA>
int by_bs(int bs, int mp, const GvParams &p, int sms, cudaStream_t st) {
  switch (bs) {
    case 32: return by_mp<DA, 32>(mp, p, sms, st);
    case 64: return by_mp<DA, 64>(mp, p, sms, st);
    case 128: return by_mp<DA, 128>(mp, p, sms, st);
    case 256: return by_mp<DA, 256>(mp, p, sms, st);
  }
  return Q4_ERR_ARG;
}
// The mma.sync kernel: one CTA per SM with all of its shared memory (the
// kernel lays out its table, buffers and ring itself).
template <int DA, int NT, int B>
int go_small(const GsParams &p, int sms, cudaStream_t st) {
  // 16-row groups per compute warp: M <= 8 fits 16 compute warps (+ the
  // producer) in the registers; M <= 16 uses 8 warps of 32 rows
  constexpr int R = NT == 1 ? 1 : 2;
  auto kern = gemv_small_kernel<DA, NT, B, R>;
  static bool attr = false;
  if (!attr) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kGsSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared) != cudaSuccess)
      return Q4_ERR_CUDA;
    attr = true;
  }
  const int grid = (int)std::min<int64_t>(p.total_stages, (int64_t)std::min(sms, kGsMaxCtas));
  kern<<<grid, GsShape<R>::kThreads, kGsSmemBytes, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? Q4_OK : Q4_ERR_CUDA;
}
template <int DA, int NT>
int small_bs(int bs, const GsParams &p, int sms, cudaStream_t st) {
  switch (bs) {
    case 32: return go_small<DA, NT, 32>(p, sms, st);
    case 64: return go_small<DA, NT, 64>(p, sms, st);
    case 128: return go_small<DA, NT, 128>(p, sms, st);
    case 256: return go_small<DA, NT, 256>(p, sms, st);
  }
  return Q4_ERR_ARG;
}
template <int DA>
int small_m(int M, int bs, const GsParams &p, int sms, cudaStream_t st) {
  if (M <= 8) return small_bs<DA, 1>(bs, p, sms, st);
  return small_bs<DA, 2>(bs, p, sms, st);
}
}  // namespace

int run_gemv_small(int da, int bs, int M, const GsParams &p, int sms, cudaStream_t st) {
  return da == Q4_F16 ? small_m<Q4_F16>(M, bs, p, sms, st) : small_m<Q4_BF16>(M, bs, p, sms, st);
}

int run_gemv(int da, int bs, int mp, const GvParams &p, int sms, cudaStream_t st) {
  return da == Q4_F16 ? by_bs<Q4_F16>(bs, mp, p, sms, st) : by_bs<Q4_BF16>(bs, mp, p, sms, st);
}
}  // namespace q4
