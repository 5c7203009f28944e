// k_gemv.cu -- launchers of the fused dequant-GEMV kernel.
#include <algorithm>

#include "q4_internal.h"

namespace q4 {
namespace {
constexpr int kUnitK = 1024;  // k per work unit (must match the host plan)

template <int DA, int NT, int R, int B>
int go(const GemvParams &p, int sms, cudaStream_t st) {
  constexpr int UB = kUnitK / B;
  constexpr int PF = (R == 1) ? (UB < 8 ? UB : 8) : (UB < 4 ? UB : 4);
  auto kern = gemv_kernel<DA, NT, R, B, UB, PF>;
  const int smem = 256 * 32 * (DA == Q4_BF16 ? 8 : 4);
  static int occ = 0;
  if (occ == 0) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return Q4_ERR_CUDA;
    int o = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, kern, kGemvWarps * 32, smem) != cudaSuccess || o < 1)
      return Q4_ERR_CUDA;
    occ = o;
  }
  const int64_t want = (p.total_units + kGemvWarps - 1) / kGemvWarps;
  const int grid = (int)std::min<int64_t>(want, (int64_t)sms * occ);
  kern<<<grid, kGemvWarps * 32, smem, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? Q4_OK : Q4_ERR_CUDA;
}
template <int DA, int NT, int R>
int by_bs(int bs, const GemvParams &p, int sms, cudaStream_t st) {
  switch (bs) {
    case 32: return go<DA, NT, R, 32>(p, sms, st);
    case 64: return go<DA, NT, R, 64>(p, sms, st);
    case 128: return go<DA, NT, R, 128>(p, sms, st);
    case 256: return go<DA, NT, R, 256>(p, sms, st);
  }
  return Q4_ERR_ARG;
}
template <int DA>
int by_plan(int nt, int r, int bs, const GemvParams &p, int sms, cudaStream_t st) {
  if (nt == 1 && r == 1) return by_bs<DA, 1, 1>(bs, p, sms, st);
  if (nt == 2 && r == 2) return by_bs<DA, 2, 2>(bs, p, sms, st);
  if (nt == 4 && r == 2) return by_bs<DA, 4, 2>(bs, p, sms, st);
  return Q4_ERR_ARG;
}
}  // namespace

int run_gemv(int da, int nt, int r, int bs, const GemvParams &p, int sms, cudaStream_t st) {
  return da == Q4_F16 ? by_plan<Q4_F16>(nt, r, bs, p, sms, st) : by_plan<Q4_BF16>(nt, r, bs, p, sms, st);
}
}  // namespace q4
