// dequantize.cuh -- 4-bit codes back to 16-bit floats (sm_100a).
//
// n4n.ai, "What is 4-bit quantization and why does it matter?", code block
// "Conceptual NF4 dequantization" (dequantize_nf4: unpack the low nibble
// first, then NF4_VALUES[idx] times the block scale) and learn.pranaymahendrakar.com,
// "Loading a model in 4-bit", "Block-wise quantisation, stated exactly"
// (w^ = c * Q[i]).  Per element: one binary32 multiply of the block scale and
// the level, rounded once to the output format.  With double quantization the
// scale is c~ = q2 * s2 + mu, two separately rounded operations.
//
// Design: the kernel reads 0.5 B and writes 2 B per element, so it is bound
// by HBM.  A warp owns spans of 256 * kDqChunks elements; within a span, lane
// l expands the 8-element chunks l, l + 32, ... so that every 16-byte store
// instruction of the warp covers 512 contiguous bytes, and every 4-byte load
// of packed codes covers 128 contiguous bytes.  All loads of a span (codes and
// block scales) are issued before the first multiply, to keep enough bytes in
// flight per SM.  The 16 levels sit in shared memory, one copy per lane, so a
// warp's 32 lookups hit 32 distinct banks.
#pragma once
#include "q4_common.cuh"

namespace q4 {

struct DequantParams {
  const uint8_t *packed;
  const float *absmax;
  const uint8_t *zero;
  const int8_t *absmax_q;
  const float *absmax_scale;
  const float *absmax_mean;
  int64_t n;
  void *out;
  float levels[16];
};

constexpr int kDqChunks = 4;                   // 8-element chunks per lane and span
constexpr int kDqSpan = 32 * 8 * kDqChunks;      // elements per warp and span
constexpr int kDqThreads = 256;

template <int QT, int DOUT, int B, bool DQ>
__global__ void __launch_bounds__(kDqThreads, 8) dequantize_kernel(const __grid_constant__ DequantParams p) {
  static_assert(B % 8 == 0, "a chunk never straddles two blocks");
  __shared__ float s_lv[16 * 32];
  const int lane = threadIdx.x & 31;
  if (QT == Q4_NF4) {
    for (int i = threadIdx.x; i < 16 * 32; i += blockDim.x) s_lv[i] = p.levels[i >> 5];
    __syncthreads();
  }
  const float mu = DQ ? __ldg(p.absmax_mean) : 0.0f;
  uint16_t *out = reinterpret_cast<uint16_t *>(p.out);
  const int64_t n = p.n;
  const int64_t nspan = (n + kDqSpan - 1) / kDqSpan;
  const int wpb = blockDim.x >> 5;
  for (int64_t sp = (int64_t)blockIdx.x * wpb + (threadIdx.x >> 5); sp < nspan; sp += (int64_t)gridDim.x * wpb) {
    const int64_t base = sp * kDqSpan + (int64_t)lane * 8;
    uint32_t pk[kDqChunks];
    float sc[kDqChunks];
    int z[kDqChunks];
#pragma unroll
    for (int u = 0; u < kDqChunks; ++u) {
      const int64_t e = base + u * 256;
      pk[u] = 0u;
      sc[u] = 0.0f;
      z[u] = 0;
      if (e >= n) continue;
      if (e + 8 <= n) {
        pk[u] = ldg_stream_u32(p.packed + e / 2);
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (e + 2 * j < n) pk[u] |= (uint32_t)p.packed[e / 2 + j] << (8 * j);
      }
      const int64_t b = e / B;
      if (DQ) sc[u] = __fadd_rn(__fmul_rn((float)__ldg(p.absmax_q + b), __ldg(p.absmax_scale + b / Q4_DQ_GROUP)), mu);
      else sc[u] = __ldg(p.absmax + b);
      if (QT == Q4_INT4_ASYM) z[u] = (__ldg(p.zero + (b >> 1)) >> ((b & 1) * 4)) & 15;
    }
#pragma unroll
    for (int u = 0; u < kDqChunks; ++u) {
      const int64_t e = base + u * 256;
      if (e >= n) break;  // chunks past the end are all later in the span
      uint32_t o[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c0 = (pk[u] >> (8 * j)) & 15, c1 = (pk[u] >> (8 * j + 4)) & 15;
        float l0, l1;
        if (QT == Q4_NF4) {
          l0 = s_lv[c0 * 32 + lane];
          l1 = s_lv[c1 * 32 + lane];
        } else if (QT == Q4_INT4_SYM) {
          l0 = (float)((c0 ^ 8) - 8);
          l1 = (float)((c1 ^ 8) - 8);
        } else {
          l0 = (float)(c0 - z[u]);
          l1 = (float)(c1 - z[u]);
        }
        o[j] = Dt<DOUT>::pack2(__fmul_rn(sc[u], l0), __fmul_rn(sc[u], l1));
      }
      if (e + 8 <= n) {
        *reinterpret_cast<uint4 *>(out + e) = make_uint4(o[0], o[1], o[2], o[3]);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (e + j < n) out[e + j] = (uint16_t)(o[j >> 1] >> (16 * (j & 1)));
      }
    }
  }
}

}  // namespace q4
