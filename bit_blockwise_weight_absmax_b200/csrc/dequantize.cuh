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
// Design: a thread expands 16 codes (8 packed bytes, one block) into 32 bytes
// of output; reads 0.5 B and writes 2 B per element, so the kernel is bound by
// HBM.  The 16 levels sit in shared memory, one copy per lane, so a warp's
// 32 lookups hit 32 distinct banks.
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

template <int QT, int DOUT, int B, bool DQ>
__global__ void __launch_bounds__(256) dequantize_kernel(DequantParams p) {
  __shared__ float s_lv[16 * 32];
  const int lane = threadIdx.x & 31;
  if (QT == Q4_NF4) {
    for (int i = threadIdx.x; i < 16 * 32; i += blockDim.x) s_lv[i] = p.levels[i >> 5];
    __syncthreads();
  }
  const float mu = DQ ? __ldg(p.absmax_mean) : 0.0f;
  uint16_t *out = reinterpret_cast<uint16_t *>(p.out);
  const int64_t ngroups = (p.n + 15) / 16;
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < ngroups;
       t += (int64_t)gridDim.x * blockDim.x) {
    const int64_t e0 = t * 16;
    const int64_t b = e0 / B;
    float sc;
    if (DQ) sc = __fadd_rn(__fmul_rn((float)__ldg(p.absmax_q + b), __ldg(p.absmax_scale + b / Q4_DQ_GROUP)), mu);
    else sc = __ldg(p.absmax + b);
    int z = 0;
    if (QT == Q4_INT4_ASYM) z = (__ldg(p.zero + (b >> 1)) >> ((b & 1) * 4)) & 15;
    const bool full = e0 + 16 <= p.n;
    uint2 pk;
    if (full) {
      pk = ldg_stream_v2(p.packed + e0 / 2);
    } else {
      uint8_t t8[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) t8[j] = (e0 + 2 * j < p.n) ? p.packed[e0 / 2 + j] : 0;
      pk.x = t8[0] | (t8[1] << 8) | (t8[2] << 16) | ((uint32_t)t8[3] << 24);
      pk.y = t8[4] | (t8[5] << 8) | (t8[6] << 16) | ((uint32_t)t8[7] << 24);
    }
    uint32_t o[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t word = j < 4 ? pk.x : pk.y;
      const int c0 = (word >> (8 * (j & 3))) & 15, c1 = (word >> (8 * (j & 3) + 4)) & 15;
      float l0, l1;
      if (QT == Q4_NF4) {
        l0 = s_lv[c0 * 32 + lane];
        l1 = s_lv[c1 * 32 + lane];
      } else if (QT == Q4_INT4_SYM) {
        l0 = (float)((c0 ^ 8) - 8);
        l1 = (float)((c1 ^ 8) - 8);
      } else {
        l0 = (float)(c0 - z);
        l1 = (float)(c1 - z);
      }
      o[j] = Dt<DOUT>::pack2(__fmul_rn(sc, l0), __fmul_rn(sc, l1));
    }
    if (full) {
      uint4 *dst = reinterpret_cast<uint4 *>(out + e0);
      dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
      dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    } else {
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (e0 + j < p.n) out[e0 + j] = (uint16_t)(o[j >> 1] >> (16 * (j & 1)));
    }
  }
}

}  // namespace q4
