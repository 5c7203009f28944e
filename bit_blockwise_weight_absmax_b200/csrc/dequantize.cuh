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

__device__ __forceinline__ float dq_lds(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}

// One span of kDqSpan elements starting at `base` (chunks past the end of
// the tensor are skipped).  lb: this lane's level table base (entry e of the
// lane at lb + 128 e).
template <int QT, int DOUT, int B, bool DQ>
__device__ __forceinline__ void dq_span(const DequantParams &p, int64_t base, int lane, uint32_t lb, float mu,
                                        uint16_t *out) {
  const int64_t n = p.n;
  const uint8_t *pk_base = p.packed + base / 2 + lane * 4;  // chunk u at + 128 u
  const int64_t b_base = base / B;
  uint32_t pk[kDqChunks];
  float sc[kDqChunks];
  int z[kDqChunks];
#pragma unroll
  for (int u = 0; u < kDqChunks; ++u) {
    const uint32_t off = (uint32_t)(u * 256 + lane * 8);  // element offset inside the span
    pk[u] = 0u;
    sc[u] = 0.0f;
    z[u] = 0;
    if (base + off >= n) continue;
    if (base + off + 8 <= n) {
      pk[u] = ldg_stream_u32(pk_base + u * 128);
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (base + off + 2 * j < n) pk[u] |= (uint32_t)pk_base[u * 128 + j] << (8 * j);
    }
    const int64_t b = b_base + (int64_t)(off / B);
    if (DQ) sc[u] = __fadd_rn(__fmul_rn((float)__ldg(p.absmax_q + b), __ldg(p.absmax_scale + b / Q4_DQ_GROUP)), mu);
    else sc[u] = __ldg(p.absmax + b);
    if (QT == Q4_INT4_ASYM) z[u] = (__ldg(p.zero + (b >> 1)) >> ((b & 1) * 4)) & 15;
  }
#pragma unroll
  for (int u = 0; u < kDqChunks; ++u) {
    const uint32_t off = (uint32_t)(u * 256 + lane * 8);
    if (base + off >= n) break;  // chunks past the end are all later in the span
    const uint32_t w = pk[u];
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float l0, l1;
      if (QT == Q4_NF4) {
        // code 2j at bits 8j..8j+3 and code 2j+1 at bits 8j+4..8j+7, moved
        // to bits 7..10 (the entry stride of 128 bytes)
        const uint32_t a0 = (j == 0 ? (w << 7) : (w >> (8 * j - 7))) & 0x780u;
        const uint32_t a1 = (j == 0 ? (w << 3) : (w >> (8 * j - 3))) & 0x780u;
        l0 = dq_lds(lb + a0);
        l1 = dq_lds(lb + a1);
      } else {
        const int c0 = (w >> (8 * j)) & 15, c1 = (w >> (8 * j + 4)) & 15;
        if (QT == Q4_INT4_SYM) {
          l0 = (float)((c0 ^ 8) - 8);
          l1 = (float)((c1 ^ 8) - 8);
        } else {
          l0 = (float)(c0 - z[u]);
          l1 = (float)(c1 - z[u]);
        }
      }
      o[j] = Dt<DOUT>::pack2(__fmul_rn(sc[u], l0), __fmul_rn(sc[u], l1));
    }
    const int64_t e = base + off;
    if (e + 8 <= n) {
      *reinterpret_cast<uint4 *>(out + e) = make_uint4(o[0], o[1], o[2], o[3]);
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (e + j < n) out[e + j] = (uint16_t)(o[j >> 1] >> (16 * (j & 1)));
    }
  }
}

template <int QT, int DOUT, int B, bool DQ>
__global__ void __launch_bounds__(kDqThreads, QT == Q4_INT4_ASYM ? 6 : 8) dequantize_kernel(const __grid_constant__ DequantParams p) {
  pdl_launch_then_wait();
  static_assert(B % 8 == 0, "a chunk never straddles two blocks");
  __shared__ float s_lv[16 * 32];  // [level][lane]
  const int lane = threadIdx.x & 31;
  if (QT == Q4_NF4) {
    for (int i = threadIdx.x; i < 16 * 32; i += blockDim.x) s_lv[i] = p.levels[i >> 5];
    __syncthreads();
  }
  const uint32_t lb = (uint32_t)__cvta_generic_to_shared(s_lv) + 4u * (uint32_t)lane;
  const float mu = DQ ? __ldg(p.absmax_mean) : 0.0f;
  uint16_t *out = reinterpret_cast<uint16_t *>(p.out);
  const int64_t n = p.n;
  const int64_t nspan = (n + kDqSpan - 1) / kDqSpan;
  const int wpb = blockDim.x >> 5;
  for (int64_t sp = (int64_t)blockIdx.x * wpb + (threadIdx.x >> 5); sp < nspan; sp += (int64_t)gridDim.x * wpb) {
    const int64_t base = sp * kDqSpan;
    dq_span<QT, DOUT, B, DQ>(p, base, lane, lb, mu, out);
  }
}

}  // namespace q4
