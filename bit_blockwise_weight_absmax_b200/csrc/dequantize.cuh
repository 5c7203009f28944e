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
// of packed codes covers 128 contiguous bytes.  The raw inputs of a warp's
// next span (codes, scale codes, group scales) are loaded while the current
// one is expanded, so two spans' loads overlap.  The 16 levels sit in shared
// memory, one copy per lane, so a warp's 32 lookups hit 32 distinct banks.
// A grouped launch walks the spans of several matrices (one layer) at once,
// so the launch ramp and tail are paid once per group.
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
// The raw inputs of one span: loaded a span ahead, used a span later.
struct DqRaw {
  uint32_t pk[kDqChunks];  // 8 codes per chunk
  int q[kDqChunks];        // int8 scale code (double quant) / zero-point byte (INT4 asym)
  float s[kDqChunks];      // second-level scale (double quant) or the block scale
};

template <int QT, int B, bool DQ, typename PP>
__device__ __forceinline__ void dq_load(const PP &p, int64_t base, int lane, DqRaw &r) {
  const int64_t n = p.n;
  const uint8_t *pk_base = p.packed + base / 2 + lane * 4;  // chunk u at + 128 u
  const int64_t b_base = base / B;
#pragma unroll
  for (int u = 0; u < kDqChunks; ++u) {
    const uint32_t off = (uint32_t)(u * 256 + lane * 8);  // element offset inside the span
    r.pk[u] = 0u;
    r.q[u] = 0;
    r.s[u] = 0.0f;
    if (base + off >= n) continue;
    if (base + off + 8 <= n) {
      r.pk[u] = ldg_stream_u32(pk_base + u * 128);
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (base + off + 2 * j < n) r.pk[u] |= (uint32_t)pk_base[u * 128 + j] << (8 * j);
    }
    const int64_t b = b_base + (int64_t)(off / B);
    if (DQ) {
      r.q[u] = __ldg(p.absmax_q + b);
      r.s[u] = __ldg(p.absmax_scale + b / Q4_DQ_GROUP);
    } else {
      r.s[u] = __ldg(p.absmax + b);
      if (QT == Q4_INT4_ASYM) r.q[u] = __ldg(p.zero + (b >> 1)) >> ((b & 1) * 4);
    }
  }
}

template <int QT, int DOUT, int B, bool DQ, typename PP>
__device__ __forceinline__ void dq_emit(const PP &p, int64_t base, int lane, uint32_t lb, float mu,
                                        uint16_t *out, const DqRaw &r) {
  const int64_t n = p.n;
#pragma unroll
  for (int u = 0; u < kDqChunks; ++u) {
    const uint32_t off = (uint32_t)(u * 256 + lane * 8);
    if (base + off >= n) break;  // chunks past the end are all later in the span
    const float sc = DQ ? __fadd_rn(__fmul_rn((float)r.q[u], r.s[u]), mu) : r.s[u];
    const int z = QT == Q4_INT4_ASYM ? (r.q[u] & 15) : 0;
    const uint32_t w = r.pk[u];
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float l0, l1;
      if (QT == Q4_NF4) {
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
          l0 = (float)(c0 - z);
          l1 = (float)(c1 - z);
        }
      }
      o[j] = Dt<DOUT>::pack2(__fmul_rn(sc, l0), __fmul_rn(sc, l1));
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

// Resident CTAs per SM: the registers of two spans' raw inputs.
template <int QT> constexpr int dq_ctas_per_sm() { return QT == Q4_INT4_ASYM ? 4 : 5; }

template <int QT, int DOUT, int B, bool DQ>
__global__ void __launch_bounds__(kDqThreads, dq_ctas_per_sm<QT>()) dequantize_kernel(const __grid_constant__ DequantParams p) {
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
  const int64_t nspan = (p.n + kDqSpan - 1) / kDqSpan;
  const int wpb = blockDim.x >> 5;
  const int64_t stride = (int64_t)gridDim.x * wpb;
  int64_t sp = (int64_t)blockIdx.x * wpb + (threadIdx.x >> 5);
  if (sp >= nspan) return;
  DqRaw cur;
  dq_load<QT, B, DQ>(p, sp * kDqSpan, lane, cur);
  for (; sp < nspan; sp += stride) {
    // the next span's loads are in flight while this one is expanded
    DqRaw nxt;
    if (sp + stride < nspan) dq_load<QT, B, DQ>(p, (sp + stride) * kDqSpan, lane, nxt);
    dq_emit<QT, DOUT, B, DQ>(p, sp * kDqSpan, lane, lb, mu, out, cur);
    cur = nxt;
  }
}

// One matrix of a grouped dequantize.
struct DqGMat {
  const uint8_t *packed;
  const float *absmax;
  const uint8_t *zero;
  const int8_t *absmax_q;
  const float *absmax_scale;
  const float *absmax_mean;
  int64_t n;
  void *out;
  int64_t span_begin;  // first global span of this matrix
};
constexpr int kDqMaxGroup = 16;
struct DequantGroupParams {
  DqGMat mat[kDqMaxGroup];
  int32_t count;
  int64_t total_spans;
  float levels[16];
};

// Every matrix of a group in one launch: the warps walk the spans of all
// matrices with a grid stride (the next span's loads, in whichever matrix it
// lies, are in flight while the current one is expanded).
template <int QT, int DOUT, int B, bool DQ>
__global__ void __launch_bounds__(kDqThreads, dq_ctas_per_sm<QT>())
    dequantize_grouped_kernel(const __grid_constant__ DequantGroupParams p) {
  pdl_launch_then_wait();
  static_assert(B % 8 == 0, "a chunk never straddles two blocks");
  __shared__ float s_lv[16 * 32];  // [level][lane]
  const int lane = threadIdx.x & 31;
  if (QT == Q4_NF4) {
    for (int i = threadIdx.x; i < 16 * 32; i += blockDim.x) s_lv[i] = p.levels[i >> 5];
    __syncthreads();
  }
  const uint32_t lb = (uint32_t)__cvta_generic_to_shared(s_lv) + 4u * (uint32_t)lane;
  const int wpb = blockDim.x >> 5;
  const int64_t stride = (int64_t)gridDim.x * wpb;
  int64_t sp = (int64_t)blockIdx.x * wpb + (threadIdx.x >> 5);
  if (sp >= p.total_spans) return;
  int mi = 0;
  while (mi + 1 < p.count && sp >= p.mat[mi + 1].span_begin) ++mi;
  DqRaw cur;
  dq_load<QT, B, DQ>(p.mat[mi], (sp - p.mat[mi].span_begin) * kDqSpan, lane, cur);
  while (sp < p.total_spans) {
    const int64_t nsp = sp + stride;
    int nmi = mi;
    DqRaw nxt;
    if (nsp < p.total_spans) {
      while (nmi + 1 < p.count && nsp >= p.mat[nmi + 1].span_begin) ++nmi;
      dq_load<QT, B, DQ>(p.mat[nmi], (nsp - p.mat[nmi].span_begin) * kDqSpan, lane, nxt);
    }
    const DqGMat &m = p.mat[mi];
    const float mu = DQ ? __ldg(m.absmax_mean) : 0.0f;
    dq_emit<QT, DOUT, B, DQ>(m, (sp - m.span_begin) * kDqSpan, lane, lb, mu, reinterpret_cast<uint16_t *>(m.out),
                             cur);
    cur = nxt;
    sp = nsp;
    mi = nmi;
  }
}

}  // namespace q4
