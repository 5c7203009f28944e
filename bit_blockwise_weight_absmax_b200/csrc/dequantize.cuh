// dequantize.cuh -- 4-bit codes back to 16-bit floats (sm_100a).
//
// n4n.ai, "What is 4-bit quantization and why does it matter?", code block
// "Conceptual NF4 dequantization" (dequantize_nf4: unpack the low nibble
// first, then NF4_VALUES[idx] times the block scale) and learn.pranaymahendrakar.com,
// "Loading a model in 4-bit", "Block-wise quantisation, stated exactly"
// (w^ = c * Q[i]); INT4 symmetric (n4n.ai "INT4 symmetric": w^ = q s) and
// asymmetric (robotsatlas.com "INT4", "How it works": w^ = (q - z) s).  Per
// element: one binary32 multiply of the block scale and the level (for
// INT4 asymmetric the exact integer q - z), rounded once to the output
// format.  With double quantization the scale is c~ = q2 * s2 + mu, two
// separately rounded operations.
//
// Design: the kernel reads 0.5 B and writes 2 B per element, so it is bound
// by HBM, and per byte of codes it must stay within a few instructions:
//   * a byte maps to the pair of its two levels (binary32: NF4 codebook
//     values, q - 8, or q) through a 256-entry table in shared memory, one
//     copy per lane, placed at a 64 KB-aligned shared address so that one
//     PRMT forms the entry's address (byte 1 = the code byte, byte 0 = the
//     lane's offset, bytes 2-3 = the table base); the two products come
//     from one packed f32x2 multiply and one convert-and-pack;
//   * one CTA of 32 warps per SM walks the spans of every matrix of the call
//     (one or a group) with a grid stride: a warp owns spans of 1024
//     elements; lane l expands the 8-element chunks l, l + 32, l + 64,
//     l + 96 of the span, so every 16-byte store instruction of the warp
//     covers 512 contiguous bytes and every 4-byte load of codes 128;
//   * the raw inputs of a warp's next span (codes, scale codes, group scales)
//     are loaded while the current one is expanded;
//   * spans that lie inside their matrix take a path without bounds checks.
#pragma once
#include "q4_common.cuh"

namespace q4 {

constexpr int kDqChunks = 4;                   // 8-element chunks per lane and span
constexpr int kDqSpan = 32 * 8 * kDqChunks;    // elements per warp and span
constexpr int kDqThreads = 1024;
constexpr int kDqSmem = 2 * 65536;             // room for a 64 KB-aligned table

// One matrix of a dequantize call.
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
  int32_t scale_f16;  // INT4: binary16 scales
  int64_t total_spans;
  float levels[16];
};

// The raw inputs of one span: loaded a span ahead, used a span later.
struct DqRaw {
  uint32_t pk[kDqChunks];  // 8 codes per chunk
  int q[kDqChunks];        // int8 scale code (double quant) / zero-point byte (INT4 asym)
  float s[kDqChunks];      // second-level scale (double quant) or the block scale
};

// Raw inputs of the span starting at element `base` of matrix m; WHOLE: the
// span lies inside the matrix (no bounds checks).
template <int QT, int B, bool DQ, bool WHOLE>
__device__ __forceinline__ void dq_load(const DqGMat &m, int64_t base, int lane, bool sf16, DqRaw &r) {
  const int64_t n = m.n;
  const uint8_t *pk_base = m.packed + base / 2 + lane * 4;  // chunk u at + 128 u
  const int64_t b_base = base / B;
#pragma unroll
  for (int u = 0; u < kDqChunks; ++u) {
    const uint32_t off = (uint32_t)(u * 256 + lane * 8);  // element offset inside the span
    r.pk[u] = 0u;
    r.q[u] = 0;
    r.s[u] = 0.0f;
    if (!WHOLE) {
      if (base + off >= n) continue;
      if (base + off + 8 > n) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (base + off + 2 * j < n) r.pk[u] |= (uint32_t)pk_base[u * 128 + j] << (8 * j);
      } else {
        r.pk[u] = ldg_stream_u32(pk_base + u * 128);
      }
    } else {
      r.pk[u] = ldg_stream_u32(pk_base + u * 128);
    }
    const int64_t b = b_base + (int64_t)(off / B);
    if (DQ) {
      r.q[u] = __ldg(m.absmax_q + b);
      r.s[u] = __ldg(m.absmax_scale + b / Q4_DQ_GROUP);
    } else {
      r.s[u] = ld_scale(m.absmax, b, sf16);
      if (QT == Q4_INT4_ASYM) r.q[u] = __ldg(m.zero + (b >> 1)) >> ((b & 1) * 4);
    }
  }
}

// Table entry of byte j of `word`: byte 1 of the address is the code byte;
// bytes 0, 2, 3 come from `lb` (64 KB-aligned table base + 8 * lane).
__device__ __forceinline__ uint64_t dq_pair(uint32_t word, int j, uint32_t lb) {
  const uint32_t a = __byte_perm(word, lb, 0x7604u | ((uint32_t)j << 4));
  uint64_t v;
  asm("ld.shared.b64 %0, [%1];" : "=l"(v) : "r"(a));
  return v;
}

// Expands one span (chunks past the end of the matrix are skipped unless
// WHOLE).
template <int QT, int DOUT, int B, bool DQ, bool WHOLE>
__device__ __forceinline__ void dq_emit(const DqGMat &m, int64_t base, int lane, uint32_t lb, float mu,
                                        const DqRaw &r) {
  const int64_t n = m.n;
  uint16_t *out = reinterpret_cast<uint16_t *>(m.out);
#pragma unroll
  for (int u = 0; u < kDqChunks; ++u) {
    const uint32_t off = (uint32_t)(u * 256 + lane * 8);
    if (!WHOLE && base + off >= n) break;  // chunks past the end are all later in the span
    const float sc = DQ ? __fadd_rn(__fmul_rn((float)r.q[u], r.s[u]), mu) : r.s[u];
    const uint64_t sc2 = f2_pack(sc, sc);
    const float nz = QT == Q4_INT4_ASYM ? -(float)(r.q[u] & 15) : 0.0f;
    const uint64_t nz2 = f2_pack(nz, nz);
    const uint32_t w = r.pk[u];
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint64_t l2 = dq_pair(w, j, lb);
      if (QT == Q4_INT4_ASYM) l2 = f2_add(l2, nz2);  // q - z, exact
      float p0, p1;
      f2_unpack(f2_mul(sc2, l2), p0, p1);
      o[j] = Dt<DOUT>::pack2(p0, p1);
    }
    const int64_t e = base + off;
    if (WHOLE || e + 8 <= n) {
      *reinterpret_cast<uint4 *>(out + e) = make_uint4(o[0], o[1], o[2], o[3]);
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (e + j < n) out[e + j] = (uint16_t)(o[j >> 1] >> (16 * (j & 1)));
    }
  }
}

// Every matrix of a call in one launch: the warps walk the spans of all
// matrices with a grid stride (the next span's loads, in whichever matrix it
// lies, are in flight while the current one is expanded).
template <int QT, int DOUT, int B, bool DQ>
__global__ void __launch_bounds__(kDqThreads, 1) dequantize_kernel(const __grid_constant__ DequantGroupParams p) {
  pdl_launch_dependents();  // the table below is built while the previous kernel drains
  static_assert(B % 8 == 0, "a chunk never straddles two blocks");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const int lane = threadIdx.x & 31;
  // the table at the first 64 KB boundary of the shared window
  const uint32_t lut = ((uint32_t)__cvta_generic_to_shared(smem_raw) + 0xFFFFu) & ~0xFFFFu;
  for (int i = threadIdx.x; i < 256 * 32; i += kDqThreads) {
    const int b = i >> 5, l = i & 31, c0 = b & 15, c1 = b >> 4;
    float v0, v1;
    if (QT == Q4_NF4) v0 = p.levels[c0], v1 = p.levels[c1];
    else if (QT == Q4_INT4_SYM) v0 = (float)((c0 ^ 8) - 8), v1 = (float)((c1 ^ 8) - 8);
    else v0 = (float)c0, v1 = (float)c1;
    asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(lut + (uint32_t)b * 256u + 8u * l), "f"(v0), "f"(v1)
                 : "memory");
  }
  __syncthreads();
  pdl_wait();
  const uint32_t lb = lut + 8u * (uint32_t)lane;
  const int wpb = kDqThreads / 32;
  const int64_t stride = (int64_t)gridDim.x * wpb;
  int64_t sp = (int64_t)blockIdx.x * wpb + (threadIdx.x >> 5);
  if (sp >= p.total_spans) return;
  int mi = 0;
  while (mi + 1 < p.count && sp >= p.mat[mi + 1].span_begin) ++mi;
  const bool sf16 = p.scale_f16 != 0;
  auto load = [&](int k, int64_t s, DqRaw &r) {
    const DqGMat &m = p.mat[k];
    const int64_t base = (s - m.span_begin) * kDqSpan;
    if (base + kDqSpan <= m.n) dq_load<QT, B, DQ, true>(m, base, lane, sf16, r);
    else dq_load<QT, B, DQ, false>(m, base, lane, sf16, r);
  };
  DqRaw cur;
  load(mi, sp, cur);
  while (sp < p.total_spans) {
    const int64_t nsp = sp + stride;
    int nmi = mi;
    DqRaw nxt;
    if (nsp < p.total_spans) {
      while (nmi + 1 < p.count && nsp >= p.mat[nmi + 1].span_begin) ++nmi;
      load(nmi, nsp, nxt);
    }
    const DqGMat &m = p.mat[mi];
    const float mu = DQ ? __ldg(m.absmax_mean) : 0.0f;
    const int64_t base = (sp - m.span_begin) * kDqSpan;
    if (base + kDqSpan <= m.n) dq_emit<QT, DOUT, B, DQ, true>(m, base, lane, lb, mu, cur);
    else dq_emit<QT, DOUT, B, DQ, false>(m, base, lane, lb, mu, cur);
    cur = nxt;
    sp = nsp;
    mi = nmi;
  }
}

}  // namespace q4
