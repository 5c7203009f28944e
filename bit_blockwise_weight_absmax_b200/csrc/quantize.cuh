// quantize.cuh -- blockwise 4-bit quantization kernels (sm_100a).
//
// Defines (learn.pranaymahendrakar.com, "Loading a model in 4-bit", section
// "Block-wise quantisation, stated exactly"): contiguous blocks of B over the
// flattened row-major weights; per block c = max|w|; every weight is divided
// by c and mapped to the nearest of the 16 levels (NF4 levels from n4n.ai,
// "What is 4-bit quantization and why does it matter?", code block
// "Conceptual NF4 dequantization"); two codes per byte, low nibble first.
// INT4 symmetric (n4n.ai "INT4 symmetric": -8..7, s = max|w|/7) and INT4
// asymmetric (robotsatlas.com "INT4", "How it works"/"Components": [0,15]
// with an integer zero-point) share the kernel.  Double quantization of the
// absmax ("blocks of 256, to 8 bits") is a second kernel.
//
// Design: one streaming pass over W.  A thread owns 16 consecutive elements
// (one 128-bit load); B/8 adjacent lanes own one block and reduce its absmax
// with xor shuffles.  A CTA (256 threads) walks 256-block chunks (the
// double-quant groups); each CTA owns a contiguous, power-of-two-aligned run
// of chunks so that the fp64 pairwise sum of the block absmax values used for
// the double-quant mean is formed in the exact order of the definition (an
// aligned binary tree) without atomics: lanes -> chunk (shared memory tree)
// -> CTA run (streaming pairwise stack) -> the last CTA to finish combines the
// per-CTA partial sums and writes the mean.  The grouped launch over every
// matrix of a layer (quantize_grouped.cuh) shares the per-thread step,
// quant16; one second launch then quantizes every matrix's groups of absmax
// values.
#pragma once

#include "q4_common.cuh"

namespace q4 {

constexpr int kQThreads = 256;
constexpr int kChunkBlocks = Q4_DQ_GROUP;  // 256 blocks per chunk
constexpr int kMaxRunPartials = 2048;      // per-CTA partial sums combined by the last CTA

// NF4 coding table: x (the exact binary32 quotient w / c) falls in bin
// j = round(15 x) + 15 computed as the low 5 bits of fmaf(x, 15, 2^23*1.5 + 15);
// each bin holds at most one decision threshold t, so
// code = base[j] + (x >= thr[j]) with thr = +inf for bins without one.
struct Nf4BinTable {
  float thr[32];
  int base[32];
};

__device__ __forceinline__ uint32_t nf4_bin(float x) {
  return __float_as_uint(__fmaf_rn(x, 15.0f, 12582927.0f)) & 31u;
}

struct QuantParams {
  const uint16_t *W;
  int64_t n, nb;
  int64_t n_chunks;       // ceil(nb / 256)
  int64_t run;            // chunks per CTA (power of two)
  uint8_t *packed;
  float *absmax;
  uint8_t *zero;
  double *partials;       // [gridDim.x] fp64 pairwise sums (double quant)
  unsigned *counter;      // arrival counter (double quant), left at 0
  float *absmax_mean;     // mean output (double quant)
  int *status;            // sticky status word
  int32_t scale_f16;      // INT4: binary16 scales
  Nf4BinTable tab;
};

// One matrix of a grouped launch.
struct QMat {
  const uint16_t *W;
  int64_t n, nb;
  int64_t n_chunks;
  int64_t chunk_begin;  // first global chunk of this matrix
  uint8_t *packed;
  float *absmax;
  uint8_t *zero;
  float *absmax_mean;   // double quant
  double *partials;     // [n_chunks] fp64 pairwise sums of the chunks (double quant)
  unsigned *counter;    // chunks done (double quant), left at 0
};
constexpr int kQMaxGroup = 16;

struct QuantGroupParams {
  QMat mat[kQMaxGroup];
  int32_t count;
  int32_t stall_copies;  // test hook: the producer never fills a stage
  int64_t total_chunks;
  uint64_t wait_ns;      // bound of every mbarrier wait
  int *status;
  int32_t scale_f16;     // INT4: binary16 scales
  Nf4BinTable tab;
};

// Absolute value of eight 16-bit floats as a max over (bits & 0x7fff): the
// order of magnitudes of IEEE 16-bit floats is the integer order of these
// patterns, and NaN / Inf sort above every finite value.
__device__ __forceinline__ uint32_t absmax_bits8(uint4 v) {
  uint32_t a = __vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu);
  uint32_t b = __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu);
  uint32_t m = __vmaxu2(a, b);
  return max(m & 0xFFFFu, m >> 16);
}

// NF4 code of x = RN(w / c) for |x| <= 1 (w finite) from `bits`, the
// pattern of fmaf(x, 15, 1.5 * 2^23 + 15): the bin is its low byte (0..30),
// the pattern is 0x4B4000jj, so (bits << 8) = 0x40000000 + 256 j and `tb` =
// table address of this lane minus 0x40000000 gives the entry of bin j
// (32-bit shared addresses wrap).
__device__ __forceinline__ uint32_t nf4_code_bits(uint32_t bits, float x, uint32_t tb) {
  float thr;
  int base;
  asm("ld.shared.v2.b32 {%0,%1}, [%2];" : "=f"(thr), "=r"(base) : "r"((bits << 8) + tb));
  return (uint32_t)(base + (x >= thr ? 1 : 0));
}

// Codes of a thread's 16 consecutive elements (element 8k + j in bits
// 4j..4j+3 of codes[k]) and its block's scale; the B/16 lanes of one block
// (adjacent lanes) agree on `scale` and `z`.  Must be called by all 32 lanes.
// tb: this lane's bin-table address minus 2^30; s_tab: the lane-private
// bin tables ([bin][lane]); nonfinite is set when the block holds Inf / NaN.
// sf16 (INT4): the scale is rounded to binary16 as soon as it is formed and
// the codes are computed against the rounded value.
template <int DT, int QT, int B>
__device__ __forceinline__ void quant16(const uint4 (&v)[2], float &scale, int &z, uint32_t (&codes)[2], int lane,
                                        uint32_t tb, const float2 *s_tab, int &nonfinite, bool sf16 = false) {
  constexpr int E = 16, V = 2, LPB = B / E;
  float f[E];
#pragma unroll
  for (int k = 0; k < V; ++k) {
    const uint32_t w[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      f[8 * k + 2 * j] = lo16<DT>(w[j]);
      f[8 * k + 2 * j + 1] = hi16<DT>(w[j]);
    }
    codes[k] = 0;
  }
  if (QT == Q4_NF4 || QT == Q4_INT4_SYM) {
    uint32_t m = absmax_bits8(v[0]);
#pragma unroll
    for (int k = 1; k < V; ++k) m = max(m, absmax_bits8(v[k]));
#pragma unroll
    for (int o = LPB / 2; o >= 1; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float c = Dt<DT>::to_f((uint16_t)m);
    if (!(c <= 3.4028235e38f)) nonfinite = 1;
    if (QT == Q4_NF4) {
      scale = c;
      if (__all_sync(0xffffffffu, markstein_ok(c))) {
        // every lane: finite weights with |w| <= c, so |x| <= 1; the
        // quotients and bins of two weights per packed instruction
        const float y = __frcp_rn(c);
        const uint64_t yy = f2_pack(y, y), nc = f2_pack(-c, -c);
        const uint64_t k15 = f2_pack(15.0f, 15.0f), kbin = f2_pack(12582927.0f, 12582927.0f);
#pragma unroll
        for (int k = 0; k < V; ++k)
#pragma unroll
          for (int j = 3; j >= 0; --j) {
            const uint64_t x2 = div_markstein2(f2_pack(f[8 * k + 2 * j], f[8 * k + 2 * j + 1]), nc, yy);
            const uint64_t b2 = f2_fma(x2, k15, kbin);
            float x0, x1, b0, b1;
            f2_unpack(x2, x0, x1);
            f2_unpack(b2, b0, b1);
            codes[k] = (codes[k] << 4) + nf4_code_bits(__float_as_uint(b1), x1, tb);
            codes[k] = (codes[k] << 4) + nf4_code_bits(__float_as_uint(b0), x0, tb);
          }
      } else {
        const bool fast = markstein_ok(c);
        const float y = fast ? __frcp_rn(c) : 0.0f;
#pragma unroll
        for (int j = 0; j < E; ++j) {
          float x = fast ? div_markstein(f[j], c, y) : (c == 0.0f ? 0.0f : __fdiv_rn(f[j], c));
          const float2 e = s_tab[nf4_bin(x) * 32 + lane];
          const int code = __float_as_int(e.y) + (x >= e.x ? 1 : 0);
          codes[j >> 3] |= (uint32_t)code << (4 * (j & 7));
        }
      }
    } else {
      float s = __fdiv_rn(c, 7.0f);
      if (sf16) s = __half2float(__float2half_rn(s));
      scale = s;
      if (__all_sync(0xffffffffu, markstein_ok(s))) {
        // binary32 s: |w / s| <= 7 / (1 - 2^-24), so rint never leaves
        // [-7, 7], and adding 1.5 * 2^23 rounds to the nearest integer, ties
        // to even, leaving its 4-bit two's complement in the low nibble
        const float y = __frcp_rn(s);
        const uint64_t yy = f2_pack(y, y), ns = f2_pack(-s, -s);
        const uint64_t kr = f2_pack(12582912.0f, 12582912.0f);
        if (!sf16) {
#pragma unroll
          for (int k = 0; k < V; ++k)
#pragma unroll
            for (int j = 3; j >= 0; --j) {
              const uint64_t r2 =
                  f2_add(div_markstein2(f2_pack(f[8 * k + 2 * j], f[8 * k + 2 * j + 1]), ns, yy), kr);
              float r0, r1;
              f2_unpack(r2, r0, r1);
              codes[k] = (codes[k] << 8) | ((__float_as_uint(r1) & 15u) << 4) | (__float_as_uint(r0) & 15u);
            }
        } else {
          // a binary16 s can lie well below c / 7 (a subnormal keeps few
          // bits), so the rounded quotient is clamped to [-8, 7]; it stays
          // far below 2^22, where the 1.5 * 2^23 rounding holds
#pragma unroll
          for (int k = 0; k < V; ++k)
#pragma unroll
            for (int j = 3; j >= 0; --j) {
              const uint64_t r2 =
                  f2_add(div_markstein2(f2_pack(f[8 * k + 2 * j], f[8 * k + 2 * j + 1]), ns, yy), kr);
              float r0, r1;
              f2_unpack(r2, r0, r1);
              const int q0 = min(max((int)(__float_as_uint(r0) - 0x4B400000u), -8), 7);
              const int q1 = min(max((int)(__float_as_uint(r1) - 0x4B400000u), -8), 7);
              codes[k] = (codes[k] << 8) | ((uint32_t)(q1 & 15) << 4) | (uint32_t)(q0 & 15);
            }
        }
      } else {
        const bool fast = markstein_ok(s);
        const float y = fast ? __frcp_rn(s) : 0.0f;
#pragma unroll
        for (int j = 0; j < E; ++j) {
          int q = 0;
          if (s != 0.0f) {
            float x = fast ? div_markstein(f[j], s, y) : __fdiv_rn(f[j], s);
            q = min(max(__float2int_rn(x), -8), 7);
          }
          codes[j >> 3] |= (uint32_t)(q & 15) << (4 * (j & 7));
        }
      }
    }
  } else {  // Q4_INT4_ASYM
    float mn = 0.0f, mx = 0.0f;
#pragma unroll
    for (int j = 0; j < E; ++j) {
      mn = fminf(mn, f[j]);
      mx = fmaxf(mx, f[j]);
    }
    uint32_t m = absmax_bits8(v[0]);
#pragma unroll
    for (int k = 1; k < V; ++k) m = max(m, absmax_bits8(v[k]));
#pragma unroll
    for (int o = LPB / 2; o >= 1; o >>= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    }
    if (!(Dt<DT>::to_f((uint16_t)m) <= 3.4028235e38f)) nonfinite = 1;
    float s = __fdiv_rn(__fsub_rn(mx, mn), 15.0f);
    if (sf16) s = __half2float(__float2half_rn(s));
    scale = s;
    z = 0;
    if (__all_sync(0xffffffffu, markstein_ok(s))) {
      // mn <= 0 <= mx and s = (mx - mn) / 15, so |w / s| <= 15 (1 + 2^-23)
      // (a few times that for a binary16 s rounded to a subnormal; the code
      // is clamped): adding 1.5 * 2^23 rounds the quotient to the nearest
      // integer, ties to even, with the integer in the low bits of the
      // sum's pattern
      const float y = __frcp_rn(s);
      z = min(max(__float2int_rn(div_markstein(-mn, s, y)), 0), 15);
      const uint64_t yy = f2_pack(y, y), ns = f2_pack(-s, -s);
      const uint64_t kr = f2_pack(12582912.0f, 12582912.0f);
#pragma unroll
      for (int k = 0; k < V; ++k)
#pragma unroll
        for (int j = 3; j >= 0; --j) {
          const uint64_t r2 = f2_add(div_markstein2(f2_pack(f[8 * k + 2 * j], f[8 * k + 2 * j + 1]), ns, yy), kr);
          float r0, r1;
          f2_unpack(r2, r0, r1);
          const int q0 = min(max((int)(__float_as_uint(r0) - 0x4B400000u) + z, 0), 15);
          const int q1 = min(max((int)(__float_as_uint(r1) - 0x4B400000u) + z, 0), 15);
          codes[k] = (codes[k] << 8) | ((uint32_t)q1 << 4) | (uint32_t)q0;
        }
    } else {
      if (s != 0.0f) z = min(max(__float2int_rn(__fdiv_rn(-mn, s)), 0), 15);
      const bool fast = markstein_ok(s);
      const float y = fast ? __frcp_rn(s) : 0.0f;
#pragma unroll
      for (int j = 0; j < E; ++j) {
        int q = 0;
        if (s != 0.0f) {
          float x = fast ? div_markstein(f[j], s, y) : __fdiv_rn(f[j], s);
          q = min(max(__float2int_rn(x) + z, 0), 15);
        }
        codes[j >> 3] |= (uint32_t)q << (4 * (j & 7));
      }
    }
  }
}

// Four resident CTAs of 256 threads per SM (at most 64 registers): more
// warps to hide the division and table latencies, with four 16-byte loads
// in flight per thread.
// One matrix; each CTA owns one run of chunks.
template <int DT, int QT, int B, bool DQ>
__global__ void __launch_bounds__(kQThreads, 4) quantize_kernel(const __grid_constant__ QuantParams p) {
  pdl_launch_then_wait();
  constexpr int E = 16;                          // consecutive elements per thread (one block)
  constexpr int V = E / 8;                       // 16-byte words per thread
  constexpr int LPB = B / E;                     // lanes per block
  constexpr int ELEMS_IT = kQThreads * E;        // elements per CTA iteration
  constexpr int IT_PER_CHUNK = kChunkBlocks * B / ELEMS_IT;  // = B / 16
  constexpr int BLK_IT = ELEMS_IT / B;           // blocks per CTA iteration
  constexpr int BATCH = IT_PER_CHUNK < 2 ? IT_PER_CHUNK : 2;  // iterations of loads in flight
  static_assert(B % E == 0, "a thread's elements lie in one block");
  static_assert(V == 2, "the packed codes of a thread are one 8-byte store");
  constexpr int64_t CHUNK_ELEMS = (int64_t)kChunkBlocks * B;

  __shared__ float2 s_tab[32 * 32];              // lane-private copies of the bin table
  __shared__ double s_blk[2][kChunkBlocks];      // block absmax of a chunk, by chunk parity
  __shared__ uint8_t s_zero[BLK_IT];             // INT4_ASYM zero-points of one iteration
  __shared__ double s_stack[24];                 // streaming pairwise stack (thread 0)
  __shared__ int s_last;

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  if (QT == Q4_NF4) {
    for (int i = tid; i < 32 * 32; i += kQThreads) {
      int e = i >> 5;
      s_tab[i] = make_float2(p.tab.thr[e], __int_as_float(p.tab.base[e]));
    }
  }
  __syncthreads();
  const uint32_t tlane = (uint32_t)__cvta_generic_to_shared(s_tab) + 8u * lane;  // bin 0, this lane
  const uint32_t tb = tlane - 0x40000000u;

  int nonfinite = 0;
  int depth = 0;  // stack depth (thread 0)
  int cpar = 0;   // parity of s_blk for the current chunk

  // One chunk (256 blocks) of a matrix; with double quantization returns the
  // fp64 pairwise sum of its block absmax values (valid in thread 0).
  auto do_chunk = [&](const uint16_t *W, int64_t n, int64_t nb, uint8_t *packed, float *absmax, uint8_t *zero,
                      int64_t chunk) -> double {
    double chunk_sum = 0.0;
    const int64_t chunk_e0 = chunk * CHUNK_ELEMS;
    const int64_t chunk_b0 = chunk * kChunkBlocks;
    // FULL: the whole chunk lies inside the tensor (every chunk but the last)
    auto run_chunk = [&](auto full_tag) {
      constexpr bool FULL = decltype(full_tag)::value;
      const uint16_t *wp = W + chunk_e0 + tid * E;
      uint8_t *pp = packed + chunk_e0 / 2 + tid * (E / 2);
      for (int it0 = 0; it0 < IT_PER_CHUNK; it0 += BATCH) {
        uint4 v[BATCH][V];
#pragma unroll
        for (int b = 0; b < BATCH; ++b) {
          const int off = (it0 + b) * ELEMS_IT;
#pragma unroll
          for (int k = 0; k < V; ++k) {
            if (FULL) {
              v[b][k] = ldg_stream_v4(wp + off + 8 * k);
            } else {
              const int64_t e0 = chunk_e0 + off + tid * E + 8 * k;
              if (e0 + 8 <= n) {
                v[b][k] = ldg_stream_v4(wp + off + 8 * k);
              } else {
                uint16_t t[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) t[j] = (e0 + j < n) ? W[e0 + j] : (uint16_t)0;
                v[b][k] = make_uint4(t[0] | (t[1] << 16), t[2] | (t[3] << 16), t[4] | (t[5] << 16),
                                     t[6] | (t[7] << 16));
              }
            }
          }
        }
#pragma unroll
        for (int b = 0; b < BATCH; ++b) {
          const int it = it0 + b;
          const int off = it * ELEMS_IT;
          const int bl = it * BLK_IT + (tid * E) / B;  // block within the chunk
          float scale = 0.0f;
          int z = 0;
          uint32_t codes[V];
          quant16<DT, QT, B>(v[b], scale, z, codes, lane, tb, s_tab, nonfinite, p.scale_f16 != 0);
          if (QT == Q4_INT4_ASYM && (tid % LPB) == 0) s_zero[(tid * E) / B] = (uint8_t)z;
          // ---- stores
          const int64_t e0 = chunk_e0 + off + tid * E;
          if (FULL || e0 + E <= n) {
            *reinterpret_cast<uint2 *>(pp + off / 2) = make_uint2(codes[0], codes[1]);
          } else if (e0 < n) {
            const int valid = (int)(n - e0);
#pragma unroll
            for (int j = 0; j < E / 2; ++j) {
              if (2 * j < valid) {
                uint32_t byte = (codes[j >> 2] >> (8 * (j & 3))) & 0xFFu;
                if (2 * j + 1 >= valid) byte &= 0x0Fu;  // odd n: high nibble is padding
                pp[off / 2 + j] = (uint8_t)byte;
              }
            }
          }
          if ((tid % LPB) == 0) {
            const bool in = FULL || chunk_b0 + bl < nb;
            if (in) st_scale(absmax, chunk_b0 + bl, scale, p.scale_f16 != 0);
            if (DQ) s_blk[cpar][bl] = in ? (double)scale : 0.0;
          }
          if (QT == Q4_INT4_ASYM) {
            __syncthreads();
            if (tid < BLK_IT / 2) {
              const int64_t b0 = chunk_b0 + it * BLK_IT + 2 * tid;
              if (b0 < nb) zero[b0 / 2] = (uint8_t)(s_zero[2 * tid] | (s_zero[2 * tid + 1] << 4));
            }
            __syncthreads();
          }
        }
      }
    };
    if (chunk_e0 + CHUNK_ELEMS <= n) run_chunk(std::true_type{});
    else run_chunk(std::false_type{});
    if (DQ) {
      // Pairwise fp64 sum of the chunk's 256 block values in tree order:
      // lane l reduces blocks 8l..8l+7 as ((0+1)+(2+3))+((4+5)+(6+7)), then
      // xor shuffles at distance 1, 2, 4, 8, 16 pair adjacent subtrees.  One
      // barrier: the next chunk writes the other parity.
      __syncthreads();
      if (tid < 32) {
        const double *q = s_blk[cpar] + 8 * tid;
        double s = ((q[0] + q[1]) + (q[2] + q[3])) + ((q[4] + q[5]) + (q[6] + q[7]));
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) s = s + __shfl_xor_sync(0xffffffffu, s, o);
        if (tid == 0) {
          // streaming pairwise stack over the CTA's run of chunks: merging
          // equal-size neighbours reproduces the aligned binary tree
          chunk_sum = s;
        }
      }
      cpar ^= 1;
    }
    return chunk_sum;
  };

  {
    const int64_t c0 = (int64_t)blockIdx.x * p.run;
    const int64_t c1 = min(c0 + p.run, p.n_chunks);
    for (int64_t chunk = c0; chunk < c1; ++chunk) {
      const double cs = do_chunk(p.W, p.n, p.nb, p.packed, p.absmax, p.zero, chunk);
      if (DQ && tid == 0) {
        // streaming pairwise stack over the CTA's run of chunks: merging
        // equal-size neighbours reproduces the aligned binary tree
        s_stack[depth++] = cs;
        for (int64_t k = chunk - c0 + 1; (k & 1) == 0; k >>= 1) {
          s_stack[depth - 2] = s_stack[depth - 2] + s_stack[depth - 1];
          --depth;
        }
      }
    }
  }

  if (nonfinite) raise_status(p.status, Q4_STATUS_NONFINITE);

  if constexpr (DQ) {
    const int64_t c0 = (int64_t)blockIdx.x * p.run;
    const int64_t c1 = min(c0 + p.run, p.n_chunks);
    if (tid == 0) {
      // pad the run with zero chunks up to its power-of-two length
      for (int64_t k = c1 - c0; k < p.run; ++k) {
        s_stack[depth++] = 0.0;
        for (int64_t kk = k + 1; (kk & 1) == 0; kk >>= 1) {
          s_stack[depth - 2] = s_stack[depth - 2] + s_stack[depth - 1];
          --depth;
        }
      }
      p.partials[blockIdx.x] = (c1 > c0 || p.run > 0) ? s_stack[0] : 0.0;
      __threadfence();
      const unsigned ticket = atomicAdd(p.counter, 1u);
      s_last = (ticket == gridDim.x - 1);
    }
    __syncthreads();
    if (s_last) {
      // the last CTA: pairwise tree over the per-CTA partials (aligned
      // subtrees of `run` chunks), level by level, odd last carried up
      __threadfence();
      __shared__ double s_red[kMaxRunPartials];
      int len = gridDim.x;
      for (int i = tid; i < len; i += kQThreads) {
        s_red[i] = __ldcg(p.partials + i);
        __stcg(p.partials + i, 0.0);  // the workspace is left zeroed
      }
      __syncthreads();
      while (len > 1) {
        const int half = len >> 1;
        double t[kMaxRunPartials / kQThreads / 2 + 1];
        int cnt = 0;
        for (int i = tid; i < half; i += kQThreads) t[cnt++] = s_red[2 * i] + s_red[2 * i + 1];
        double carry = s_red[len - 1];
        __syncthreads();
        cnt = 0;
        for (int i = tid; i < half; i += kQThreads) s_red[i] = t[cnt++];
        if ((len & 1) && tid == 0) s_red[half] = carry;
        __syncthreads();
        len = half + (len & 1);
      }
      if (tid == 0) {
        const double S = s_red[0];
        p.absmax_mean[0] = __double2float_rn(__ddiv_rn(S, (double)p.nb));
        *p.counter = 0u;  // leave the workspace zeroed for the next call
      }
    }
  }
}

// One matrix's double-quant state for the grouped second-level kernel.
struct DqMat {
  const float *absmax;
  int64_t nb;
  const float *mean;
  int8_t *absmax_q;
  float *absmax_scale;
  int64_t group_begin;  // first global group of this matrix
};
struct DqGroupParams {
  DqMat mat[kQMaxGroup];
  int32_t count;
  int64_t total_groups;
};

// One group of 256 block absmax values, by one warp:
// m2 = max|c - mu|, s2 = m2 / 127, q2 = clamp(rint((c - mu) / s2), -128, 127).
// Lane l owns blocks 8l..8l+7 of the group: two 16-byte loads and one 8-byte
// store when the group is whole and the arrays are aligned for them.  The
// quotients are correctly rounded (Markstein's correction where the divisor
// allows it, as in the first-level quantizer; IEEE division otherwise).
__device__ __forceinline__ void double_quant_group(const float *__restrict__ absmax, int64_t nb, float mu,
                                                   int8_t *__restrict__ absmax_q, float *__restrict__ absmax_scale,
                                                   int64_t g, int lane) {
  const int64_t b0 = g * Q4_DQ_GROUP + lane * 8;
  const bool vec = g * Q4_DQ_GROUP + Q4_DQ_GROUP <= nb && ((uintptr_t)absmax & 15u) == 0 &&
                   ((uintptr_t)absmax_q & 7u) == 0;
  float d[8];
  float m2 = 0.0f;
  if (vec) {
    const float4 x0 = __ldg(reinterpret_cast<const float4 *>(absmax + b0));
    const float4 x1 = __ldg(reinterpret_cast<const float4 *>(absmax + b0 + 4));
    const float x[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      d[j] = __fsub_rn(x[j], mu);
      m2 = fmaxf(m2, fabsf(d[j]));
    }
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      d[j] = (b0 + j < nb) ? __fsub_rn(__ldg(absmax + b0 + j), mu) : 0.0f;
      if (b0 + j < nb) m2 = fmaxf(m2, fabsf(d[j]));
    }
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) m2 = fmaxf(m2, __shfl_xor_sync(0xffffffffu, m2, o));
  const float s2 = __fdiv_rn(m2, 127.0f);
  if (lane == 0) absmax_scale[g] = s2;
  const bool fast = markstein_ok(s2);
  const float y = fast ? __frcp_rn(s2) : 0.0f;
  uint32_t q[2] = {0u, 0u};
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    int q2 = 0;
    if (s2 != 0.0f) {
      const float x = fast ? div_markstein(d[j], s2, y) : __fdiv_rn(d[j], s2);
      q2 = min(max(__float2int_rn(x), -128), 127);
    }
    q[j >> 2] |= (uint32_t)(q2 & 0xFF) << (8 * (j & 3));
  }
  if (vec) {
    *reinterpret_cast<uint2 *>(absmax_q + b0) = make_uint2(q[0], q[1]);
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (b0 + j < nb) absmax_q[b0 + j] = (int8_t)(q[j >> 2] >> (8 * (j & 3)));
  }
}

// The groups of every matrix of a grouped quantize, one warp per group.
static __global__ void __launch_bounds__(256) double_quant_grouped_kernel(const __grid_constant__ DqGroupParams p) {
  pdl_launch_then_wait();
  const int64_t g = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (g >= p.total_groups) return;
  int mi = 0;
  while (mi + 1 < p.count && g >= p.mat[mi + 1].group_begin) ++mi;
  const DqMat &m = p.mat[mi];
  double_quant_group(m.absmax, m.nb, __ldg(m.mean), m.absmax_q, m.absmax_scale, g - m.group_begin,
                     threadIdx.x & 31);
}

// Second-level quantization of the block absmax, one warp per group of 256:
// m2 = max|c - mu|, s2 = m2 / 127, q2 = clamp(rint((c - mu) / s2), -128, 127).
static __global__ void __launch_bounds__(256) double_quant_kernel(const float *__restrict__ absmax,
                                                           int64_t nb,
                                                           const float *__restrict__ mean,
                                                           int8_t *__restrict__ absmax_q,
                                                           float *__restrict__ absmax_scale) {
  pdl_launch_then_wait();
  const int64_t g = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int64_t ng = (nb + Q4_DQ_GROUP - 1) / Q4_DQ_GROUP;
  if (g >= ng) return;
  double_quant_group(absmax, nb, __ldg(mean), absmax_q, absmax_scale, g, threadIdx.x & 31);
}

}  // namespace q4
