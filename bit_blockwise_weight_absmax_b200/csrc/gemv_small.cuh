// gemv_small.cuh -- fused NF4 dequant-GEMV for decode batches 1 <= M <= 16
// (sm_100a), Y[M,N] = A[M,K] . W^[N,K]^T.
//
// What it computes: n4n.ai, "What is 4-bit quantization and why does it
// matter?", "Why it matters for deployment" (decode at batch < 32 reads every
// weight once per token and is memory bound) and learn.pranaymahendrakar.com,
// "Loading a model in 4-bit", "Where the accuracy goes" (weights dequantized
// to the compute dtype, then a 16-bit matmul); the dequantization is fused
// into the streaming of the packed weights.
//
// Design (B200, decode sizes): at M <= 16 the per-instruction cost of a
// tcgen05 MMA (128 x 16 x 16 takes ~44 cycles) would cap the kernel at about
// the HBM rate, while the warp-level mma.sync path (m16n8k16, ~0.44 per clock
// per SM) has 2.5x headroom at M <= 8; what limits it is the number of
// instructions spent per weight.  So:
//   * a warp owns R tiles of 16 weight rows (MMA rows; swap-AB) for a unit of
//     1024 k, taken from a work counter (balanced, self-resetting);
//   * the unit's block scales c~ are fetched once, as 4-byte vectors of the
//     int8 double-quant codes, and formed per block in registers;
//   * packed bytes stream with 8-byte non-allocating loads PF blocks ahead;
//   * a byte maps to a pair of fp16 codebook values through a 256-entry table
//     in shared memory (one copy per lane: conflict-free), the MMA runs on
//     the unscaled values and the fp32 partial of each block is scaled once;
//     the k order inside a block is permuted identically on both operands so
//     that each lane reads B/8 consecutive bytes of a block row;
//   * split rows add fp32 partials into a workspace; the last warp of a row
//     tile writes Y and zeroes its rows again.
// bf16 activations multiply the exact w^ = bf16(c~ * level) (the definition
// dequantizes to the compute dtype first), with a binary32 pair table.
#pragma once
#include "q4_common.cuh"

namespace q4 {

constexpr int kGsWarps = 8;
constexpr int kGsUnitK = 1024;
constexpr int kGsMaxGroup = 16;

struct GsMat {
  const uint8_t *packed;
  const float *absmax;
  const int8_t *absmax_q;
  const float *absmax_scale;
  const float *absmax_mean;
  const uint16_t *A;
  void *Y;
  float *acc;      // split-K workspace [N][M] fp32 (n_splits > 1)
  unsigned *cnt;   // per 16R-row tile arrival counters
  int64_t unit_begin;
  int32_t N, K;
  int32_t n_tiles, n_splits;
};

struct GsParams {
  GsMat mat[kGsMaxGroup];
  int32_t count;
  int32_t M;
  int32_t y_dtype;
  int32_t dq;
  int64_t total_units;
  unsigned *work;   // [2]: next unit, finished warps (both left at 0)
  float levels[16];
};

template <int DA> struct MmaS;
template <> struct MmaS<Q4_F16> {
  static __device__ __forceinline__ void run(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                             uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
};
template <> struct MmaS<Q4_BF16> {
  static __device__ __forceinline__ void run(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                             uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
};

__device__ __forceinline__ void gs_store(void *Y, int ydt, int64_t idx, float v) {
  if (ydt == Q4_F32) reinterpret_cast<float *>(Y)[idx] = v;
  else if (ydt == Q4_F16) reinterpret_cast<uint16_t *>(Y)[idx] = Dt<Q4_F16>::from_f(v);
  else reinterpret_cast<uint16_t *>(Y)[idx] = Dt<Q4_BF16>::from_f(v);
}

// Lane slice of one block row: B/8 bytes = NW words.
template <int B> struct GsRow {
  static constexpr int NW = B / 32;
  uint32_t w[NW];
  __device__ __forceinline__ void load(const uint8_t *p) {
    if constexpr (NW == 1) {
      w[0] = __ldg(reinterpret_cast<const unsigned int *>(p));
    } else if constexpr (NW == 2) {
      const uint2 v = ldg_stream_v2(p);
      w[0] = v.x;
      w[1] = v.y;
    } else {
#pragma unroll
      for (int i = 0; i < NW; i += 4) {
        const uint4 v = ldg_stream_v4(p + 4 * i);
        w[i] = v.x; w[i + 1] = v.y; w[i + 2] = v.z; w[i + 3] = v.w;
      }
    }
  }
};

// Shared-memory byte address of the table entry for byte j of `word`
// (lane-private copies: entry e of lane l at e * 128 + 4 l; `lb` = table base
// + 4 l): one byte extract and one shift-add.
__device__ __forceinline__ uint32_t lut_addr(uint32_t word, int j, uint32_t lb) {
  return (__byte_perm(word, 0u, 0x4440u | (uint32_t)j) << 7) + lb;
}
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ float2 lds64f(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0,%1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr));
  return v;
}

// DA: activation dtype; NT: n8 tiles (M <= 8NT); R: 16-row tiles per warp;
// B: blocksize; PF: prefetch distance in blocks.
template <int DA, int NT, int R, int B, int PF>
__global__ void __launch_bounds__(kGsWarps * 32, R == 1 ? 3 : 2) gemv_small_kernel(const __grid_constant__ GsParams p) {
  constexpr bool EXACT = (DA == Q4_BF16);
  constexpr int UB = kGsUnitK / B;     // blocks per unit
  constexpr int STEPS = B / 16;        // MMA k-steps per block
  constexpr int ROWS = 16 * R;         // rows per unit
  constexpr int QW = (UB + 3) / 4;     // words of int8 codes per row per unit
  extern __shared__ uint8_t s_lut_raw[];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tig = lane & 3;
  // byte -> (level(lo nibble), level(hi nibble)): an fp16 pair, or a float2
  for (int i = tid; i < 256 * 32; i += kGsWarps * 32) {
    const int b = i >> 5;
    if constexpr (EXACT) {
      reinterpret_cast<float2 *>(s_lut_raw)[i] = make_float2(p.levels[b & 15], p.levels[b >> 4]);
    } else {
      reinterpret_cast<uint32_t *>(s_lut_raw)[i] = Dt<DA>::pack2(p.levels[b & 15], p.levels[b >> 4]);
    }
  }
  __syncthreads();
  const uint32_t lb = (uint32_t)__cvta_generic_to_shared(s_lut_raw) + (EXACT ? 8u : 4u) * lane;
  const int M = p.M;

  while (true) {
    // ---- next unit from the work counter (warp-uniform)
    unsigned u = 0;
    if (lane == 0) u = atomicAdd(p.work, 1u);
    u = __shfl_sync(0xffffffffu, u, 0);
    if (u >= p.total_units) break;
    int mi = 0;
#pragma unroll 1
    while (mi + 1 < p.count && (int64_t)u >= p.mat[mi + 1].unit_begin) ++mi;
    const GsMat &mt = p.mat[mi];
    const int64_t local = (int64_t)u - mt.unit_begin;
    const int tile = (int)(local % mt.n_tiles);
    const int split = (int)(local / mt.n_tiles);
    const int K = mt.K, N = mt.N;
    const int nbk = K / B;
    const int blk0 = split * UB;
    const int nblk = min(UB, nbk - blk0);
    const int r_base = tile * ROWS;

    // ---- block scales of this lane's rows (g, g+8 of each row tile)
    uint32_t q2w[R][2][QW];
    float s2a[R][2], s2b[R][2], mu = 0.0f;
    int bsplit[R][2];  // first block (relative) whose second-level group is g1
    const bool dq = p.dq != 0;
    if (dq) mu = __ldg(mt.absmax_mean);
#pragma unroll
    for (int rt = 0; rt < R; ++rt)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int row = min(r_base + rt * 16 + h * 8 + g, N - 1);
        const int64_t bi0 = (int64_t)row * nbk + blk0;
        if (dq) {
          const int64_t g0 = bi0 >> 8;
          s2a[rt][h] = __ldg(mt.absmax_scale + g0);
          s2b[rt][h] = __ldg(mt.absmax_scale + ((bi0 + nblk - 1) >> 8));
          bsplit[rt][h] = (int)(((g0 + 1) << 8) - bi0);
          if (((bi0 & 3) == 0) && nblk == UB) {
#pragma unroll
            for (int qw = 0; qw < QW; ++qw)
              q2w[rt][h][qw] = __ldg(reinterpret_cast<const unsigned int *>(mt.absmax_q + bi0) + qw);
          } else {
#pragma unroll
            for (int qw = 0; qw < QW; ++qw) {
              uint32_t v = 0;
#pragma unroll
              for (int e = 0; e < 4; ++e)
                if (4 * qw + e < nblk) v |= (uint32_t)(uint8_t)__ldg(mt.absmax_q + bi0 + 4 * qw + e) << (8 * e);
              q2w[rt][h][qw] = v;
            }
          }
        }
      }
    auto scale_of = [&](int rt, int h, int i) -> float {  // block i of the unit
      if (dq) {
        const int code = (int)(int8_t)((q2w[rt][h][i >> 2] >> (8 * (i & 3))) & 0xFFu);
        const float s2 = (i < bsplit[rt][h]) ? s2a[rt][h] : s2b[rt][h];
        return __fadd_rn(__fmul_rn((float)code, s2), mu);
      }
      const int row = min(r_base + rt * 16 + h * 8 + g, N - 1);
      return __ldg(mt.absmax + (int64_t)row * nbk + blk0 + i);
    };

    // ---- packed weights, PF blocks ahead
    const uint8_t *wrow[R][2];
#pragma unroll
    for (int rt = 0; rt < R; ++rt)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int row = min(r_base + rt * 16 + h * 8 + g, N - 1);
        wrow[rt][h] = mt.packed + (int64_t)row * (K / 2) + (int64_t)blk0 * (B / 2) + tig * (B / 8);
      }
    GsRow<B> buf[PF][R][2];
#pragma unroll
    for (int i = 0; i < PF; ++i)
#pragma unroll
      for (int rt = 0; rt < R; ++rt)
#pragma unroll
        for (int h = 0; h < 2; ++h)
          if (i < nblk) buf[i][rt][h].load(wrow[rt][h] + i * (B / 2));

    // activations: lane (g, tig) feeds n = nt*8 + g, k = block + tig*B/4 + [0, B/4)
    const uint16_t *arow[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int m = min(nt * 8 + g, M - 1);
      arow[nt] = mt.A + (int64_t)m * K + (int64_t)blk0 * B + tig * (B / 4);
    }
    bool mact[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) mact[nt] = (nt * 8 + g) < M;

    float acc[R][NT][4];
#pragma unroll
    for (int rt = 0; rt < R; ++rt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[rt][nt][j] = 0.0f;

#pragma unroll
    for (int i = 0; i < UB; ++i) {
      if (i >= nblk) break;
      GsRow<B> cur[R][2];
#pragma unroll
      for (int rt = 0; rt < R; ++rt)
#pragma unroll
        for (int h = 0; h < 2; ++h) cur[rt][h] = buf[i % PF][rt][h];
      if (i + PF < nblk) {
#pragma unroll
        for (int rt = 0; rt < R; ++rt)
#pragma unroll
          for (int h = 0; h < 2; ++h) buf[i % PF][rt][h].load(wrow[rt][h] + (i + PF) * (B / 2));
      }
      // activation words of this block: B/8 per n8 tile (zero for m >= M)
      uint32_t act[NT][B / 8];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int v = 0; v < B / 32; ++v) {
          uint4 x = make_uint4(0, 0, 0, 0);
          if (mact[nt]) x = __ldg(reinterpret_cast<const uint4 *>(arow[nt] + i * B) + v);
          act[nt][4 * v] = x.x; act[nt][4 * v + 1] = x.y; act[nt][4 * v + 2] = x.z; act[nt][4 * v + 3] = x.w;
        }
      }
      float sc[R][2];
#pragma unroll
      for (int rt = 0; rt < R; ++rt)
#pragma unroll
        for (int h = 0; h < 2; ++h) sc[rt][h] = scale_of(rt, h, i);

      if constexpr (EXACT) {
#pragma unroll
        for (int s = 0; s < STEPS; ++s)
#pragma unroll
          for (int rt = 0; rt < R; ++rt) {
            uint32_t a[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int h = q & 1, byte = 2 * s + (q >> 1);
              const float2 e = lds64f((__byte_perm(cur[rt][h].w[byte >> 2], 0u, 0x4440u | (uint32_t)(byte & 3)) << 8) + lb);
              a[q] = Dt<DA>::pack2(__fmul_rn(sc[rt][h], e.x), __fmul_rn(sc[rt][h], e.y));
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
              MmaS<DA>::run(acc[rt][nt], a[0], a[1], a[2], a[3], act[nt][2 * s], act[nt][2 * s + 1]);
          }
      } else {
        float part[R][NT][4];
#pragma unroll
        for (int rt = 0; rt < R; ++rt)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 4; ++j) part[rt][nt][j] = 0.0f;
#pragma unroll
        for (int s = 0; s < STEPS; ++s)
#pragma unroll
          for (int rt = 0; rt < R; ++rt) {
            const int byte = 2 * s;
            const uint32_t w0 = cur[rt][0].w[byte >> 2], w1 = cur[rt][1].w[byte >> 2];
            const uint32_t a0 = lds32(lut_addr(w0, byte & 3, lb));
            const uint32_t a1 = lds32(lut_addr(w1, byte & 3, lb));
            const uint32_t a2 = lds32(lut_addr(w0, (byte & 3) + 1, lb));
            const uint32_t a3 = lds32(lut_addr(w1, (byte & 3) + 1, lb));
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
              MmaS<DA>::run(part[rt][nt], a0, a1, a2, a3, act[nt][2 * s], act[nt][2 * s + 1]);
          }
#pragma unroll
        for (int rt = 0; rt < R; ++rt)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            acc[rt][nt][0] = fmaf(sc[rt][0], part[rt][nt][0], acc[rt][nt][0]);
            acc[rt][nt][1] = fmaf(sc[rt][0], part[rt][nt][1], acc[rt][nt][1]);
            acc[rt][nt][2] = fmaf(sc[rt][1], part[rt][nt][2], acc[rt][nt][2]);
            acc[rt][nt][3] = fmaf(sc[rt][1], part[rt][nt][3], acc[rt][nt][3]);
          }
      }
    }

    // ---- D fragment: rows g / g+8, columns m = nt*8 + 2 tig + {0, 1}
    if (mt.n_splits == 1) {
#pragma unroll
      for (int rt = 0; rt < R; ++rt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int row = r_base + rt * 16 + (j >> 1) * 8 + g;
            const int m = nt * 8 + 2 * tig + (j & 1);
            if (m < M && row < N) gs_store(mt.Y, p.y_dtype, (int64_t)m * N + row, acc[rt][nt][j]);
          }
    } else {
#pragma unroll
      for (int rt = 0; rt < R; ++rt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int row = r_base + rt * 16 + (j >> 1) * 8 + g;
            const int m = nt * 8 + 2 * tig + (j & 1);
            if (m < M && row < N) atomicAdd(mt.acc + (int64_t)row * M + m, acc[rt][nt][j]);
          }
      __threadfence();
      unsigned ticket = 0;
      if (lane == 0) ticket = atomicAdd(mt.cnt + tile, 1u);
      ticket = __shfl_sync(0xffffffffu, ticket, 0);
      if (ticket == (unsigned)(mt.n_splits - 1)) {
        __threadfence();
        const int rows = min(ROWS, N - r_base);
        for (int idx = lane; idx < rows * M; idx += 32) {
          const int m = idx / rows, r = idx - m * rows;
          float *ap = mt.acc + (int64_t)(r_base + r) * M + m;
          const float v = __ldcg(ap);
          __stcg(ap, 0.0f);
          gs_store(mt.Y, p.y_dtype, (int64_t)m * N + r_base + r, v);
        }
        if (lane == 0) mt.cnt[tile] = 0u;
      }
    }
  }

  // ---- leave the work counter at zero for the next launch: the last warp
  // to run out of work resets it
  if (lane == 0) {
    __threadfence();
    const unsigned done = atomicAdd(p.work + 1, 1u);
    if (done == gridDim.x * kGsWarps - 1) {
      p.work[0] = 0u;
      p.work[1] = 0u;
      __threadfence();
    }
  }
}

}  // namespace q4
