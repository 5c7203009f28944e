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
// per SM) has 2.5x headroom at M <= 8; what limits it is the load/store pipe
// (each decoded byte is one shared-memory lookup) and the instructions spent
// per weight.  So:
//   * a CTA takes units of 128 weight rows x 1024 k from a work counter
//     (balanced, self-resetting); its producer warp streams each 64-k stage
//     of packed bytes ([128 x 32 B]) and activations ([8 NT x 64], 128-byte
//     swizzle, rows >= M zero-filled) with TMA into a ring of stages;
//   * each of 8 compute warps owns 16 rows (the MMA rows; swap-AB) and reads
//     its bytes and the activations from shared memory without conflicts;
//   * a byte maps to a pair of fp16 codebook values through a 256-entry table
//     in shared memory (one copy per lane), the MMA runs on the unscaled
//     values and each block's fp32 partial is scaled once by its c~; the k
//     order inside a segment of min(B, 64) is permuted identically on both
//     operands so that a lane reads consecutive bytes;
//   * the unit's block scales come from a few vector loads of the int8
//     double-quant codes;
//   * split rows add fp32 partials into a workspace; the last warp of a
//     16-row group writes Y and zeroes its rows again.
// bf16 activations multiply the exact w^ = bf16(c~ * level) (the definition
// dequantizes to the compute dtype first), with a binary32 pair table.
#pragma once
#include <cuda.h>

#include "gemm.cuh"  // mbarrier / TMA wrappers
#include "q4_common.cuh"

namespace q4 {

constexpr int kGsWarps = 8;                 // compute warps (16 rows each)
constexpr int kGsThreads = (kGsWarps + 1) * 32;  // + the TMA producer warp
constexpr int kGsRows = 16 * kGsWarps;      // rows per unit (one CTA tile)
constexpr int kGsUnitK = 1024;
constexpr int kGsMaxGroup = 16;
constexpr int kGsWTile = kGsRows * 32;      // packed bytes per 64-k stage

struct alignas(64) GsMat {
  CUtensorMap tmW;  // packed [N, K/2] bytes, box {32, 128}
  CUtensorMap tmA;  // activations [M, K] 16-bit, box {64, 8 NT}, 128-byte swizzle
  const uint8_t *packed;
  const float *absmax;
  const int8_t *absmax_q;
  const float *absmax_scale;
  const float *absmax_mean;
  const uint16_t *A;
  void *Y;
  float *acc;      // split-K workspace [N][M] fp32 (n_splits > 1)
  unsigned *cnt;   // per 16-row arrival counters
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
  unsigned *work;   // [2]: next unit, finished producers (both left at 0)
  int *status;
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

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.b32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ float2 lds64f(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0,%1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr));
  return v;
}
// Table entry address for byte j of `word` (lane-private copies: entry e of
// lane l at e * stride + esize * l; `lb` = table base + esize * l).
template <int SHIFT>
__device__ __forceinline__ uint32_t lut_addr(uint32_t word, int j, uint32_t lb) {
  return (__byte_perm(word, 0u, 0x4440u | (uint32_t)j) << SHIFT) + lb;
}

// DA: activation dtype; NT: n8 tiles (M <= 8 NT); B: blocksize; S: stages.
template <int DA, int NT, int B, int S>
__global__ void __launch_bounds__(kGsThreads, 2) gemv_small_kernel(const __grid_constant__ GsParams p) {
  constexpr bool EXACT = (DA == Q4_BF16);
  constexpr int SEG = B < 64 ? B : 64;         // k per scale segment inside a stage
  constexpr int SEGS = 64 / SEG;               // segments per stage
  constexpr int STEPS = SEG / 16;              // MMA k-steps per segment
  constexpr int LB = SEG / 8;                  // packed bytes per lane per segment and row
  constexpr int UB = kGsUnitK / B;             // blocks per unit
  constexpr int QW = (UB + 3) / 4;             // words of int8 codes per row per unit
  constexpr int ATILE = 8 * NT * 128;          // activation tile bytes per stage
  constexpr int STAGE = kGsWTile + ATILE;
  constexpr int LUTB = EXACT ? 256 * 32 * 8 : 256 * 32 * 4;
  static_assert(STAGE % 1024 == 0, "stage alignment");

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t *sStage = smem;                                  // [S][act tile | weight tile]
  uint8_t *sLut = smem + S * STAGE;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sLut + LUTB);  // sfull[S], sempty[S]
  unsigned *sUnit = reinterpret_cast<unsigned *>(bars + 2 * S);  // [S] unit ring
  __shared__ int s_abort;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tig = lane & 3;
  const uint32_t bar0 = smem_u32(bars);
  auto sfull = [&](int s) { return bar0 + 8u * s; };
  auto sempty = [&](int s) { return bar0 + 8u * (S + s); };

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(sfull(s), 1);
      mbar_init(sempty(s), kGsWarps);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    s_abort = 0;
  }
  for (int i = tid; i < 256 * 32; i += kGsThreads) {
    const int b = i >> 5;
    if constexpr (EXACT) reinterpret_cast<float2 *>(sLut)[i] = make_float2(p.levels[b & 15], p.levels[b >> 4]);
    else reinterpret_cast<uint32_t *>(sLut)[i] = Dt<DA>::pack2(p.levels[b & 15], p.levels[b >> 4]);
  }
  __syncthreads();
  volatile int *abort = &s_abort;
  const int M = p.M;

  if (warp == kGsWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t gs = 0;
      bool sent = false;
      unsigned next = atomicAdd(p.work, 1u);
      for (uint32_t gu = 0;; ++gu) {
        const unsigned u = next;
        const bool last = u >= p.total_units;
        if (!last) next = atomicAdd(p.work, 1u);  // claimed now, used one unit later
        const int s0 = gs % S;
        if (!mbar_wait(sempty(s0), ((gs / S) & 1) ^ 1, p.status, abort)) break;
        sUnit[gu % S] = u;
        if (last) {
          mbar_arrive(sfull(s0));  // completes the phase without data: the end marker
          sent = true;
          break;
        }
        int mi = 0;
        while (mi + 1 < p.count && (int64_t)u >= p.mat[mi + 1].unit_begin) ++mi;
        const GsMat &mt = p.mat[mi];
        const int64_t local = (int64_t)u - mt.unit_begin;
        const int tile = (int)(local % mt.n_tiles), split = (int)(local / mt.n_tiles);
        const int k0 = split * kGsUnitK;
        const int nst = (min(kGsUnitK, mt.K - k0) + 63) / 64;
        bool ok = true;
        for (int t = 0; t < nst; ++t, ++gs) {
          const int s = gs % S;
          if (t > 0 && !mbar_wait(sempty(s), ((gs / S) & 1) ^ 1, p.status, abort)) { ok = false; break; }
          mbar_arrive_expect_tx(sfull(s), STAGE);
          uint8_t *st = sStage + s * STAGE;
          tma_load_2d(smem_u32(st), &mt.tmA, sfull(s), k0 + t * 64, 0);
          tma_load_2d(smem_u32(st + ATILE), &mt.tmW, sfull(s), (k0 + t * 64) / 2, tile * kGsRows);
        }
        if (!ok) break;
      }
      if (*abort) {
        // The compute warps may have left: let the copies still in flight land
        // before the CTA exits (stages before gs - S were released, so complete).
        for (uint32_t j = (gs > (uint32_t)S ? gs - S : 0u); j < gs; ++j) {
          if (sent && j % S == gs % S) continue;  // that slot's last phase was the end marker
          int dummy = 0;
          volatile int no_abort = 0;
          mbar_wait(sfull(j % S), (j / S) & 1, &dummy, &no_abort);
        }
      }
      // The producer that finishes last leaves both counters at 0 for the next launch.
      __threadfence();
      if (atomicAdd(p.work + 1, 1u) == gridDim.x - 1) {
        p.work[0] = 0u;
        p.work[1] = 0u;
        __threadfence();
      }
    }
    return;
  }

  // -------------------------------------------------------------- compute warps
  const uint32_t lb = smem_u32(sLut) + (EXACT ? 8u : 4u) * lane;
  uint32_t gs = 0;
  for (uint32_t gu = 0;; ++gu) {
    {
      const int s0 = gs % S;
      if (!mbar_wait_warp(sfull(s0), (gs / S) & 1, p.status, abort)) break;
    }
    const unsigned u = sUnit[gu % S];
    if (u >= p.total_units) break;
    int mi = 0;
#pragma unroll 1
    while (mi + 1 < p.count && (int64_t)u >= p.mat[mi + 1].unit_begin) ++mi;
    const GsMat &mt = p.mat[mi];
    const int64_t local = (int64_t)u - mt.unit_begin;
    const int tile = (int)(local % mt.n_tiles), split = (int)(local / mt.n_tiles);
    const int K = mt.K, N = mt.N;
    const int k0 = split * kGsUnitK;
    const int klen = min(kGsUnitK, K - k0);
    const int nst = (klen + 63) / 64;
    const int nbk = K / B;
    const int blk0 = k0 / B;
    const int nblk = (klen + B - 1) / B;
    const int r_base = tile * kGsRows + warp * 16;

    // ---- block scales of this lane's rows g, g+8 for the unit
    uint32_t q2w[2][QW];
    float s2a[2], s2b[2], mu = 0.0f;
    int bsplit[2];
    const bool dq = p.dq != 0;
    if (dq) mu = __ldg(mt.absmax_mean);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int row = min(r_base + h * 8 + g, N - 1);
      const int64_t bi0 = (int64_t)row * nbk + blk0;
      if (dq) {
        const int64_t g0 = bi0 >> 8;
        s2a[h] = __ldg(mt.absmax_scale + g0);
        s2b[h] = __ldg(mt.absmax_scale + ((bi0 + nblk - 1) >> 8));
        bsplit[h] = (int)(((g0 + 1) << 8) - bi0);
        if (((bi0 & 3) == 0) && nblk == UB) {
#pragma unroll
          for (int qw = 0; qw < QW; ++qw) q2w[h][qw] = __ldg(reinterpret_cast<const unsigned int *>(mt.absmax_q + bi0) + qw);
        } else {
#pragma unroll
          for (int qw = 0; qw < QW; ++qw) {
            uint32_t v = 0;
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (4 * qw + e < nblk) v |= (uint32_t)(uint8_t)__ldg(mt.absmax_q + bi0 + 4 * qw + e) << (8 * e);
            q2w[h][qw] = v;
          }
        }
      }
    }
    // Scales of the unit's blocks in order: the int8 codes are consumed from
    // the front of q2w (register moves only, no dynamic register indexing).
    int bi = 0;  // next block of the unit
    float sc0 = 0.0f, sc1 = 0.0f;
    auto next_scales = [&]() {
      float v[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (dq) {
          const int code = (int)(int8_t)(q2w[h][0] & 0xFFu);
          const float s2 = (bi < bsplit[h]) ? s2a[h] : s2b[h];
          v[h] = __fadd_rn(__fmul_rn((float)code, s2), mu);
          q2w[h][0] >>= 8;
          if ((bi & 3) == 3) {
#pragma unroll
            for (int qw = 0; qw + 1 < QW; ++qw) q2w[h][qw] = q2w[h][qw + 1];
          }
        } else {
          const int row = min(r_base + h * 8 + g, N - 1);
          v[h] = __ldg(mt.absmax + (int64_t)row * nbk + blk0 + bi);
        }
      }
      sc0 = v[0];
      sc1 = v[1];
      ++bi;
    };

    float acc[NT][4], part[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[nt][j] = part[nt][j] = 0.0f;

    bool ok = true;
#pragma unroll 1
    for (int t = 0; t < nst; ++t, ++gs) {
      const int s = gs % S;
      if (t > 0 && !mbar_wait_warp(sfull(s), (gs / S) & 1, p.status, abort)) { ok = false; break; }
      const uint32_t st = smem_u32(sStage + s * STAGE);
      // packed bytes of rows g and g+8 of this warp's tile (32 bytes per row)
      uint32_t wv[2][2 * SEGS];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t ra = st + ATILE + (warp * 16 + h * 8 + g) * 32;
        if constexpr (SEG == 64) {
          const uint2 v = lds64(ra + tig * 8);
          wv[h][0] = v.x;
          wv[h][1] = v.y;
        } else {
#pragma unroll
          for (int sg = 0; sg < SEGS; ++sg) wv[h][sg] = lds32(ra + sg * 16 + tig * 4);
        }
      }
      // activation rows nt*8 + g: halves [seg*SEG + tig*SEG/4, + SEG/4), 128-byte swizzle
      uint32_t av[NT][SEGS][SEG / 8];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int ar = nt * 8 + g;
        const uint32_t aa = st + ar * 128;
#pragma unroll
        for (int sg = 0; sg < SEGS; ++sg) {
          if constexpr (SEG == 64) {
            const uint4 x0 = lds128(aa + (((2 * tig) ^ (ar & 7)) << 4));
            const uint4 x1 = lds128(aa + (((2 * tig + 1) ^ (ar & 7)) << 4));
            av[nt][sg][0] = x0.x; av[nt][sg][1] = x0.y; av[nt][sg][2] = x0.z; av[nt][sg][3] = x0.w;
            av[nt][sg][4] = x1.x; av[nt][sg][5] = x1.y; av[nt][sg][6] = x1.z; av[nt][sg][7] = x1.w;
          } else {
            const uint4 x0 = lds128(aa + (((sg * 4 + tig) ^ (ar & 7)) << 4));
            av[nt][sg][0] = x0.x; av[nt][sg][1] = x0.y; av[nt][sg][2] = x0.z; av[nt][sg][3] = x0.w;
          }
        }
      }
#pragma unroll
      for (int sg = 0; sg < SEGS; ++sg) {
        const int kseg = t * 64 + sg * SEG;          // k offset of the segment in the unit
        if (kseg >= klen) break;
        if (kseg % B == 0) next_scales();
#pragma unroll
        for (int q = 0; q < STEPS; ++q) {
          // bytes 2q, 2q+1 of the lane's LB bytes of this segment
          const int b0 = (sg * LB + 2 * q), b1 = b0 + 1;
          const uint32_t w00 = wv[0][b0 >> 2], w10 = wv[1][b0 >> 2];
          uint32_t a0, a1, a2, a3;
          if constexpr (EXACT) {
            const float2 e0 = lds64f(lut_addr<8>(w00, b0 & 3, lb));
            const float2 e1 = lds64f(lut_addr<8>(w10, b0 & 3, lb));
            const float2 e2 = lds64f(lut_addr<8>(w00, b1 & 3, lb));
            const float2 e3 = lds64f(lut_addr<8>(w10, b1 & 3, lb));
            a0 = Dt<DA>::pack2(__fmul_rn(sc0, e0.x), __fmul_rn(sc0, e0.y));
            a1 = Dt<DA>::pack2(__fmul_rn(sc1, e1.x), __fmul_rn(sc1, e1.y));
            a2 = Dt<DA>::pack2(__fmul_rn(sc0, e2.x), __fmul_rn(sc0, e2.y));
            a3 = Dt<DA>::pack2(__fmul_rn(sc1, e3.x), __fmul_rn(sc1, e3.y));
          } else {
            a0 = lds32(lut_addr<7>(w00, b0 & 3, lb));
            a1 = lds32(lut_addr<7>(w10, b0 & 3, lb));
            a2 = lds32(lut_addr<7>(w00, b1 & 3, lb));
            a3 = lds32(lut_addr<7>(w10, b1 & 3, lb));
          }
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
            MmaS<DA>::run(EXACT ? acc[nt] : part[nt], a0, a1, a2, a3, av[nt][sg][2 * q], av[nt][sg][2 * q + 1]);
        }
        if (!EXACT && (((kseg + SEG) % B) == 0 || kseg + SEG >= klen)) {
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            acc[nt][0] = fmaf(sc0, part[nt][0], acc[nt][0]);
            acc[nt][1] = fmaf(sc0, part[nt][1], acc[nt][1]);
            acc[nt][2] = fmaf(sc1, part[nt][2], acc[nt][2]);
            acc[nt][3] = fmaf(sc1, part[nt][3], acc[nt][3]);
#pragma unroll
            for (int j = 0; j < 4; ++j) part[nt][j] = 0.0f;
          }
        }
      }
      // Release the stage only now: the MMAs above have consumed every value
      // loaded from it, so none of those shared-memory reads can still be in
      // flight when the producer's next copy overwrites the slot (an arrive
      // issued right after the loads may overtake them).
      __syncwarp();
      if (lane == 0) mbar_arrive(sempty(s));
    }
    if (!ok) break;

    // ---- D fragment: rows g / g+8, columns m = nt*8 + 2 tig + {0, 1}
    if (mt.n_splits == 1) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int row = r_base + (j >> 1) * 8 + g;
          const int m = nt * 8 + 2 * tig + (j & 1);
          if (m < M && row < N) gs_store(mt.Y, p.y_dtype, (int64_t)m * N + row, acc[nt][j]);
        }
    } else if (r_base < N) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int row = r_base + (j >> 1) * 8 + g;
          const int m = nt * 8 + 2 * tig + (j & 1);
          if (m < M && row < N) atomicAdd(mt.acc + (int64_t)row * M + m, acc[nt][j]);
        }
      __threadfence();
      const int sub = r_base / 16;  // 16-row counter index
      unsigned ticket = 0;
      if (lane == 0) ticket = atomicAdd(mt.cnt + sub, 1u);
      ticket = __shfl_sync(0xffffffffu, ticket, 0);
      if (ticket == (unsigned)(mt.n_splits - 1)) {
        __threadfence();
        const int rows = min(16, N - r_base);
        for (int idx = lane; idx < rows * M; idx += 32) {
          const int m = idx / rows, r = idx - m * rows;
          float *ap = mt.acc + (int64_t)(r_base + r) * M + m;
          const float v = __ldcg(ap);
          __stcg(ap, 0.0f);
          gs_store(mt.Y, p.y_dtype, (int64_t)m * N + r_base + r, v);
        }
        if (lane == 0) mt.cnt[sub] = 0u;
      }
    }
  }
}

}  // namespace q4
