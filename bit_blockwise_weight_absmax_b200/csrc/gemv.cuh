// gemv.cuh -- fused NF4 dequant-GEMV for decode on tcgen05 (sm_100a):
// Y[M,N] = A[M,K] . W^[N,K]^T, 1 <= M <= 32.
//
// What it computes: n4n.ai, "What is 4-bit quantization and why does it
// matter?", "Why it matters for deployment" (decode at batch < 32 reads every
// weight once per token and is memory bound) and learn.pranaymahendrakar.com,
// "Loading a model in 4-bit", "Where the accuracy goes" (weights dequantized
// to the compute dtype, then a 16-bit matmul).  The dequantization is fused:
// the 16-bit weights never exist in HBM.
//
// Design (B200): a CTA owns a tile of 128 weight rows (TMEM lane = row) and
// walks work units of 1024 k.
//   warp 12 TMA producer: per 64-k stage the packed bytes of the 128 rows
//           ([128 x 32 B], 32-byte swizzle) and the activation tile
//           ([NB x 64] 16-bit, 128-byte swizzle, rows >= M zero-filled) into
//           a ring of shared-memory stages.
//   warps 0-7 decode: warps w and w+4 own TMEM lane quadrant w (32 rows),
//           each takes 16 of a row's 32 packed bytes, maps each byte to a
//           pair of 16-bit codebook values (256-entry table, one copy per
//           lane so lookups never conflict) and writes them straight into
//           tensor memory (tcgen05.st): the A operand.
//   warp 13 MMA issuer: tcgen05.mma kind::f16 with A from tensor memory
//           (M=128 rows, K=16) and the activation tile as B (N = NB = 16 or
//           32).  The k-steps of a quantization block go round-robin into CH
//           independent accumulators (4 at N=16, 2 at N=32): at these small
//           N an MMA is latency bound, and one dependent chain per block
//           would serialize them.
//   warps 8-11 accumulate (TMEM lane quadrants 0-3): read each block's CH
//           accumulator rows (tcgen05.ld), sum them, add that times the block scale
//           c~ into registers; at the end of a unit, store Y (or add it to a
//           split-K workspace; the last unit of a row tile writes Y and
//           zeroes the workspace rows again).
// Decode never waits for an MMA to finish except to reuse one of the four A
// buffers, and the accumulators run four blocks behind the MMAs.
// fp16 activations multiply the unscaled codebook (fp16 pairs) and apply c~
// per block in fp32; bf16 activations multiply the exact w^ = bf16(c~ *
// level) (binary32 table, scale applied before rounding), as the definition
// dequantizes to the compute dtype first.  Every mbarrier wait is bounded.
#pragma once
#include <cuda.h>

#include "gemm.cuh"  // PTX wrappers: mbarriers, TMA, tcgen05 fences, descriptors
#include "q4_common.cuh"

namespace q4 {

constexpr int kGvRows = 128;       // rows per tile = TMEM lanes
constexpr int kGvStageK = 64;      // k per pipeline stage
constexpr int kGvUnitK = 1024;     // k per work unit
constexpr int kGvThreads = 448;    // 8 decode + 4 accumulate warps, TMA warp, MMA warp
constexpr int kGvABuf = 4;         // decoded A tiles in TMEM (32 columns each)
constexpr int kGvDBuf = 2;         // accumulator sets in TMEM (64 columns each)
constexpr int kGvTmemCols = 256;
constexpr int kGvDecWarps = 8;     // two per TMEM lane quadrant, each half of the k pairs
constexpr int kGvWTile = kGvRows * kGvStageK / 2;  // 4 KB packed bytes per stage
constexpr int kGvMaxGroup = 16;

struct alignas(64) GvMat {
  CUtensorMap tmW;  // packed [N, K/2] bytes, box {32, 128}, 32-byte swizzle
  CUtensorMap tmA;  // activations [M, K] 16-bit, box {64, NB}, 128-byte swizzle
  const int8_t *absmax_q;
  const float *absmax_scale;
  const float *absmax_mean;
  const float *absmax;
  void *Y;
  float *acc;      // split-K workspace [N][M] fp32 (n_splits > 1)
  unsigned *cnt;   // arrival counters [n_tiles]
  int64_t unit_begin;
  int32_t N, K;
  int32_t n_tiles, n_splits;
};

struct GvParams {
  GvMat mat[kGvMaxGroup];
  int32_t count;
  int32_t M;
  int32_t y_dtype;
  int32_t dq;
  int64_t total_units;
  int *status;
  float levels[16];
};

template <int NCOL>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, float (&v)[NCOL]);
template <> __device__ __forceinline__ void tmem_ld_cols<1>(uint32_t taddr, float (&v)[1]) {
  uint32_t r;
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r) : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
  v[0] = __uint_as_float(r);
}
template <> __device__ __forceinline__ void tmem_ld_cols<2>(uint32_t taddr, float (&v)[2]) {
  uint32_t r0, r1;
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
  v[0] = __uint_as_float(r0);
  v[1] = __uint_as_float(r1);
}
template <> __device__ __forceinline__ void tmem_ld_cols<4>(uint32_t taddr, float (&v)[4]) {
  uint32_t r[4];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 4; ++i) v[i] = __uint_as_float(r[i]);
}
template <> __device__ __forceinline__ void tmem_ld_cols<8>(uint32_t taddr, float (&v)[8]) {
  uint32_t r[8];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                 "=r"(r[7])
               : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}
template <> __device__ __forceinline__ void tmem_ld_cols<16>(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
template <> __device__ __forceinline__ void tmem_ld_cols<32>(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  tmem_ld32(taddr, r);
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// 32 consecutive 32-bit columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// 16 consecutive 32-bit columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void umma_f16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t db, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %4, 0; "
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p; }" ::"r"(tmem_d),
      "r"(tmem_a), "l"(db), "r"(idesc), "r"(accumulate)
      : "memory");
}

struct GvUnit {
  int mi, tile, split;
};
__device__ __forceinline__ GvUnit gv_unit(const GvParams &p, int64_t u) {
  int mi = 0;
  while (mi + 1 < p.count && u >= p.mat[mi + 1].unit_begin) ++mi;
  const int64_t local = u - p.mat[mi].unit_begin;
  const int nt = p.mat[mi].n_tiles;
  return GvUnit{mi, (int)(local % nt), (int)(local / nt)};
}

// Output store in the requested dtype.
__device__ __forceinline__ void gv_store(void *Y, int ydt, int64_t idx, float v) {
  if (ydt == Q4_F32) reinterpret_cast<float *>(Y)[idx] = v;
  else if (ydt == Q4_F16) reinterpret_cast<uint16_t *>(Y)[idx] = Dt<Q4_F16>::from_f(v);
  else reinterpret_cast<uint16_t *>(Y)[idx] = Dt<Q4_BF16>::from_f(v);
}

// DA: activation dtype; B: blocksize; MP: M rounded up to 1/2/4/8/16/32;
// NB: MMA N (16 or 32); S: pipeline stages.
template <int DA, int B, int MP, int NB, int S>
__global__ void __launch_bounds__(kGvThreads, MP >= 32 ? 1 : 2) gemv_tc_kernel(const __grid_constant__ GvParams p) {
  constexpr int ATILE = NB * kGvStageK * 2;            // activation bytes per stage
  constexpr int STAGE = ATILE + kGvWTile;              // multiple of 1024
  constexpr bool EXACT = (DA == Q4_BF16);              // scale before rounding
  constexpr int LUTB = EXACT ? 256 * 32 * 8 : 256 * 32 * 4;
  constexpr int UBLK = kGvUnitK / B;                   // blocks per unit
  constexpr int CH = NB == 16 ? 4 : 2;                 // independent accumulator chains
  static_assert(STAGE % 1024 == 0, "stage alignment");

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t *sStage = smem;                               // [S][act tile | weight tile]
  uint8_t *sLut = smem + S * STAGE;                     // [256][32] words (or float2)
  float *sScale = reinterpret_cast<float *>(sLut + LUTB);  // [2][128][UBLK + 1] block scales
  uint64_t *bars = reinterpret_cast<uint64_t *>(sScale + 2 * kGvRows * (UBLK + 1));
  // bars: sfull[S] (TMA landed), sempty[S] (weights read by the decode warps),
  // sdone[S] (the stage's MMAs completed: one commit per stage frees the TMA
  // slot and the A buffer), afull[4] (A buffer written), dfull/dempty[2]
  // (accumulator set complete / read; the issuer is never more than two sets
  // ahead, so their phases cannot wrap), cfull/cempty[2] (unit block scales
  // staged / consumed)
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t bar0 = smem_u32(bars);
  auto sfull = [&](int s) { return bar0 + 8u * s; };
  auto sempty = [&](int s) { return bar0 + 8u * (S + s); };
  auto sdone = [&](int s) { return bar0 + 8u * (2 * S + s); };
  auto afull = [&](int a) { return bar0 + 8u * (3 * S + a); };
  auto dempty = [&](int d) { return bar0 + 8u * (3 * S + 4 + d); };
  auto dfull = [&](int d) { return bar0 + 8u * (3 * S + 6 + d); };
  auto cfull = [&](int c) { return bar0 + 8u * (3 * S + 8 + c); };
  auto cempty = [&](int c) { return bar0 + 8u * (3 * S + 10 + c); };

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(sfull(s), 1);
      mbar_init(sempty(s), kGvDecWarps);
      mbar_init(sdone(s), 1);
    }
    for (int i = 0; i < 4; ++i) mbar_init(afull(i), kGvDecWarps);
    for (int i = 0; i < 2; ++i) {
      mbar_init(dempty(i), 4);
      mbar_init(dfull(i), 1);
      mbar_init(cfull(i), 4);
      mbar_init(cempty(i), 4);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    s_abort = 0;
  }
  if constexpr (EXACT) {
    float2 *lut = reinterpret_cast<float2 *>(sLut);
    for (int i = tid; i < 256 * 32; i += kGvThreads) {
      const int b = i >> 5;
      lut[i] = make_float2(p.levels[b & 15], p.levels[b >> 4]);
    }
  } else {
    uint32_t *lut = reinterpret_cast<uint32_t *>(sLut);
    for (int i = tid; i < 256 * 32; i += kGvThreads) {
      const int b = i >> 5;
      lut[i] = Dt<DA>::pack2(p.levels[b & 15], p.levels[b >> 4]);
    }
  }
  if (warp == 13) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                 "r"(kGvTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const uint32_t tA = tmem;                                   // A tiles: columns [0, 128)
  const uint32_t tD = tmem + kGvABuf * (kGvStageK / 2);       // accumulator sets: [128, 256)
  volatile int *abort = &s_abort;
  const int M = p.M;

  if (warp == 12) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t gs = 0;
      for (int64_t u = blockIdx.x; u < p.total_units && !*abort; u += gridDim.x) {
        const GvUnit w = gv_unit(p, u);
        const GvMat &m = p.mat[w.mi];
        const int k0 = w.split * kGvUnitK;
        const int nst = (min(kGvUnitK, m.K - k0) + kGvStageK - 1) / kGvStageK;
        bool ok = true;
        for (int t = 0; t < nst; ++t, ++gs) {
          const int s = gs % S;
          if (!mbar_wait(sempty(s), ((gs / S) & 1) ^ 1, p.status, abort) ||
              !mbar_wait(sdone(s), ((gs / S) & 1) ^ 1, p.status, abort)) { ok = false; break; }
          mbar_arrive_expect_tx(sfull(s), STAGE);
          uint8_t *st = sStage + s * STAGE;
          tma_load_2d(smem_u32(st), &m.tmA, sfull(s), k0 + t * kGvStageK, 0);
          tma_load_2d(smem_u32(st + ATILE), &m.tmW, sfull(s), (k0 + t * kGvStageK) / 2, w.tile * kGvRows);
        }
        if (!ok) break;
      }
      for (uint32_t j = (gs > (uint32_t)S ? gs - S : 0); j < gs; ++j) {
        int dummy = 0;
        volatile int no_abort = 0;
        mbar_wait(sfull(j % S), (j / S) & 1, &dummy, &no_abort);
      }
    }
  } else if (warp == 13) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_f16(DA == Q4_BF16 ? 1 : 0, kGvRows, NB);
      uint32_t gs = 0, gseg = 0;
      for (int64_t u = blockIdx.x; u < p.total_units && !*abort; u += gridDim.x) {
        const GvUnit w = gv_unit(p, u);
        const int klen = min(kGvUnitK, p.mat[w.mi].K - w.split * kGvUnitK);
        const int nst = (klen + kGvStageK - 1) / kGvStageK;
        bool ok = true;
        for (int t = 0; t < nst && ok; ++t, ++gs) {
          const int s = gs % S;
          const int a = gs % kGvABuf;
          if (!mbar_wait(sfull(s), (gs / S) & 1, p.status, abort) ||
              !mbar_wait(afull(a), (gs / kGvABuf) & 1, p.status, abort)) { ok = false; break; }
          tc_fence_after();
          const uint64_t db0 = umma_desc_sw128(smem_u32(sStage + s * STAGE));
          const uint32_t ta = tA + a * (kGvStageK / 2);
#pragma unroll
          for (int j = 0; j < kGvStageK / 16; ++j) {
            const int kk = t * kGvStageK + j * 16;   // k offset inside the unit
            if (kk >= klen) break;
            // accumulator set per quantization block (fp16), or per unit (bf16,
            // exact w^); inside a set k-step i goes to chain i % CH
            const int kin = EXACT ? kk : (kk % B);
            if (kin == 0) {
              if (!mbar_wait(dempty(gseg % 2), ((gseg / 2) & 1) ^ 1, p.status, abort)) { ok = false; break; }
              tc_fence_after();
            }
            const uint32_t td = tD + (gseg % 2) * (CH * NB) + ((kin / 16) % CH) * NB;
            umma_f16_ts(td, ta + j * 8, db0 + 2 * j /* +32 bytes */, idesc, (kin / 16) < CH ? 0u : 1u);
            if (EXACT ? (kk + 16 >= klen) : (((kk + 16) % B) == 0 || kk + 16 >= klen)) {
              umma_commit(dfull(gseg % 2));
              ++gseg;
            }
          }
          umma_commit(sdone(s));
        }
        if (!ok) break;
      }
      // the last commit must have arrived before the CTA may exit
      if (gs > 0) {
        int dummy = 0;
        volatile int no_abort = 0;
        mbar_wait(sdone((gs - 1) % S), ((gs - 1) / S) & 1, &dummy, &no_abort);
      }
    }
  } else if (warp < kGvDecWarps) {
    // ------------------------------------------------------------ decode (A producer)
    const int qd = warp & 3, half = warp >> 2;
    const int r = qd * 32 + lane;  // row within the tile = TMEM lane
    const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
    uint32_t gs = 0, gu = 0;
    for (int64_t u = blockIdx.x; u < p.total_units && !*abort; u += gridDim.x, ++gu) {
      const GvUnit w = gv_unit(p, u);
      const GvMat &m = p.mat[w.mi];
      const int k0 = w.split * kGvUnitK;
      const int klen = min(kGvUnitK, m.K - k0);
      const int nst = (klen + kGvStageK - 1) / kGvStageK;
      const int row = w.tile * kGvRows + r;
      const bool row_ok = row < m.N;
      const int nbk = m.K / B;
      const int blk0 = k0 / B;
      const int nblk = (klen + B - 1) / B;
      // stage this row's block scales c~ of the unit (double buffered across
      // units): contiguous bytes (or floats) per row, 4-byte loads if aligned
      const int cb = gu & 1;
      float *myScale = sScale + (cb * kGvRows + r) * (UBLK + 1);
      if (half == 0 && gu >= 2 && !mbar_wait_warp(cempty(cb), ((gu >> 1) & 1) ^ 1, p.status, abort)) break;
      if (half == 1) {
        // scales are staged by the other warp of this quadrant
      } else if (row_ok) {
        const int64_t bi0 = (int64_t)row * nbk + blk0;
        if (p.dq) {
          const float mu = __ldg(m.absmax_mean);
          const int g0 = (int)(bi0 >> 8), g1 = (int)((bi0 + nblk - 1) >> 8);
          const float s2a = __ldg(m.absmax_scale + g0), s2b = __ldg(m.absmax_scale + g1);
          const bool vec = ((bi0 & 3) == 0) && ((nblk & 3) == 0);
          for (int b = 0; b < nblk; b += 4) {
            int8_t q[4];
            if (vec) {
              const uint32_t wv = __ldg(reinterpret_cast<const unsigned int *>(m.absmax_q + bi0 + b));
              q[0] = (int8_t)(wv & 0xFF); q[1] = (int8_t)((wv >> 8) & 0xFF);
              q[2] = (int8_t)((wv >> 16) & 0xFF); q[3] = (int8_t)(wv >> 24);
            } else {
#pragma unroll
              for (int e = 0; e < 4; ++e) q[e] = (b + e < nblk) ? __ldg(m.absmax_q + bi0 + b + e) : (int8_t)0;
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              if (b + e < nblk) {
                const float s2 = (((bi0 + b + e) >> 8) == g0) ? s2a : s2b;
                myScale[b + e] = __fadd_rn(__fmul_rn((float)q[e], s2), mu);
              }
            }
          }
        } else {
          for (int b = 0; b < nblk; ++b) myScale[b] = __ldg(m.absmax + bi0 + b);
        }
      } else {
        for (int b = 0; b < nblk; ++b) myScale[b] = 0.0f;
      }
      __syncwarp();
      if (half == 0 && lane == 0) mbar_arrive(cfull(cb));
      bool ok = true;
      if (EXACT && half == 1 && !mbar_wait_warp(cfull(cb), (gu >> 1) & 1, p.status, abort)) break;
      for (int t = 0; t < nst; ++t, ++gs) {
        const int s = gs % S;
        const int a = gs % kGvABuf;
        if (!mbar_wait_warp(sfull(s), (gs / S) & 1, p.status, abort)) { ok = false; break; }
        // this row's 32 packed bytes, 32-byte swizzle: 16-byte chunk c sits at
        // c ^ ((r >> 2) & 1); this warp decodes chunk `half` (k pairs 16h..16h+15)
        const uint8_t *wt = sStage + s * STAGE + ATILE + r * 32;
        const uint4 c0 = *reinterpret_cast<const uint4 *>(wt + 16 * (half ^ ((r >> 2) & 1)));
        __syncwarp();
        if (lane == 0) mbar_arrive(sempty(s));
        const uint32_t words[4] = {c0.x, c0.y, c0.z, c0.w};
        // A buffer a was last read by the MMAs of stage gs - 4
        if (gs >= kGvABuf && !mbar_wait_warp(sdone((gs - kGvABuf) % S), ((gs - kGvABuf) / S) & 1, p.status, abort)) { ok = false; break; }
        uint32_t dec[16];
        if constexpr (EXACT) {
          const float2 *lut = reinterpret_cast<const float2 *>(sLut) + lane;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int blk = (k0 + t * kGvStageK + 32 * half + 2 * j) / B;
            const float sc = myScale[blk - blk0];
            const float2 e = lut[((words[j >> 2] >> (8 * (j & 3))) & 0xFFu) * 32];
            dec[j] = Dt<DA>::pack2(__fmul_rn(sc, e.x), __fmul_rn(sc, e.y));
          }
        } else {
          const uint32_t *lut = reinterpret_cast<const uint32_t *>(sLut) + lane;
#pragma unroll
          for (int j = 0; j < 16; ++j) dec[j] = lut[((words[j >> 2] >> (8 * (j & 3))) & 0xFFu) * 32];
        }
        tmem_st16(tA + a * (kGvStageK / 2) + 16 * half + lane_base, dec);
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(afull(a));
      }
      if (!ok) break;
    }
  } else if (warp < kGvDecWarps + 4) {
    // ------------------------------------------------------------ accumulate (D consumer)
    const int q = warp & 3;
    const int r = q * 32 + lane;  // row within the tile = TMEM lane
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    uint32_t gseg = 0, gu = 0;
    for (int64_t u = blockIdx.x; u < p.total_units && !*abort; u += gridDim.x, ++gu) {
      const GvUnit w = gv_unit(p, u);
      const GvMat &m = p.mat[w.mi];
      const int k0 = w.split * kGvUnitK;
      const int klen = min(kGvUnitK, m.K - k0);
      const int row = w.tile * kGvRows + r;
      const bool row_ok = row < m.N;
      const int cb = gu & 1;
      if (!mbar_wait_warp(cfull(cb), (gu >> 1) & 1, p.status, abort)) break;
      const float *myScale = sScale + (cb * kGvRows + r) * (UBLK + 1);
      const int nseg = EXACT ? 1 : (klen + B - 1) / B;
      float acc[MP];
#pragma unroll
      for (int i = 0; i < MP; ++i) acc[i] = 0.0f;
      bool ok = true;
      for (int sg = 0; sg < nseg; ++sg, ++gseg) {
        const uint32_t d = gseg % 2;
        if (!mbar_wait_warp(dfull(d), (gseg / 2) & 1, p.status, abort)) { ok = false; break; }
        tc_fence_after();
        // chains written for this set: min(CH, its k-steps), as the MMA issuer does
        const int set_len = EXACT ? klen : min(B, klen - sg * B);
        const int nch = min(CH, (set_len + 15) / 16);
        float v[MP];
        tmem_ld_cols<MP>(tD + d * (CH * NB) + lane_base, v);
#pragma unroll
        for (int c = 1; c < CH; ++c) {
          if (c >= nch) break;
          float w2[MP];
          tmem_ld_cols<MP>(tD + d * (CH * NB) + c * NB + lane_base, w2);
#pragma unroll
          for (int i = 0; i < MP; ++i) v[i] += w2[i];
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(dempty(d));
        if (EXACT) {
#pragma unroll
          for (int i = 0; i < MP; ++i) acc[i] += v[i];
        } else {
          const float sc = myScale[sg];
#pragma unroll
          for (int i = 0; i < MP; ++i) acc[i] = fmaf(sc, v[i], acc[i]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(cempty(cb));
      if (!ok) break;
      // ---- unit result: Y directly, or split-K through the workspace
      if (m.n_splits == 1) {
        if (row_ok)
#pragma unroll
          for (int i = 0; i < MP; ++i)
            if (i < M) gv_store(m.Y, p.y_dtype, (int64_t)i * m.N + row, acc[i]);
      } else {
        if (row_ok)
#pragma unroll
          for (int i = 0; i < MP; ++i)
            if (i < M) atomicAdd(m.acc + (int64_t)row * M + i, acc[i]);
        __threadfence();
        __syncwarp();
        unsigned ticket = 0;
        if (lane == 0) ticket = atomicAdd(m.cnt + w.tile, 1u);
        ticket = __shfl_sync(0xffffffffu, ticket, 0);
        // the last of the tile's 4 * n_splits warp arrivals writes the tile
        if (ticket == 4u * (unsigned)m.n_splits - 1u) {
          __threadfence();
          const int row0 = w.tile * kGvRows;
          const int rows = min(kGvRows, m.N - row0);
          for (int i = 0; i < M; ++i)
            for (int rr = lane; rr < rows; rr += 32) {
              float *ap = m.acc + (int64_t)(row0 + rr) * M + i;
              const float v = __ldcg(ap);
              __stcg(ap, 0.0f);
              gv_store(m.Y, p.y_dtype, (int64_t)i * m.N + row0 + rr, v);
            }
          if (lane == 0) m.cnt[w.tile] = 0u;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 13) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kGvTmemCols));
  }
}

}  // namespace q4
