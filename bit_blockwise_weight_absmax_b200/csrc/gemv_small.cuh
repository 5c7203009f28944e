// gemv_small.cuh -- fused 4-bit dequant-GEMV for decode batches (sm_100a),
// Y[M,N] = A[M,K] . W^[N,K]^T for 1 <= M <= 32 activation rows in one pass
// (one, two or four n8 column tiles).  NF4 states use the 16-level
// codebook and the block absmax c~; INT4 symmetric states the integers -8..7
// and the group scale; INT4 asymmetric states the integers 0..15, the group
// scale s and zero-point z (robotsatlas.com, "INT4", "How it works":
// w^ = (q - z) s).
//
// What it computes: n4n.ai, "What is 4-bit quantization and why does it
// matter?", "Why it matters for deployment" (decode at batch < 32 reads every
// weight once per token and is memory bound) and learn.pranaymahendrakar.com,
// "Loading a model in 4-bit", "Where the accuracy goes" (weights dequantized
// to the compute dtype, then a 16-bit matmul); the dequantization is fused
// into the streaming of the packed weights.
//
// Design (B200, decode sizes).  At M <= 16 a tcgen05 MMA (128 x 16 x 16
// takes ~44 cycles) would cap the kernel near the HBM rate, while the
// warp-level mma.sync path (m16n8k16) has ample headroom; what limits a
// decode GEMV on this part is the issue rate and the shared-memory pipe (one
// table lookup per packed byte).  So the kernel spends as few instructions
// per weight as it can:
//   * one CTA per SM; a producer warp streams 128-k stages of packed bytes
//     ([256 rows x 64 B], TMA) and of the M activation rows (two [M x 64]
//     halves, 128-byte swizzle) into a ring in shared memory;
//   * the work is the concatenation of every matrix's (256-row tile,
//     128-k stage) pairs, cut into equal contiguous ranges, one per CTA: no tail,
//     no work counter, and a CTA meets only a few tiles, so the split-K
//     reduction runs a few times per CTA;
//   * 16 compute warps own 16 rows each (the MMA rows; swap-AB) and read
//     their bytes and the activation rows from the ring without conflicts;
//     the two halves of a stage are independent chains (more work in flight
//     per warp, half the barrier traffic of 64-k stages); a warp holds the
//     activation fragments of one 64-k segment at a time, which keeps every
//     batch size within the 96 registers a thread gets with 17 warps;
//   * a byte maps to the pair of its two codebook values through a
//     256-entry table in shared memory (one copy per lane) placed at a
//     64 KB-aligned shared address, so a single PRMT forms the address
//     (byte 1 = the packed byte, the other bytes = table base + lane);
//   * the MMA runs on the unscaled fp16 levels and each block's fp32 partial
//     is scaled once by its absmax c~ (INT4 asymmetric: s (P - z S), with
//     P the partial over the codes q and S the activations' sum over the
//     segment, from one more MMA of an all-ones tile); the k order inside a segment of
//     min(B, 64) is permuted identically on both operands so that a lane
//     reads consecutive bytes;
//   * each warp computes the c~ of its rows for the next 16 blocks one unit
//     ahead (loads issued a whole unit before they are needed) into a small
//     buffer of its own;
//   * only a CTA's first and last tiles can be partial: their fp32 partial
//     rows go to two per-CTA slots with plain stores; after its last stage
//     each warp counts its contributions per 16-row group, and the one that
//     completes a group sums the slots of all contributors, in CTA order,
//     into Y and zeroes them (deterministic; nothing waits mid-stream).
// bf16 activations multiply the exact w^ = bf16(c~ * level) (the definition
// dequantizes to the compute dtype first; INT4 asymmetric bf16(s (q - z))),
// with a binary32 pair table.
#pragma once
#include <cuda.h>

#include "gemm.cuh"  // mbarrier / TMA wrappers
#include "q4_common.cuh"

namespace q4 {

constexpr int kGsRows = 256;                      // rows per tile (16 per MMA row group)
constexpr int kGsMaxCtas = 256;                   // grid bound (split-K slots are per CTA)
constexpr int kGsStageK = 128;                    // k per stage (two 64-k halves)
constexpr int kGsWTile = kGsRows * kGsStageK / 2; // packed bytes per stage
constexpr int kGsMaxGroup = 16;
constexpr int kGsMaxStages = 16;
constexpr int kGsWinBlocks = 16;                  // blocks per scale window
constexpr int kGsScaleBuf = kGsWinBlocks * 16 * 4;        // c~ of one 16-row group's unit
constexpr int kGsScaleBytes = (kGsRows / 16) * 2 * kGsScaleBuf;  // two per row group
constexpr int kGsBarBytes = 2 * kGsMaxStages * 8 + 16;  // barriers + abort flag
constexpr int kGsInfoBytes = 16 * 80;             // per-matrix fields, copied to shared memory
constexpr int kGsZeroBytes = (kGsRows / 16) * 2 * kGsWinBlocks * 16;  // zero-points of a window, per row group and parity
constexpr int kGsSmemBytes = 227 * 1024;          // dynamic shared memory of a CTA

struct alignas(64) GsMat {
  CUtensorMap tmW;  // packed [N, K/2] bytes, box {32, 256}
  CUtensorMap tmA;  // activations [M, K] 16-bit, box {64, M}, 128-byte swizzle
  const float *absmax;
  const int8_t *absmax_q;
  const float *absmax_scale;
  const float *absmax_mean;
  const uint8_t *zero;  // INT4 asymmetric zero-points, two per byte
  void *Y;
  unsigned *cnt;    // per 16-row group: stages counted so far (zero between calls)
  uint32_t stage_begin;  // first global stage index of this matrix
  int32_t N, K;
  int32_t n_tiles, n_stages;  // 256-row tiles; 128-k stages per tile
};

// The fields the kernel reads per unit, copied once into shared memory (a
// dynamic index into the parameter block would miss the constant cache).
struct alignas(16) GsInfo {
  uint32_t stage_begin;
  int32_t N, K, n_stages;
  const float *absmax;
  const int8_t *absmax_q;
  const float *absmax_scale;
  const float *absmax_mean;
  const uint8_t *zero;
  void *Y;
  unsigned *cnt;
};
static_assert(sizeof(GsInfo) == 80, "GsInfo layout");

struct GsParams {
  GsMat mat[kGsMaxGroup];
  int32_t count;
  int32_t M;
  int32_t y_dtype;
  int32_t dq;
  uint32_t total_stages;  // below 2^32 / kGsMaxCtas, so c * T fits 32 bits
  float *slots;     // [grid][2][256 rows][8 NT] fp32 partial rows of each CTA's first / last tile
  int *status;
  uint64_t wait_ns;  // bound of every mbarrier wait
  int32_t stall_copies;  // test hook: issue no copies, so every stage wait runs out
  int32_t scale_f16;     // INT4: binary16 scales
  float levels[16];
};

// CTA c covers global stages [c T / G, (c+1) T / G); the CTA holding stage x.
__device__ __forceinline__ uint32_t gs_range_begin(uint32_t c, uint32_t T, uint32_t G) { return c * T / G; }
__device__ __forceinline__ int gs_cta_of(uint32_t x, uint32_t T, uint32_t G) {
  uint32_t c = x * G / T;
  while (c + 1 < G && gs_range_begin(c + 1, T, G) <= x) ++c;
  while (c > 0 && gs_range_begin(c, T, G) > x) --c;
  return (int)c;
}

template <int DA> struct MmaS;
template <> struct MmaS<Q4_F16> {
  static __device__ __forceinline__ void run(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                             uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
  // d = A . B (the accumulator starts at zero)
  static __device__ __forceinline__ void run0(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                              uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%10,%10,%10,%10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
  }
};
template <> struct MmaS<Q4_BF16> {
  static __device__ __forceinline__ void run(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                             uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
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

// Loads from the ring and the c~ buffer (ordered after the barrier waits:
// volatile).
__device__ __forceinline__ uint32_t lds32v(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint2 lds64v(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.b32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint4 lds128v(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ float2 lds64fv(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0,%1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr));
  return v;
}
// Table lookups: the table is constant after the start-up barrier and the
// address depends on ring data, so these need no ordering of their own.
__device__ __forceinline__ uint32_t lut32(uint32_t addr) {
  uint32_t v;
  asm("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ float2 lut64f(uint32_t addr) {
  float2 v;
  asm("ld.shared.v2.f32 {%0,%1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint32_t lds16v(uint32_t addr) {
  uint16_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ void sts8(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.u8 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void sts32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void sts64(uint32_t addr, uint32_t a, uint32_t b) {
  asm volatile("st.shared.v2.b32 [%0], {%1,%2};" ::"r"(addr), "r"(a), "r"(b) : "memory");
}
__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }

// Prefetch of one box of a tensor into L2 (no shared memory, no barrier).
// L2 is where the GPU's memory is coherent, so a box prefetched while an
// earlier kernel may still write it is read correctly by the copy that
// follows the dependency wait.
__device__ __forceinline__ void tma_prefetch_l2_2d(const CUtensorMap *map, int x, int y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(map), "r"(x), "r"(y)
               : "memory");
}

// Address of the table entry of byte j of `word`: byte 1 of the address is
// the packed byte; bytes 0, 2, 3 come from `lb` (table base + lane offset,
// whose byte 1 is zero because the table is 64 KB aligned).
__device__ __forceinline__ uint32_t lut_addr(uint32_t word, int j, uint32_t lb) {
  return __byte_perm(word, lb, 0x7604u | ((uint32_t)j << 4));
}

// One unit: the stages of one tile inside one window of 16 blocks, clipped
// to the CTA's range.  A pure function of the global stage index, so the
// producer and every compute warp walk the same sequence without talking.
struct GsUnit {
  int mi, tile, q0, q1;
  bool first, last;  // first / last unit of this CTA on the tile
};
template <int B>
__device__ __forceinline__ GsUnit gs_describe(const GsInfo *info, int count, int &mi, uint32_t g, uint32_t g0,
                                             uint32_t g1) {
  constexpr int W = kGsWinBlocks * B / kGsStageK;  // stages per window of 16 blocks
#pragma unroll 1
  while (mi + 1 < count && g >= info[mi + 1].stage_begin) ++mi;
  const GsInfo &mt = info[mi];
  const int local = (int)(g - mt.stage_begin);
  GsUnit u;
  u.mi = mi;
  u.tile = local / mt.n_stages;
  u.q0 = local - u.tile * mt.n_stages;
  int q1 = min((u.q0 / W + 1) * W, mt.n_stages);
  q1 = min(q1, u.q0 + (int)(g1 - g));
  u.q1 = q1;
  u.first = (u.q0 == 0) || (g == g0);
  u.last = (q1 == mt.n_stages) || (g + (q1 - u.q0) == g1);
  return u;
}

// The unit after `c`, which ended at global stage g: the same tile's next
// window, else the next tile of the matrix, else the next matrix (the same
// sequence gs_describe gives, without its division).
template <int B>
__device__ __forceinline__ GsUnit gs_next(const GsInfo *info, int count, const GsUnit &c, uint32_t g, uint32_t g0,
                                         uint32_t g1) {
  constexpr int W = kGsWinBlocks * B / kGsStageK;
  GsUnit u;
  u.mi = c.mi;
  u.tile = c.tile;
  u.q0 = c.q1;
  if (c.q1 == info[c.mi].n_stages) {
    u.q0 = 0;
    u.tile = c.tile + 1;
#pragma unroll 1
    while (u.mi + 1 < count && g >= info[u.mi + 1].stage_begin) {
      ++u.mi;
      u.tile = 0;
    }
  }
  const int ns = info[u.mi].n_stages;
  int q1 = min((u.q0 / W + 1) * W, ns);
  q1 = min(q1, u.q0 + (int)(g1 - g));
  u.q1 = q1;
  u.first = (u.q0 == 0) || (g == g0);
  u.last = (q1 == ns) || (g + (q1 - u.q0) == g1);
  return u;
}

// Inputs of the c~ of 8 blocks of one row (lane: row r0 + (lane & 15),
// blocks (lane >> 4) * 8 + j of the window), loaded one unit ahead.
struct GsScaleIn {
  uint32_t c0, c1;   // int8 codes (double quant)
  float s2a, s2b, mu;
  int bsplit, nvalid;
  float f[8];        // fp32 absmax (no double quant)
  uint32_t zw;       // INT4 asymmetric: zero-points of the 8 blocks, block j in bits 4j..4j+3
};

template <int B, bool AZ>
__device__ __forceinline__ void gs_scale_load(const GsInfo *info, bool dq, bool sf16, const GsUnit &u, int r0, int lane,
                                              GsScaleIn &in) {
  constexpr int W = kGsWinBlocks * B / kGsStageK;
  const GsInfo &mt = info[u.mi];
  const int row = u.tile * kGsRows + r0 + (lane & 15);
  const int nbk = mt.K / B;
  const int b0 = (u.q0 / W) * kGsWinBlocks + (lane >> 4) * 8;  // first block of the lane
  in.nvalid = (row < mt.N) ? max(0, min(8, nbk - b0)) : 0;
  in.c0 = in.c1 = 0;
  in.s2a = in.s2b = in.mu = 0.0f;
  in.bsplit = 8;
  in.zw = 0u;
#pragma unroll
  for (int j = 0; j < 8; ++j) in.f[j] = 0.0f;
  if (in.nvalid == 0) return;
  const int64_t bi0 = (int64_t)row * nbk + b0;
  if constexpr (AZ) {
    const uint8_t *zp = mt.zero + (bi0 >> 1);
    if (in.nvalid == 8 && (bi0 & 1) == 0 && ((uintptr_t)zp & 3) == 0) {
      in.zw = __ldg(reinterpret_cast<const unsigned *>(zp));  // blocks bi0 .. bi0 + 7, low nibble first
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j < in.nvalid)
          in.zw |= (uint32_t)((__ldg(mt.zero + ((bi0 + j) >> 1)) >> (((bi0 + j) & 1) * 4)) & 15) << (4 * j);
    }
  }
  if (dq) {
    in.mu = __ldg(mt.absmax_mean);
    const int64_t g0 = bi0 >> 8;
    in.s2a = __ldg(mt.absmax_scale + g0);
    in.s2b = __ldg(mt.absmax_scale + ((bi0 + in.nvalid - 1) >> 8));
    in.bsplit = (int)min((int64_t)8, ((g0 + 1) << 8) - bi0);
    if (in.nvalid == 8 && (bi0 & 3) == 0) {
      const unsigned *q = reinterpret_cast<const unsigned *>(mt.absmax_q + bi0);
      in.c0 = __ldg(q);
      in.c1 = __ldg(q + 1);
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t b = (j < in.nvalid) ? (uint32_t)(uint8_t)__ldg(mt.absmax_q + bi0 + j) : 0u;
        if (j < 4) in.c0 |= b << (8 * j);
        else in.c1 |= b << (8 * (j - 4));
      }
    }
  } else {
    if (in.nvalid == 8) {
      ld_scales8(mt.absmax, bi0, sf16, in.f);
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j < in.nvalid) in.f[j] = ld_scale(mt.absmax, bi0 + j, sf16);
    }
  }
}

// c~ = q2 * s2 + mu (two roundings, as dequantized), 0 for blocks past the
// row end, for block blk0 + j (j = 0..7) of row r of the warp's 16.
__device__ __forceinline__ float gs_scale_value(const GsScaleIn &in, bool dq, int j) {
  if (!dq) return in.f[j];
  const uint32_t w = j < 4 ? in.c0 : in.c1;
  const int code = (int)(int8_t)((w >> (8 * (j & 3))) & 0xFFu);
  const float v = __fadd_rn(__fmul_rn((float)code, j < in.bsplit ? in.s2a : in.s2b), in.mu);
  return j < in.nvalid ? v : 0.0f;
}

// Compute warps and threads of the kernel for R row groups per warp.
template <int R> struct GsShape {
  static constexpr int kWarps = kGsRows / (16 * R);
  static constexpr int kThreads = (kWarps + 1) * 32;  // + the TMA producer warp
};

// DA: activation dtype; NT: n8 tiles (M <= 8 NT); B: blocksize; R: 16-row
// groups per compute warp; AZ: INT4 asymmetric (codes 0..15 with a
// zero-point per block).
template <int DA, int NT, int B, int R, bool AZ>
__global__ void __launch_bounds__(GsShape<R>::kThreads, 1) gemv_small_kernel(const __grid_constant__ GsParams p) {
  // set-up (barriers, matrix fields, table, tensor-map prefetch) overlaps
  // the previous kernel; each warp waits for it before touching global memory
  pdl_launch_dependents();
  constexpr int WARPS = GsShape<R>::kWarps;
  constexpr int PRODUCER = WARPS;
  constexpr bool EXACT = (DA == Q4_BF16);
  constexpr int SEG = B < 64 ? B : 64;         // k per scale segment inside a stage
  constexpr int SEGS = kGsStageK / SEG;        // segments per stage
  constexpr int SPH = 64 / SEG;                // segments per 64-k half
  constexpr int STEPS = SEG / 16;              // MMA k-steps per segment
  constexpr int LB = SEG / 8;                  // packed bytes per lane per segment and row
  constexpr int WV = SEG == 64 ? 2 * SEGS : SEGS;  // packed words per lane and row per stage
  constexpr int MW = 8 * NT;                   // columns of the MMA tile (M <= MW)
  constexpr int ATILE = MW * 128;              // activation tile bytes per 64-k half
  constexpr int STAGE = 2 * ATILE + kGsWTile;
  constexpr uint32_t ES = EXACT ? 8u : 4u;     // table entry bytes per lane
  // fp16 tables use 128 of every 256 bytes: the c~ buffers live in the gaps
  constexpr int MISC = (EXACT ? kGsScaleBytes : 0) + kGsBarBytes + kGsInfoBytes + (AZ ? kGsZeroBytes : 0);
  static_assert(STAGE % 1024 == 0, "stage alignment");
  static_assert(EXACT || kGsScaleBytes == 256 * 128, "c~ buffers fill the table gaps");

  extern __shared__ __align__(1024) uint8_t smem_raw[];

  // ---- shared-memory layout (addresses in the shared window): the table at
  // the first 64 KB boundary; barriers, the abort flag, the matrix fields
  // (and the bf16 c~ buffers) in whichever free region holds them; the ring
  // in up to two runs of stages.
  const uint32_t base = smem_u32(smem_raw);
  const uint32_t end = base + kGsSmemBytes;
  const uint32_t lut = (base + 0xFFFFu) & ~0xFFFFu;
  uint32_t lo = base, hi = lut + 0x10000u;
  uint32_t misc;
  if (lut - lo >= (uint32_t)MISC) {
    misc = lo;
    lo += MISC;
  } else {
    misc = hi;
    hi += MISC;
  }
  const uint32_t ra = (lo + 1023u) & ~1023u, rb = (hi + 1023u) & ~1023u;
  int SA = ra < lut ? (int)((lut - ra) / STAGE) : 0;
  const int SB = rb < end ? (int)((end - rb) / STAGE) : 0;
  const int S = min(kGsMaxStages, SA + SB);
  SA = min(SA, S);
  const uint32_t rb_adj = rb - (uint32_t)SA * STAGE;  // stage s >= SA at rb_adj + s * STAGE
  if (S < 4 || hi > end) {  // not reachable with this launch's shared-memory size; refuse loudly
    if (threadIdx.x == 0) {
      pdl_wait();
      raise_status(p.status, Q4_STATUS_LAYOUT);
    }
    return;
  }
  auto stage_addr = [&](int s) { return (s < SA ? ra : rb_adj) + (uint32_t)s * STAGE; };
  const uint32_t scales = misc;  // bf16 only
  const uint32_t bar0 = misc + (EXACT ? kGsScaleBytes : 0);
  auto sfull = [&](int s) { return bar0 + 8u * s; };
  auto sempty = [&](int s) { return bar0 + 8u * (kGsMaxStages + s); };
  volatile int *abort = reinterpret_cast<volatile int *>(smem_raw + (bar0 + 16u * kGsMaxStages - base));
  GsInfo *info = reinterpret_cast<GsInfo *>(smem_raw + (bar0 + kGsBarBytes - base));
  // zero-points of a window (INT4 asymmetric), per row group and parity:
  // [block][row & 7][row >> 3] bytes, so rows g and g + 8 of a block are adjacent
  const uint32_t zbase = bar0 + kGsBarBytes + kGsInfoBytes;
  // c~ buffer of 16-row group grp (0..15), parity sb, byte offset o < 1024:
  // contiguous (bf16) or in the 128-byte gaps of the table (fp16)
  auto scale_addr = [&](int grp, uint32_t sb, uint32_t o) -> uint32_t {
    if constexpr (EXACT) return scales + ((uint32_t)grp * 2u + sb) * (uint32_t)kGsScaleBuf + o;
    else return lut + 128u + (((uint32_t)grp * 2u + sb) * 8u + (o >> 7)) * 256u + (o & 127u);
  };

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tig = lane & 3;
  const int M = p.M;
  const uint32_t T = p.total_stages, G = gridDim.x;
  const uint32_t g0 = gs_range_begin(blockIdx.x, T, G);  // this CTA's stages [g0, g1)
  const uint32_t g1 = gs_range_begin(blockIdx.x + 1, T, G);
  const bool dq = p.dq != 0;
  const bool sf16 = p.scale_f16 != 0;
  if (tid < p.count) {
    const GsMat &m = p.mat[tid];
    GsInfo &d = info[tid];
    d.stage_begin = m.stage_begin;
    d.N = m.N;
    d.K = m.K;
    d.n_stages = m.n_stages;
    d.absmax = m.absmax;
    d.absmax_q = m.absmax_q;
    d.absmax_scale = m.absmax_scale;
    d.absmax_mean = m.absmax_mean;
    d.zero = m.zero;
    d.Y = m.Y;
    d.cnt = m.cnt;
  }
  if (warp == PRODUCER && lane == 0) {
    for (int b = 0; b < S; ++b) {
      mbar_init(sfull(b), 1);
      mbar_init(sempty(b), WARPS);  // one arrival per compute warp
    }
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();  // barriers and matrix fields ready

  if (warp == PRODUCER) {
    // ------------------------------------------------------------ producer
    if (lane < p.count) {
      prefetch_tensormap(&p.mat[lane].tmW);
      prefetch_tensormap(&p.mat[lane].tmA);
    }
    if (lane == 0) {
      // The weight boxes of the first ring's worth of stages into L2 before
      // the wait, so that their DRAM latency overlaps the previous kernel's
      // last CTAs (a prefetch consumes nothing: the copies below still come
      // after the wait).
      {
        int pmi = 0, n = 0;
        GsUnit v;
        if (g0 < g1) v = gs_describe<B>(info, p.count, pmi, g0, g0, g1);
        for (uint32_t gi = g0; gi < g1 && n < S;) {
          if (gi != g0) v = gs_next<B>(info, p.count, v, gi, g0, g1);
          for (int q = v.q0; q < v.q1 && n < S; ++q, ++n)
            tma_prefetch_l2_2d(&p.mat[v.mi].tmW, q * (kGsStageK / 2), v.tile * kGsRows);
          gi += (uint32_t)(v.q1 - v.q0);
        }
      }
      pdl_wait();
      const uint32_t tx = (uint32_t)kGsWTile + 2u * 128u * (uint32_t)M;
      int s = 0, mi = 0, issued = 0;
      uint32_t ph = 0;
      bool ok = true;
      GsUnit u;
      if (g0 < g1) u = gs_describe<B>(info, p.count, mi, g0, g0, g1);
      for (uint32_t gi = g0; gi < g1 && ok;) {
        if (gi != g0) u = gs_next<B>(info, p.count, u, gi, g0, g1);
        const GsMat &mt = p.mat[u.mi];
        for (int q = u.q0; q < u.q1; ++q) {
          if (!mbar_wait(sempty(s), ph ^ 1u, p.status, abort, p.wait_ns)) { ok = false; break; }
          // the compute warps' reads of this slot (generic proxy) come before
          // the copy that overwrites it (async proxy)
          if (p.stall_copies) continue;
          fence_proxy_async_smem();
          mbar_arrive_expect_tx(sfull(s), tx);
          const uint32_t st = stage_addr(s);
          tma_load_2d(st, &mt.tmA, sfull(s), q * kGsStageK, 0);
          tma_load_2d(st + ATILE, &mt.tmA, sfull(s), q * kGsStageK + 64, 0);
          tma_load_2d(st + 2 * ATILE, &mt.tmW, sfull(s), q * (kGsStageK / 2), u.tile * kGsRows);
          ++issued;
          if (++s == S) { s = 0; ph ^= 1u; }
        }
        gi += (uint32_t)(u.q1 - u.q0);
      }
      if (*abort) {
        // The compute warps may have left: let the copies still in flight
        // land before the CTA exits (older stages were released, so complete).
        int ss = s;
        uint32_t pp = ph;
        for (int j = 0; j < min(issued, S); ++j) {
          if (--ss < 0) { ss = S - 1; pp ^= 1u; }
          int dummy = 0;
          volatile int no_abort = 0;
          mbar_wait(sfull(ss), pp, &dummy, &no_abort);
        }
      }
    }
    return;
  }

  // -------------------------------------------------------------- compute warps
  // the table (launch parameters only) first, then the first unit's c~
  // inputs once the previous kernel has finished
  for (int i = tid; i < 256 * 32; i += WARPS * 32) {
    const int b = i >> 5, l = i & 31;
    const uint32_t a = lut + (uint32_t)b * 256u + (uint32_t)l * ES;
    if constexpr (EXACT) sts64(a, __float_as_uint(p.levels[b & 15]), __float_as_uint(p.levels[b >> 4]));
    else sts32(a, Dt<DA>::pack2(p.levels[b & 15], p.levels[b >> 4]));
  }
  // the table is complete for every compute warp (the producer does not wait)
  asm volatile("bar.sync 1, %0;" ::"n"(WARPS * 32) : "memory");
  pdl_wait();
  int mi = 0;
  GsScaleIn sin[R];
  GsUnit u;
  if (g0 < g1) {
    u = gs_describe<B>(info, p.count, mi, g0, g0, g1);
#pragma unroll
    for (int rt = 0; rt < R; ++rt) gs_scale_load<B, AZ>(info, dq, sf16, u, (warp * R + rt) * 16, lane, sin[rt]);
  }

  const uint32_t lb = lut + ES * (uint32_t)lane;
  uint32_t sb = 0;  // c~ buffer parity
  // partial tiles: the one holding this CTA's first stage is counted when
  // done (done0: its row groups this warp completed, summed at the end); the
  // one holding its last stage is counted at the end
  int pend_mi0 = -1, pend_tile0 = 0;
  uint32_t done0 = 0u;
  int pend_mi1 = -1, pend_tile1 = 0, pend_len1 = 0;
  float acc[R][NT][4];
  int qstart = 0;
  uint32_t av[NT][SEG / 8];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int i = 0; i < SEG / 8; ++i) av[nt][i] = 0u;
  int s = 0;
  uint32_t ph = 0;

  // c~ buffer addresses at parity 0 (parity 1 at + kSbStride): where this
  // lane writes block (lane >> 4) * 8 of its row lane & 15 (block j further at
  // + joff(j)), and where it reads the (row g, row g + 8) pair of block 0
  constexpr uint32_t kSbStride = EXACT ? (uint32_t)kGsScaleBuf : 8u * 256u;
  auto joff = [](int j) -> uint32_t {
    return EXACT ? (uint32_t)j * 64u : (uint32_t)(j >> 1) * 256u + (uint32_t)(j & 1) * 64u;
  };
  uint32_t cst[R], srd0[R], zst[R], zrd0[R];
#pragma unroll
  for (int rt = 0; rt < R; ++rt) {
    const int r = lane & 15, blk0 = (lane >> 4) * 8;
    cst[rt] = scale_addr(warp * R + rt, 0u, (uint32_t)((blk0 * 8 + (r & 7)) * 2 + (r >> 3)) * 4u);
    srd0[rt] = scale_addr(warp * R + rt, 0u, (uint32_t)g * 8u);
    // zero-points: this lane writes block blk0 + j of row r at + 16 j, reads
    // the (row g, row g + 8) byte pair of block bw at + 16 bw
    zst[rt] = zbase + (uint32_t)(warp * R + rt) * 512u + (uint32_t)((blk0 * 8 + (r & 7)) * 2 + (r >> 3));
    zrd0[rt] = zbase + (uint32_t)(warp * R + rt) * 512u + (uint32_t)g * 2u;
  }

  // A partial tile's rows (this warp's 16-row groups) are counted, and the
  // warp that completes a group's count sums the slots of all contributors
  // in CTA order, writes Y and leaves slots and count zeroed.  A CTA counts
  // its first partial tile as soon as it is done (its partner, the CTA
  // before, finishes that tile only at its own end) and its last one at its
  // end; the sums run at the end, so the end of a launch counts one tile per
  // CTA.  count_piece returns the row groups this warp completed.
  auto count_piece = [&](int pmi, int tile, unsigned len) -> uint32_t {
    fence_acq_rel_gpu();  // this thread's slot stores are visible before its count
    __syncwarp();
    const GsInfo &mt = info[pmi];
    // lane 0 counts every row group of the warp at once (the atomics are in
    // flight together), then each one is checked for completion
    unsigned olds[R];
#pragma unroll
    for (int rt = 0; rt < R; ++rt) {
      olds[rt] = 0u;
      const int r_base = tile * kGsRows + warp * 16 * R + rt * 16;
      if (lane == 0 && r_base < mt.N) olds[rt] = atomicAdd(mt.cnt + (r_base >> 4), len);
    }
    uint32_t done = 0u;
#pragma unroll
    for (int rt = 0; rt < R; ++rt) {
      const int r_base = tile * kGsRows + warp * 16 * R + rt * 16;
      const unsigned old = __shfl_sync(0xffffffffu, olds[rt], 0);
      if (r_base < mt.N && old + len == (unsigned)mt.n_stages) done |= 1u << rt;
    }
    return done;
  };
  auto sum_piece = [&](int pmi, int tile, uint32_t done) {
    const GsInfo &mt = info[pmi];
    const int N = mt.N, Q = mt.n_stages;
    const uint32_t x0 = mt.stage_begin + (uint32_t)(tile * Q);  // the tile's first stage
#pragma unroll
    for (int rt = 0; rt < R; ++rt) {
      if (!(done & (1u << rt))) continue;
      const int r_base = tile * kGsRows + warp * 16 * R + rt * 16;
      // every contributor has counted: sum their slots in CTA order
      __syncwarp();
      fence_acq_rel_gpu();
      const int c0 = gs_cta_of(x0, T, G), c1 = gs_cta_of(x0 + Q - 1, T, G);
      float sum[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int j = 0; j < 4; ++j) sum[nt][j] = 0.0f;
      for (int cb = c0; cb <= c1; cb += 4) {
        // up to four contributors' rows in flight at once, added in CTA order
        float2 v[4][NT][2];
        float *slot[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int c = min(cb + k, c1);
          const int role = (gs_range_begin(c, T, G) >= x0) ? 0 : 1;  // c starts inside the tile
          slot[k] = p.slots + ((int64_t)(c * 2 + role) * kGsRows + warp * 16 * R + rt * 16 + g) * MW + 2 * tig;
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h)
              v[k][nt][h] = __ldcg(reinterpret_cast<const float2 *>(slot[k] + (h * 8) * MW + nt * 8));
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          if (cb + k > c1) break;
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              // the workspace is left zeroed
              __stcg(reinterpret_cast<float2 *>(slot[k] + (h * 8) * MW + nt * 8), make_float2(0.0f, 0.0f));
              sum[nt][2 * h] += v[k][nt][h].x;
              sum[nt][2 * h + 1] += v[k][nt][h].y;
            }
        }
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int row = r_base + (j >> 1) * 8 + g;
          const int m = nt * 8 + 2 * tig + (j & 1);
          if (m < M && row < N) gs_store(mt.Y, p.y_dtype, (int64_t)m * N + row, sum[nt][j]);
        }
      if (lane == 0) mt.cnt[r_base >> 4] = 0u;
    }
  };

  bool ok = true;
#pragma unroll 1
  for (uint32_t gi = g0; gi < g1;) {
    // c~ of this unit into the next buffers (rewritten a unit after their last read)
    {
      bool plain = dq;  // full windows inside one 256-group: no selects
#pragma unroll
      for (int rt = 0; rt < R; ++rt) plain = plain && sin[rt].nvalid == 8 && sin[rt].bsplit == 8;
      if (__all_sync(0xffffffffu, plain)) {
#pragma unroll
        for (int rt = 0; rt < R; ++rt)
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint32_t w = j < 4 ? sin[rt].c0 : sin[rt].c1;
            const float code = (float)(int)(int8_t)(uint8_t)(w >> (8 * (j & 3)));
            sts32(cst[rt] + sb * kSbStride + joff(j), __float_as_uint(__fadd_rn(__fmul_rn(code, sin[rt].s2a), sin[rt].mu)));
          }
      } else {
#pragma unroll
        for (int rt = 0; rt < R; ++rt)
#pragma unroll
          for (int j = 0; j < 8; ++j)
            sts32(cst[rt] + sb * kSbStride + joff(j), __float_as_uint(gs_scale_value(sin[rt], dq, j)));
      }
      if constexpr (AZ) {
#pragma unroll
        for (int rt = 0; rt < R; ++rt)
#pragma unroll
          for (int j = 0; j < 8; ++j) sts8(zst[rt] + sb * 256u + 16u * j, (sin[rt].zw >> (4 * j)) & 15u);
      }
    }
    __syncwarp();
    uint32_t srd[R], zrd[R];  // this lane's (row g, row g+8) pair of block 0, per row group
#pragma unroll
    for (int rt = 0; rt < R; ++rt) {
      srd[rt] = srd0[rt] + sb * kSbStride;
      zrd[rt] = zrd0[rt] + sb * 256u;
    }
    sb ^= 1u;
    const GsUnit cu = u;
    const uint32_t gn = gi + (uint32_t)(cu.q1 - cu.q0);
    if (gn < g1) {  // next unit: issue its c~ loads now, use them a unit later
      u = gs_next<B>(info, p.count, cu, gn, g0, g1);
#pragma unroll
      for (int rt = 0; rt < R; ++rt) gs_scale_load<B, AZ>(info, dq, sf16, u, (warp * R + rt) * 16, lane, sin[rt]);
    }
    const GsInfo &mt = info[cu.mi];
    const int K = mt.K, N = mt.N;
    if (cu.first) {
      qstart = cu.q0;
#pragma unroll
      for (int rt = 0; rt < R; ++rt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[rt][nt][j] = 0.0f;
    }
    const int w_base = cu.tile * kGsRows + warp * 16 * R;  // first row of this warp

#pragma unroll 1
    for (int q = cu.q0; q < cu.q1; ++q) {
      // lane 0 waits for the copy (acquire); the shuffle keeps the other
      // lanes' reads of the stage after it
      {
        bool ready = true;
        if (lane == 0) ready = mbar_wait(sfull(s), ph, p.status, abort, p.wait_ns);
        if (!__shfl_sync(0xffffffffu, ready ? 1 : 0, 0)) { ok = false; break; }
      }
      const uint32_t st = stage_addr(s);
      // packed bytes of rows g and g+8 of each row group (64 bytes per row);
      // segment sg of a row is bytes [sg * SEG / 2, + SEG / 2), a lane's
      // share of it the tig-th quarter
      uint32_t wv[R][2][WV];
#pragma unroll
      for (int rt = 0; rt < R; ++rt)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t ra_ = st + 2 * ATILE + (uint32_t)(warp * 16 * R + rt * 16 + h * 8 + g) * (kGsStageK / 2);
#pragma unroll
          for (int sg = 0; sg < SEGS; ++sg) {
            if constexpr (SEG == 64) {
              const uint2 v = lds64v(ra_ + sg * 32 + tig * 8);
              wv[rt][h][2 * sg] = v.x;
              wv[rt][h][2 * sg + 1] = v.y;
            } else {
              wv[rt][h][sg] = lds32v(ra_ + sg * 16 + tig * 4);
            }
          }
        }
#pragma unroll
      for (int sg = 0; sg < SEGS; ++sg) {
        if (q * kGsStageK + sg * SEG >= K) break;
        // this segment's activation rows nt*8 + g (< M only; the rest stay zero): 128-byte swizzle
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int ar = nt * 8 + g;
          if (ar < M) {
            const uint32_t aa = st + (uint32_t)(sg / SPH) * ATILE + (uint32_t)ar * 128u;
            const int sgh = sg % SPH;
            if constexpr (SEG == 64) {
              const uint4 x0 = lds128v(aa + (((2 * tig) ^ (ar & 7)) << 4));
              const uint4 x1 = lds128v(aa + (((2 * tig + 1) ^ (ar & 7)) << 4));
              av[nt][0] = x0.x; av[nt][1] = x0.y; av[nt][2] = x0.z; av[nt][3] = x0.w;
              av[nt][4] = x1.x; av[nt][5] = x1.y; av[nt][6] = x1.z; av[nt][7] = x1.w;
            } else {
              const uint4 x0 = lds128v(aa + (((sgh * 4 + tig) ^ (ar & 7)) << 4));
              av[nt][0] = x0.x; av[nt][1] = x0.y; av[nt][2] = x0.z; av[nt][3] = x0.w;
            }
          }
        }
        // block of this segment within the 16-block window
        const int bw = ((q * kGsStageK + sg * SEG) / B) & (kGsWinBlocks - 1);
        const uint32_t soff = EXACT ? (uint32_t)bw * 64u : (uint32_t)(bw >> 1) * 256u + (uint32_t)(bw & 1) * 64u;
        // INT4 asymmetric, binary16: the activations' sum over the segment,
        // S, in the accumulator layout (an all-ones A tile)
        float csum[NT][4];
        if constexpr (AZ && !EXACT) {
          constexpr uint32_t kOne = 0x3C003C00u;  // binary16 1.0, twice
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int qq = 0; qq < STEPS; ++qq) {
              if (qq == 0) MmaS<DA>::run0(csum[nt], kOne, kOne, kOne, kOne, av[nt][0], av[nt][1]);
              else MmaS<DA>::run(csum[nt], kOne, kOne, kOne, kOne, av[nt][2 * qq], av[nt][2 * qq + 1]);
            }
        }
#pragma unroll
        for (int rt = 0; rt < R; ++rt) {
          const float2 sc = lds64fv(srd[rt] + soff);
          float z0 = 0.0f, z1 = 0.0f;  // zero-points of rows g and g + 8 (INT4 asymmetric)
          if constexpr (AZ) {
            const uint32_t zz = lds16v(zrd[rt] + 16u * (uint32_t)bw);
            z0 = (float)(zz & 0xFFu);
            z1 = (float)(zz >> 8);
          }
          float part[NT][4];
#pragma unroll
          for (int qq = 0; qq < STEPS; ++qq) {
            // bytes 2qq, 2qq+1 of the lane's LB bytes of this segment
            const int b0 = sg * LB + 2 * qq, b1 = b0 + 1;
            const uint32_t w0 = wv[rt][0][b0 >> 2], w1 = wv[rt][1][b0 >> 2];
            uint32_t a0, a1, a2, a3;
            if constexpr (EXACT) {
              const float2 e0 = lut64f(lut_addr(w0, b0 & 3, lb));
              const float2 e1 = lut64f(lut_addr(w1, b0 & 3, lb));
              const float2 e2 = lut64f(lut_addr(w0, b1 & 3, lb));
              const float2 e3 = lut64f(lut_addr(w1, b1 & 3, lb));
              if constexpr (AZ) {  // (q - z) s, q - z exact
                a0 = Dt<DA>::pack2(__fmul_rn(sc.x, __fsub_rn(e0.x, z0)), __fmul_rn(sc.x, __fsub_rn(e0.y, z0)));
                a1 = Dt<DA>::pack2(__fmul_rn(sc.y, __fsub_rn(e1.x, z1)), __fmul_rn(sc.y, __fsub_rn(e1.y, z1)));
                a2 = Dt<DA>::pack2(__fmul_rn(sc.x, __fsub_rn(e2.x, z0)), __fmul_rn(sc.x, __fsub_rn(e2.y, z0)));
                a3 = Dt<DA>::pack2(__fmul_rn(sc.y, __fsub_rn(e3.x, z1)), __fmul_rn(sc.y, __fsub_rn(e3.y, z1)));
              } else {
                a0 = Dt<DA>::pack2(__fmul_rn(sc.x, e0.x), __fmul_rn(sc.x, e0.y));
                a1 = Dt<DA>::pack2(__fmul_rn(sc.y, e1.x), __fmul_rn(sc.y, e1.y));
                a2 = Dt<DA>::pack2(__fmul_rn(sc.x, e2.x), __fmul_rn(sc.x, e2.y));
                a3 = Dt<DA>::pack2(__fmul_rn(sc.y, e3.x), __fmul_rn(sc.y, e3.y));
              }
#pragma unroll
              for (int nt = 0; nt < NT; ++nt)
                MmaS<DA>::run(acc[rt][nt], a0, a1, a2, a3, av[nt][2 * qq], av[nt][2 * qq + 1]);
            } else {
              a0 = lut32(lut_addr(w0, b0 & 3, lb));
              a1 = lut32(lut_addr(w1, b0 & 3, lb));
              a2 = lut32(lut_addr(w0, b1 & 3, lb));
              a3 = lut32(lut_addr(w1, b1 & 3, lb));
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) {
                if (qq == 0) MmaS<DA>::run0(part[nt], a0, a1, a2, a3, av[nt][0], av[nt][1]);
                else MmaS<DA>::run(part[nt], a0, a1, a2, a3, av[nt][2 * qq], av[nt][2 * qq + 1]);
              }
            }
          }
          if constexpr (!EXACT) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              acc[rt][nt][0] = fmaf(sc.x, part[nt][0], acc[rt][nt][0]);
              acc[rt][nt][1] = fmaf(sc.x, part[nt][1], acc[rt][nt][1]);
              acc[rt][nt][2] = fmaf(sc.y, part[nt][2], acc[rt][nt][2]);
              acc[rt][nt][3] = fmaf(sc.y, part[nt][3], acc[rt][nt][3]);
            }
            if constexpr (AZ) {  // - z s S
              const float n0 = -z0 * sc.x, n1 = -z1 * sc.y;
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) {
                acc[rt][nt][0] = fmaf(n0, csum[nt][0], acc[rt][nt][0]);
                acc[rt][nt][1] = fmaf(n0, csum[nt][1], acc[rt][nt][1]);
                acc[rt][nt][2] = fmaf(n1, csum[nt][2], acc[rt][nt][2]);
                acc[rt][nt][3] = fmaf(n1, csum[nt][3], acc[rt][nt][3]);
              }
            }
          }
        }
      }
      // Release the stage after the MMAs, which consumed every value read
      // from it: no read of the slot can still be pending when the next copy
      // overwrites it (an arrive issued right after the loads may overtake
      // them).  __syncwarp orders all lanes' reads before lane 0's arrive.
      __syncwarp();
      if (lane == 0) mbar_arrive(sempty(s));
      if (++s == S) { s = 0; ph ^= 1u; }
    }
    if (!ok) break;

    if (cu.last) {
      const int Q = mt.n_stages;
      if (qstart == 0 && cu.q1 == Q) {
        // the whole k range of these rows went through this warp
#pragma unroll
        for (int rt = 0; rt < R; ++rt)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int row = w_base + rt * 16 + (j >> 1) * 8 + g;
              const int m = nt * 8 + 2 * tig + (j & 1);
              if (m < M && row < N) gs_store(mt.Y, p.y_dtype, (int64_t)m * N + row, acc[rt][nt][j]);
            }
      } else if (w_base < N) {
        // a partial tile: its rows go to this CTA's slot for the role
        const bool role0 = gi - (uint32_t)(cu.q0 - qstart) == g0;  // the segment holds the CTA's first stage
        float *slot = p.slots + ((int64_t)(blockIdx.x * 2 + (role0 ? 0 : 1)) * kGsRows + warp * 16 * R + g) * MW + 2 * tig;
#pragma unroll
        for (int rt = 0; rt < R; ++rt)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h)
              __stcg(reinterpret_cast<float2 *>(slot + (rt * 16 + h * 8) * MW + nt * 8),
                     make_float2(acc[rt][nt][2 * h], acc[rt][nt][2 * h + 1]));
        if (role0) {
          pend_mi0 = cu.mi;
          pend_tile0 = cu.tile;
          done0 = count_piece(cu.mi, cu.tile, (unsigned)(cu.q1 - qstart));
        } else {
          pend_mi1 = cu.mi; pend_tile1 = cu.tile; pend_len1 = cu.q1 - qstart;
        }
      }
    }
    gi = gn;
  }
  if (!ok) return;
  if (pend_mi1 >= 0) sum_piece(pend_mi1, pend_tile1, count_piece(pend_mi1, pend_tile1, (unsigned)pend_len1));
  if (pend_mi0 >= 0 && done0) sum_piece(pend_mi0, pend_tile0, done0);
}

}  // namespace q4
