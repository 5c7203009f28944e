// gemv.cuh -- fused 4-bit dequant-GEMV for decode batches (sm_100a):
// Y[M,N] = A[M,K] . W^[N,K]^T for 1 <= M <= 32 in one pass over the weights.
//
// What it computes: n4n.ai, "What is 4-bit quantization and why does it
// matter?", "Why it matters for deployment" (decode at batch < 32 reads every
// weight once per generated token and is bound by that read) and
// learn.pranaymahendrakar.com, "Loading a model in 4-bit", "Where the accuracy
// goes" (the weights are dequantized to the compute dtype, then multiplied in
// 16 bits).  Here the dequantization happens in registers as the packed
// weights stream by, and the products accumulate in fp32.  NF4 states use the
// 16 printed levels and the per-block absmax (double-dequantized c~ when the
// state has double quantization); INT4 symmetric states the integers -8..7 and
// the group scale; INT4 asymmetric states the integers 0..15, the group scale
// s and the zero-point z (robotsatlas.com, "INT4", "Components"):
//   sum_k a_k (q_k - z) s = s (sum_k a_k q_k - z sum_k a_k),
// the activation sum of each block coming from one extra MMA per k-step.
//
// Design (B200, memory-bound decode).  The weights are read exactly once, so
// the kernel is built to keep enough of them in flight with as few
// instructions per weight as possible:
//   * a producer warp streams the packed weights through a ring of shared-
//     memory stages with TMA ([256 rows x 128 bytes] = one 256-k chunk of a
//     256-row tile per stage, 128-byte swizzled); the compute warps read
//     their rows with conflict-free ldmatrix and release the stage;
//   * the MMA is the warp-level mma.sync.m16n8k16 with the weights on its
//     16-row side (swap-AB) and up to 32 activation rows on its n side (NT
//     tiles of 8): decode batches are far too small for tcgen05 tiles, and
//     what limits a decode GEMV is issuing the dequantization, not MMA rate;
//   * a packed byte becomes the pair of its two 16-bit levels with one PRMT
//     (which forms the shared-memory address: the table sits on a 64 KB
//     boundary, the byte becomes address bits 8..15) and one 32-bit shared
//     load from a 256-entry table with one copy per lane (conflict-free);
//   * the k order is permuted identically for weights and activations: a
//     lane holds 4 contiguous packed bytes (8 k) of each 32-k piece of rows
//     g and g + 8, so every MMA k-step stays inside one block; each block's
//     fp32 MMA partial is scaled once by its c~ (the MMA runs on the
//     unscaled levels); the blocks of a chunk are independent MMA chains,
//     interleaved two at a time;
//   * activations are read through L1 (all warps of a CTA walk the same
//     chunks together); the producer warp prefetches them into L1.  Lanes
//     of activation columns >= M read a valid row anyway (their output
//     columns are never stored), so no load is predicated;
//   * each warp computes the c~ of its rows for a window of 16 blocks into a
//     small shared buffer, one window ahead of its use;
//   * work: the concatenation of every matrix's (tile of 256 rows, 256-k
//     chunk) units, tile-major, cut into one contiguous range per CTA; all
//     warps of a CTA own different rows of the same tiles.  Only a range's
//     first and last tiles can be partial: their fp32 rows go to per-CTA
//     slots and the last contributor to count a 16-row group sums the slots
//     of every contributor in CTA order (deterministic) and zeroes them, so
//     every call leaves the workspace zeroed.  A CTA processes its partial
//     last tile first, then its partial first tile, then the full tiles, so
//     the cross-CTA sums overlap the streaming of the full tiles;
//   * every mbarrier wait is bounded by the launch's wait limit: a wait that
//     runs out raises Q4_STATUS_TIMEOUT, the compute warps stop, and the
//     producer waits for its copies in flight before the CTA exits.
// bf16 activations multiply the exact w^ = bf16(c~ * level) (the definition
// rounds the dequantized weight to the compute dtype; bf16 has too few bits
// to leave that rounding out), built from a binary32 pair table.
#pragma once
#include <cuda.h>

#include "gemm.cuh"  // mbarrier / TMA wrappers
#include "q4_common.cuh"

namespace q4 {

constexpr int kGvChunk = 256;      // k per chunk: 128 packed bytes of a row
constexpr int kGvMaxGroup = 16;    // matrices per grouped launch
constexpr int kGvWin = 16;         // blocks per c~ window
constexpr int kGvMaxCtas = 1024;   // grid bound (slots are per CTA)
constexpr int kGvInfoBytes = kGvMaxGroup * 96;
constexpr int kGvMaxStages = 12;  // ring stages
constexpr int kGvBarBytes = 2 * kGvMaxStages * 8 + 16;  // full / empty barriers + abort flag

struct GvInfo {
  const uint8_t *packed;      // [N, K/2]
  const uint16_t *A;          // [M, K], 16-bit activations
  void *Y;                    // [M, N]
  const float *absmax;        // per block: NF4 c, or the INT4 scale s
  const int8_t *absmax_q;     // double quantization: int8 code per block
  const float *absmax_scale;  //   second-level scale per 256 blocks
  const float *absmax_mean;   //   the mean
  const uint8_t *zero;        // INT4 asymmetric zero-points, nibble per block
  unsigned *cnt;              // per 16-row group: chunks counted (zero between calls)
  uint32_t unit_begin;        // first global unit of this matrix
  int32_t N, K;
  int32_t n_tiles, n_chunks;  // tiles of TR rows; 256-k chunks per row
  int32_t pad;
};
static_assert(sizeof(GvInfo) == 96, "GvInfo layout");

struct alignas(64) GvMat {
  CUtensorMap tmW;  // packed [N, K/2] bytes, box {128 bytes, tile rows}, 128-byte swizzle
  GvInfo f;         // copied to shared memory by every CTA
};

struct GvParams {
  GvMat mat[kGvMaxGroup];
  int32_t count;
  int32_t M;
  int32_t y_dtype;
  uint32_t total_units;  // below 2^32 / kGvMaxCtas
  float *slots;          // [grid][2][TR rows][8 NT] fp32 partial rows of a CTA's first / last tile
  int *status;
  uint64_t wait_ns;      // bound of every mbarrier wait
  int32_t stall_copies;  // test hook: issue no copies, so every stage wait runs out
  int32_t scale_f16;     // INT4: binary16 scales
  float levels[16];      // the value of each 4-bit code (NF4 levels, or integers)
};

// Dynamic shared memory: the whole carve-out.  The 64 KB table sits at the
// first 64 KB boundary; the matrix fields, barriers and c~ buffers and the
// ring of weight stages fill the space below and above it.
constexpr int kGvSmemBytes = 227 * 1024;

// Kernel shape for NT activation tiles: R 16-row groups per compute warp,
// WARPS compute warps (plus the producer warp) per CTA; a tile is
// 16 * R * WARPS <= 256 rows (one TMA box).
template <int NT> struct GvShape;
template <> struct GvShape<1> { static constexpr int R = 1, WARPS = 16; };
template <> struct GvShape<2> { static constexpr int R = 1, WARPS = 16; };
template <> struct GvShape<4> { static constexpr int R = 1, WARPS = 8; };

// Scale modes: c~ source of a block.
constexpr int kGvPlain = 0;  // fp32 per block (NF4 without double quantization, INT4 symmetric)
constexpr int kGvDq = 1;     // q2 * s2 + mu (NF4 with double quantization)
constexpr int kGvAsym = 2;   // fp32 scale s and zero-point z (INT4 asymmetric)

// CTA c covers units [c T / G, (c+1) T / G).
__device__ __forceinline__ uint32_t gv_begin(uint32_t c, uint32_t T, uint32_t G) {
  return (uint32_t)(((uint64_t)c * T) / G);
}
__device__ __forceinline__ int gv_cta_of(uint32_t x, uint32_t T, uint32_t G) {
  uint32_t c = (uint32_t)(((uint64_t)x * G) / T);
  while (c + 1 < G && gv_begin(c + 1, T, G) <= x) ++c;
  while (c > 0 && gv_begin(c, T, G) > x) --c;
  return (int)c;
}

// One position of the walk: matrix, tile, chunk and unit index.
struct GvPos {
  uint32_t u;
  int mi, tile, chunk;
};
__device__ __forceinline__ GvPos gv_decode(const GvInfo *info, int count, uint32_t u) {
  GvPos p;
  p.u = u;
  p.mi = 0;
#pragma unroll 1
  while (p.mi + 1 < count && u >= info[p.mi + 1].unit_begin) ++p.mi;
  const uint32_t local = u - info[p.mi].unit_begin;
  const uint32_t nc = (uint32_t)info[p.mi].n_chunks;
  p.tile = (int)(local / nc);
  p.chunk = (int)(local - (uint32_t)p.tile * nc);
  return p;
}

// The CTA's walk is two contiguous unit runs: [a1, u1) (its partial last
// tile, when there is one), then [u0, a1).
struct GvWalk {
  uint32_t u0, u1, a1;
};

// A tile piece of the walk: chunks [q0, q1) of one tile; u is the unit index
// of chunk q0.  A piece ends at its tile's end or at its run's end.
struct GvPiece {
  int mi, tile, q0, q1;
  uint32_t u;
};
__device__ __forceinline__ GvPiece gv_piece_at(const GvInfo *info, int count, uint32_t u, uint32_t end) {
  const GvPos ps = gv_decode(info, count, u);
  GvPiece pc;
  pc.mi = ps.mi;
  pc.tile = ps.tile;
  pc.q0 = ps.chunk;
  pc.q1 = min(info[ps.mi].n_chunks, ps.chunk + (int)(end - u));
  pc.u = u;
  return pc;
}
// The piece after pc; false at the end of the walk.
__device__ __forceinline__ bool gv_piece_next(const GvInfo *info, int count, const GvWalk &wk, const GvPiece &pc,
                                              GvPiece &nx) {
  const uint32_t u = pc.u + (uint32_t)(pc.q1 - pc.q0);
  const uint32_t end = pc.u >= wk.a1 ? wk.u1 : wk.a1;  // end of pc's run
  if (u == end) {
    if (end == wk.u1 && wk.a1 != wk.u1) {  // the first run is done: continue at the CTA's first unit
      nx = gv_piece_at(info, count, wk.u0, wk.a1);
      return true;
    }
    return false;
  }
  GvPiece q;
  q.mi = pc.mi;
  q.tile = pc.tile + 1;
  if (q.tile == info[q.mi].n_tiles) {
    q.tile = 0;
    ++q.mi;
  }
  q.q0 = 0;
  q.q1 = min(info[q.mi].n_chunks, (int)(end - u));
  q.u = u;
  nx = q;
  return true;
}

template <int DA> struct GvMma;
template <> struct GvMma<Q4_F16> {
  static __device__ __forceinline__ void run(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
  // d = A . B (the accumulator starts at zero)
  static __device__ __forceinline__ void run0(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%10,%10,%10,%10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
  }
  static constexpr uint32_t kOnes = 0x3C003C00u;  // (1.0, 1.0)
};
template <> struct GvMma<Q4_BF16> {
  static __device__ __forceinline__ void run(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
  static __device__ __forceinline__ void run0(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%10,%10,%10,%10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
  }
  static constexpr uint32_t kOnes = 0x3F803F80u;
};

// Four table lookups (the A fragment of one k-step) feeding NT fp16 MMAs in
// one asm block, so the looked-up values land in the operand registers.
// ACC: accumulate into d, else d = A . B.
template <int NT, bool ACC> struct GvLutMma;
template <bool ACC> struct GvLutMma<1, ACC> {
  static __device__ __forceinline__ void run(float (&d)[1][4], uint32_t x0, uint32_t x1, uint32_t x2, uint32_t x3,
                                             const uint32_t (&b)[1][2]) {
    if constexpr (ACC)
      asm("{ .reg .b32 t0, t1, t2, t3;\n"
          "ld.shared.b32 t0, [%6]; ld.shared.b32 t1, [%7]; ld.shared.b32 t2, [%8]; ld.shared.b32 t3, [%9];\n"
          "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {t0,t1,t2,t3}, {%4,%5}, {%0,%1,%2,%3}; }"
          : "+f"(d[0][0]), "+f"(d[0][1]), "+f"(d[0][2]), "+f"(d[0][3])
          : "r"(b[0][0]), "r"(b[0][1]), "r"(x0), "r"(x1), "r"(x2), "r"(x3));
    else
      asm("{ .reg .b32 t0, t1, t2, t3;\n"
          "ld.shared.b32 t0, [%6]; ld.shared.b32 t1, [%7]; ld.shared.b32 t2, [%8]; ld.shared.b32 t3, [%9];\n"
          "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {t0,t1,t2,t3}, {%4,%5}, {%10,%10,%10,%10}; }"
          : "=f"(d[0][0]), "=f"(d[0][1]), "=f"(d[0][2]), "=f"(d[0][3])
          : "r"(b[0][0]), "r"(b[0][1]), "r"(x0), "r"(x1), "r"(x2), "r"(x3), "f"(0.0f));
  }
};
template <bool ACC> struct GvLutMma<2, ACC> {
  static __device__ __forceinline__ void run(float (&d)[2][4], uint32_t x0, uint32_t x1, uint32_t x2, uint32_t x3,
                                             const uint32_t (&b)[2][2]) {
    if constexpr (ACC)
      asm("{ .reg .b32 t0, t1, t2, t3;\n"
          "ld.shared.b32 t0, [%12]; ld.shared.b32 t1, [%13]; ld.shared.b32 t2, [%14]; ld.shared.b32 t3, [%15];\n"
          "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {t0,t1,t2,t3}, {%8,%9}, {%0,%1,%2,%3};\n"
          "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%4,%5,%6,%7}, {t0,t1,t2,t3}, {%10,%11}, {%4,%5,%6,%7}; }"
          : "+f"(d[0][0]), "+f"(d[0][1]), "+f"(d[0][2]), "+f"(d[0][3]), "+f"(d[1][0]), "+f"(d[1][1]), "+f"(d[1][2]),
            "+f"(d[1][3])
          : "r"(b[0][0]), "r"(b[0][1]), "r"(b[1][0]), "r"(b[1][1]), "r"(x0), "r"(x1), "r"(x2), "r"(x3));
    else
      asm("{ .reg .b32 t0, t1, t2, t3;\n"
          "ld.shared.b32 t0, [%12]; ld.shared.b32 t1, [%13]; ld.shared.b32 t2, [%14]; ld.shared.b32 t3, [%15];\n"
          "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {t0,t1,t2,t3}, {%8,%9}, {%16,%16,%16,%16};\n"
          "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%4,%5,%6,%7}, {t0,t1,t2,t3}, {%10,%11}, {%16,%16,%16,%16}; }"
          : "=f"(d[0][0]), "=f"(d[0][1]), "=f"(d[0][2]), "=f"(d[0][3]), "=f"(d[1][0]), "=f"(d[1][1]), "=f"(d[1][2]),
            "=f"(d[1][3])
          : "r"(b[0][0]), "r"(b[0][1]), "r"(b[1][0]), "r"(b[1][1]), "r"(x0), "r"(x1), "r"(x2), "r"(x3), "f"(0.0f));
  }
};
template <bool ACC> struct GvLutMma<4, ACC> {
  static __device__ __forceinline__ void run(float (&d)[4][4], uint32_t x0, uint32_t x1, uint32_t x2, uint32_t x3,
                                             const uint32_t (&b)[4][2]) {
    float (&h0)[2][4] = *reinterpret_cast<float (*)[2][4]>(&d[0]);
    float (&h1)[2][4] = *reinterpret_cast<float (*)[2][4]>(&d[2]);
    const uint32_t(&c0)[2][2] = *reinterpret_cast<const uint32_t(*)[2][2]>(&b[0]);
    const uint32_t(&c1)[2][2] = *reinterpret_cast<const uint32_t(*)[2][2]>(&b[2]);
    GvLutMma<2, ACC>::run(h0, x0, x1, x2, x3, c0);
    GvLutMma<2, ACC>::run(h1, x0, x1, x2, x3, c1);
  }
};

__device__ __forceinline__ void gv_store(void *Y, int ydt, int64_t idx, float v) {
  if (ydt == Q4_F32) reinterpret_cast<float *>(Y)[idx] = v;
  else if (ydt == Q4_F16) reinterpret_cast<uint16_t *>(Y)[idx] = Dt<Q4_F16>::from_f(v);
  else reinterpret_cast<uint16_t *>(Y)[idx] = Dt<Q4_BF16>::from_f(v);
}

__device__ __forceinline__ uint32_t gv_lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ float2 gv_lds64f(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0,%1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr));
  return v;
}
__device__ __forceinline__ float4 gv_lds128f(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
  return v;
}
// Table lookups: the table is constant after the start-up barrier.
__device__ __forceinline__ uint32_t gv_lut32(uint32_t addr) {
  uint32_t v;
  asm("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ float2 gv_lut64f(uint32_t addr) {
  float2 v;
  asm("ld.shared.v2.f32 {%0,%1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr));
  return v;
}
__device__ __forceinline__ void gv_sts32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void gv_sts64(uint32_t addr, uint32_t a, uint32_t b) {
  asm volatile("st.shared.v2.b32 [%0], {%1,%2};" ::"r"(addr), "r"(a), "r"(b) : "memory");
}
// Address of the table entry of byte j of `word`: byte 1 of the address is
// the packed byte; bytes 0, 2, 3 come from `lb` (table base + lane offset,
// whose byte 1 is zero because the table is 64 KB aligned).
__device__ __forceinline__ uint32_t gv_lut_addr(uint32_t word, int j, uint32_t lb) {
  return __byte_perm(word, lb, 0x7604u | ((uint32_t)j << 4));
}
__device__ __forceinline__ void gv_fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }

// Loads of a lane's packed bytes from a ring stage (ordered after the
// stage's barrier wait) and L1-cached loads of activations.
template <int BYTES> struct GvLds;
template <> struct GvLds<4> {
  static __device__ __forceinline__ void run(uint32_t a, uint32_t *w) {
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(w[0]) : "r"(a));
  }
};
template <> struct GvLds<8> {
  static __device__ __forceinline__ void run(uint32_t a, uint32_t *w) {
    asm volatile("ld.shared.v2.b32 {%0,%1}, [%2];" : "=r"(w[0]), "=r"(w[1]) : "r"(a));
  }
};
template <> struct GvLds<16> {
  static __device__ __forceinline__ void run(uint32_t a, uint32_t *w) {
    asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];" : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]) : "r"(a));
  }
};
// Wait by every lane of a warp (each lane acquires the phase itself; the
// common case -- the stage landed long ago -- is one probe and no branch on
// the lane).  Bounded like mbar_wait.
__device__ __forceinline__ bool gv_wait_all(uint32_t bar, uint32_t parity, int *status, volatile int *abort,
                                            uint64_t limit_ns) {
  if (__all_sync(0xffffffffu, mbar_try(bar, parity))) return true;
  const bool ok = mbar_wait(bar, parity, status, abort, limit_ns);
  return __all_sync(0xffffffffu, ok);
}
// Arrive on a barrier from lane 0 only, as one predicated instruction.
__device__ __forceinline__ void gv_arrive_lane0(uint32_t bar, int lane) {
  asm volatile("{ .reg .pred p; .reg .b64 st; setp.eq.u32 p, %1, 0; @p mbarrier.arrive.shared::cta.b64 st, [%0]; }" ::"r"(bar),
               "r"(lane)
               : "memory");
}

// Four 8x8 b16 matrices from shared memory (lane l supplies the row address
// of matrix l / 8); register i of lane (g, tig) holds row g, b16 elements
// 2 tig and 2 tig + 1 of matrix i -- here 4 packed bytes of a weight row.
__device__ __forceinline__ void gv_ldmatrix_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ uint4 gv_ldg_act(const uint16_t *p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}
__device__ __forceinline__ void gv_prefetch_l1(const void *p) {
  asm volatile("prefetch.global.L1 [%0];" ::"l"(p));
}

// Inputs of the c~ of 8 blocks of one row (blocks half*8 + j of a window),
// loaded one window ahead of their use.
template <int MODE> struct GvScaleIn;
template <> struct GvScaleIn<kGvPlain> {
  float f[8];
  int nvalid;
};
template <> struct GvScaleIn<kGvDq> {
  uint32_t c0, c1;
  float s2a, s2b, mu;
  int bsplit, nvalid;
};
template <> struct GvScaleIn<kGvAsym> {
  float f[8];
  uint32_t z;  // 8 zero-point nibbles
  int nvalid;
};

// Load the c~ inputs of row `row` (< N, else nothing), blocks b0 .. b0+7.
template <int MODE>
__device__ __forceinline__ void gv_scale_load(const GvInfo &mt, int B, int row, int b0, bool sf16,
                                              GvScaleIn<MODE> &in) {
  const int nbk = mt.K / B;
  in.nvalid = (row < mt.N) ? max(0, min(8, nbk - b0)) : 0;
  if constexpr (MODE == kGvDq) {
    in.c0 = in.c1 = 0;
    in.s2a = in.s2b = in.mu = 0.0f;
    in.bsplit = 8;
    if (in.nvalid == 0) return;
    const int64_t bi0 = (int64_t)row * nbk + b0;
    in.mu = __ldg(mt.absmax_mean);
    const int64_t g0 = bi0 >> 8;
    in.s2a = __ldg(mt.absmax_scale + g0);
    in.s2b = __ldg(mt.absmax_scale + ((bi0 + in.nvalid - 1) >> 8));
    in.bsplit = (int)min((int64_t)8, ((g0 + 1) << 8) - bi0);
    if (in.nvalid == 8 && ((uintptr_t)(mt.absmax_q + bi0) & 3u) == 0) {
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
#pragma unroll
    for (int j = 0; j < 8; ++j) in.f[j] = 0.0f;
    if constexpr (MODE == kGvAsym) in.z = 0;
    if (in.nvalid == 0) return;
    const int64_t bi0 = (int64_t)row * nbk + b0;
    if (in.nvalid == 8) {
      ld_scales8(mt.absmax, bi0, sf16, in.f);
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j < in.nvalid) in.f[j] = ld_scale(mt.absmax, bi0 + j, sf16);
    }
    if constexpr (MODE == kGvAsym) {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j < in.nvalid) {
          const int64_t b = bi0 + j;
          in.z |= (uint32_t)((__ldg(mt.zero + (b >> 1)) >> (4 * (b & 1))) & 15) << (4 * j);
        }
    }
  }
}

// c~ of block j (0..7) of the inputs: q2 * s2 + mu with double quantization
// (two roundings, as the state dequantizes), else the stored fp32 value; 0
// past the row's end.
template <int MODE>
__device__ __forceinline__ float gv_scale_value(const GvScaleIn<MODE> &in, int j) {
  if constexpr (MODE == kGvDq) {
    const uint32_t w = j < 4 ? in.c0 : in.c1;
    const float code = (float)(int)(int8_t)(uint8_t)(w >> (8 * (j & 3)));
    const float v = __fadd_rn(__fmul_rn(code, j < in.bsplit ? in.s2a : in.s2b), in.mu);
    return j < in.nvalid ? v : 0.0f;
  } else {
    return in.f[j];
  }
}

template <int DA, int MODE, int NT, int B>
__global__ void __launch_bounds__((GvShape<NT>::WARPS + 1) * 32, 1) gemv_kernel(const __grid_constant__ GvParams p) {
  constexpr int R = GvShape<NT>::R;
  constexpr int WARPS = GvShape<NT>::WARPS;
  constexpr int PRODUCER = WARPS;
  constexpr bool EXACT = (DA == Q4_BF16);
  constexpr bool ASYM = (MODE == kGvAsym);
  constexpr int PB = B / 32;                        // 32-k pieces per block
  constexpr int MW = 8 * NT;
  constexpr int TR = 16 * R * WARPS;                 // rows per tile
  constexpr int STAGE = TR * (kGvChunk / 2);         // bytes per ring stage
  constexpr int WC = kGvWin * B / kGvChunk;          // chunks per c~ window
  constexpr uint32_t ES = EXACT ? 8u : 4u;           // table entry bytes per lane
  constexpr int SV = ASYM ? 8 : 4;                   // c~ buffer bytes per (row, block)
  constexpr uint32_t kBuf = 16u * kGvWin * SV;       // one c~ buffer: 16 rows x 16 blocks
  static_assert(TR <= 256, "a tile is one TMA box");
  static_assert(WC >= 1 && kGvWin * B % kGvChunk == 0, "a window is whole chunks");

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // ---- shared memory: the table at the first 64 KB boundary; the matrix
  // fields, barriers and c~ buffers in whichever free region holds them; the
  // ring in up to two runs of stages.  The fp16 pair table fills 128 of
  // every 256 bytes: with 4-byte c~ values the buffers live in those gaps.
  constexpr bool GAPS = !EXACT && !ASYM && WARPS * R * 2 * kBuf == 256 * 128;
  const uint32_t base = (uint32_t)__cvta_generic_to_shared(smem_raw);
  const uint32_t end = base + kGvSmemBytes;
  const uint32_t lut = (base + 0xFFFFu) & ~0xFFFFu;
  constexpr uint32_t kMisc = kGvInfoBytes + kGvBarBytes + (GAPS ? 0u : (uint32_t)WARPS * R * 2u * kBuf);
  uint32_t lo = base, hi = lut + 0x10000u, misc;
  if (lut - lo >= kMisc) {
    misc = lo;
    lo += kMisc;
  } else {
    misc = hi;
    hi += kMisc;
  }
  const uint32_t ra = (lo + 1023u) & ~1023u, rb = (hi + 1023u) & ~1023u;
  int SA = ra + STAGE <= lut ? (int)((lut - ra) / STAGE) : 0;
  const int SB = rb + STAGE <= end ? (int)((end - rb) / STAGE) : 0;
  const int S = min(kGvMaxStages, SA + SB);
  SA = min(SA, S);
  const uint32_t rb_adj = rb - (uint32_t)SA * STAGE;  // stage s >= SA at rb_adj + s * STAGE
  if (S < 2 || hi > end) {  // not reachable with this launch's shared-memory size; refuse loudly
    if (threadIdx.x == 0) raise_status(p.status, Q4_STATUS_LAYOUT);
    return;
  }
  auto stage_addr = [&](int st) { return (st < SA ? ra : rb_adj) + (uint32_t)st * STAGE; };
  GvInfo *info = reinterpret_cast<GvInfo *>(smem_raw + (misc - base));
  const uint32_t bar0 = misc + kGvInfoBytes;
  auto sfull = [&](int st) { return bar0 + 8u * st; };
  auto sempty = [&](int st) { return bar0 + 8u * (kGvMaxStages + st); };
  volatile int *abort = reinterpret_cast<volatile int *>(smem_raw + (bar0 + 16u * kGvMaxStages - base));
  const uint32_t cbuf0 = bar0 + kGvBarBytes;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tig = lane & 3;

  // ---- set-up that touches no global memory, before waiting for the
  // previous kernel of the stream: matrix fields, barriers, pair table
  if (tid < p.count) info[tid] = p.mat[tid].f;
  if (warp == PRODUCER && lane == 0) {
    for (int b = 0; b < S; ++b) {
      mbar_init(sfull(b), 1);
      mbar_init(sempty(b), WARPS);  // one arrival per compute warp
    }
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int i = tid; i < 256 * 32; i += (WARPS + 1) * 32) {
    const int b = i >> 5, l = i & 31;
    const uint32_t a = lut + (uint32_t)b * 256u + (uint32_t)l * ES;
    if constexpr (EXACT) gv_sts64(a, __float_as_uint(p.levels[b & 15]), __float_as_uint(p.levels[b >> 4]));
    else gv_sts32(a, Dt<DA>::pack2(p.levels[b & 15], p.levels[b >> 4]));
  }
  __syncthreads();
  pdl_launch_then_wait();

  const int count = p.count;
  const int M = p.M;
  const uint32_t T = p.total_units, G = gridDim.x;
  GvWalk wk;
  wk.u0 = gv_begin(blockIdx.x, T, G);
  wk.u1 = gv_begin(blockIdx.x + 1, T, G);
  if (wk.u0 >= wk.u1) return;
  {
    // the last tile of the range goes first when it is partial and is not
    // also the first tile
    const GvPos last = gv_decode(info, count, wk.u1 - 1);
    const uint32_t tile_start = wk.u1 - 1 - (uint32_t)last.chunk;
    wk.a1 = (tile_start > wk.u0 && last.chunk != info[last.mi].n_chunks - 1) ? tile_start : wk.u1;
  }
  const uint32_t n_units = wk.u1 - wk.u0;
  const GvPiece start = wk.a1 != wk.u1 ? gv_piece_at(info, count, wk.a1, wk.u1)
                                         : gv_piece_at(info, count, wk.u0, wk.u1);

  if (warp == PRODUCER) {
    // ---------------------------------------------------------- producer
    GvPiece pc = start;
    int q = pc.q0, s = 0, issued = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (uint32_t left = n_units; left && ok; --left) {
      if (q == pc.q1) {
        GvPiece nx;
        gv_piece_next(info, count, wk, pc, nx);
        pc = nx;
        q = nx.q0;
      }
      if (lane == 0) {
        if (!mbar_wait(sempty(s), ph ^ 1u, p.status, abort, p.wait_ns)) {
          ok = false;
        } else if (!p.stall_copies) {
          // the compute warps' reads of this slot (generic proxy) come before
          // the copy that overwrites it (async proxy)
          fence_proxy_async_smem();
          mbar_arrive_expect_tx(sfull(s), (uint32_t)STAGE);
          tma_load_2d(stage_addr(s), &p.mat[pc.mi].tmW, sfull(s), q * (kGvChunk / 2), pc.tile * TR);
          ++issued;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (ok) {
        // this chunk's activation rows (four 128-byte lines per row) into L1
        // for the compute warps
        const GvInfo &mt = info[pc.mi];
        const int kk = q * kGvChunk + (lane & 3) * 64;
#pragma unroll
        for (int c0 = 0; c0 < MW; c0 += 8) {
          const int col = c0 + (lane >> 2);
          if (col < M && kk < mt.K) gv_prefetch_l1(mt.A + (int64_t)col * mt.K + kk);
        }
      }
      ++q;
      if (++s == S) {
        s = 0;
        ph ^= 1u;
      }
    }
    if (lane == 0 && *abort) {
      // The compute warps may have left: let the copies still in flight land
      // before the CTA exits (older stages were released, so complete).
      int ss = s;
      uint32_t pp = ph;
      if (!ok && --ss < 0) {  // the stage whose wait failed was not issued: step back over it
        ss = S - 1;
        pp ^= 1u;
      }
      for (int j = 0; j < min(issued, S); ++j) {
        if (--ss < 0) { ss = S - 1; pp ^= 1u; }
        // issued copies complete within microseconds: wait with the full
        // default bound whatever the launch's limit
        int dummy = 0;
        volatile int no_abort = 0;
        mbar_wait(sfull(ss), pp, &dummy, &no_abort, kWaitLimitNs);
      }
    }
    return;
  }

  // ------------------------------------------------------------ compute warps
  const uint32_t lb = lut + ES * (uint32_t)lane;
  const int wrow = warp * 16 * R;  // first row of this warp inside a tile

  // ---- c~ windows.  Lane (rr = lane & 15, hh = lane >> 4) fills blocks
  // hh * 8 + j of row rr of each row group; block bw of rows (g, g + 8) is
  // read as one vector at (bw * 8 + g) * 2 * SV.
  GvScaleIn<MODE> sin[R];
  auto window_load = [&](int mi, int tile, int chunk) {
    const GvInfo &mt = info[mi];
    const int wb0 = (chunk / WC) * kGvWin + (lane >> 4) * 8;
#pragma unroll
    for (int rt = 0; rt < R; ++rt)
      gv_scale_load<MODE>(mt, B, tile * TR + wrow + rt * 16 + (lane & 15), wb0, p.scale_f16 != 0, sin[rt]);
  };
  // byte o of c~ buffer (row group rt, parity par): contiguous, or spread
  // over the table's 128-byte gaps
  auto caddr = [&](int rt, uint32_t par, uint32_t o) -> uint32_t {
    const uint32_t id = (uint32_t)(warp * R + rt) * 2u + par;
    if constexpr (GAPS) return lut + 128u + (id * (kBuf / 128u) + (o >> 7)) * 256u + (o & 127u);
    else return cbuf0 + id * kBuf + o;
  };
  uint32_t sb = 0;  // parity of the buffer the next window is written to
  auto window_store = [&]() {
    const int rr = lane & 15, hh = lane >> 4;
#pragma unroll
    for (int rt = 0; rt < R; ++rt) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int bw = hh * 8 + j;
        const uint32_t o = ((uint32_t)(bw * 8 + (rr & 7)) * 2u + (uint32_t)(rr >> 3)) * (uint32_t)SV;
        const float v = gv_scale_value<MODE>(sin[rt], j);
        if constexpr (ASYM) {
          // (s, s z) for the integer-code MMA, (s, z) for the exact bf16 weights
          const float z = (float)((sin[rt].z >> (4 * j)) & 15u);
          gv_sts64(caddr(rt, sb, o), __float_as_uint(v), __float_as_uint(EXACT ? z : __fmul_rn(v, z)));
        } else {
          gv_sts32(caddr(rt, sb, o), __float_as_uint(v));
        }
      }
    }
  };
  window_load(start.mi, start.tile, start.q0);

  // per piece: the lane's activation pointers (column nt * 8 + g, clamped to
  // a valid row; its k offset inside a segment) and the matrix fields
  GvPiece cpc = start;
  int cq = start.q0, cK = 0;
  const uint16_t *ap[NT];
  auto c_setup = [&]() {
    const GvInfo &mt = info[cpc.mi];
    cK = mt.K;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
      ap[nt] = mt.A + (int64_t)min(nt * 8 + g, M - 1) * mt.K + 8 * tig;
  };
  c_setup();

  // c~ buffer bases of this lane (rows g, g + 8 of block 0) per row group
  // and parity
  uint32_t cbs[R][2];
#pragma unroll
  for (int rt = 0; rt < R; ++rt)
#pragma unroll
    for (uint32_t par = 0; par < 2; ++par) cbs[rt][par] = caddr(rt, par, (uint32_t)(g * 2 * SV));

  // ldmatrix offsets inside a stage: lane l addresses row (l & 15) of its
  // row group and piece 2 jj + (l >> 4), 16-byte unit u of row r at u ^ (r & 7)
  uint32_t lmo[R][4];
#pragma unroll
  for (int rt = 0; rt < R; ++rt) {
    const int row = wrow + rt * 16 + (lane & 15);
#pragma unroll
    for (int jj = 0; jj < 4; ++jj)
      lmo[rt][jj] = (uint32_t)row * 128u + (uint32_t)(((2 * jj + (lane >> 4)) ^ (row & 7)) << 4);
  }

  float acc[R][NT][4];
#pragma unroll
  for (int rt = 0; rt < R; ++rt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[rt][nt][j] = 0.0f;
  uint32_t crd = 0;  // parity of the c~ buffers of the current window
  int s = 0;         // ring stage
  uint32_t ph = 0;
  bool ok = true;

#pragma unroll 1
  for (uint32_t left = n_units; left; --left) {
    if (cq == cpc.q0 || cq % WC == 0) {
      // a new window: publish its c~, then load the inputs of the next
      // window (in this piece, else at the start of the next piece)
      window_store();
      __syncwarp();
      crd = sb;
      sb ^= 1u;
      const int wend = (cq / WC + 1) * WC;
      if (wend < cpc.q1) {
        window_load(cpc.mi, cpc.tile, wend);
      } else {
        GvPiece nx;
        if (gv_piece_next(info, count, wk, cpc, nx)) window_load(nx.mi, nx.tile, nx.q0);
      }
    }
    const int kb = cq * kGvChunk;

    // ---- this chunk's packed bytes from the ring.  The stage holds the
    // tile's [rows x 128 bytes] with the 128-byte swizzle (16-byte unit u of
    // row r at unit u ^ (r & 7)); ldmatrix.x4 at piece pair jj gives
    // wq[jj][0..3] = rows (g, g + 8) x pieces (2 jj, 2 jj + 1): lane (g, tig)
    // holds bytes 4 tig .. 4 tig + 3 of each 16-byte piece, i.e. k =
    // 32 j + 8 tig + [0, 8) of piece j.  A piece lies inside one block.
    if (!gv_wait_all(sfull(s), ph, p.status, abort, p.wait_ns)) {
      ok = false;
      break;
    }
    uint32_t wq[R][4][4];
    {
      const uint32_t st = stage_addr(s);
#pragma unroll
      for (int rt = 0; rt < R; ++rt)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) gv_ldmatrix_x4(st + lmo[rt][jj], wq[rt][jj]);
    }
    // wq[rt][jj] = {row g piece 2jj, row g+8 piece 2jj, row g piece 2jj+1, row g+8 piece 2jj+1}
    // (ldmatrix matrix i is addressed by lanes 8i..8i+7: rows lr = lane & 15,
    // so matrices 0/1 are rows 0-7 / 8-15 of piece 2jj + 0, 2/3 of piece 2jj+1)

    // ---- 16 k-steps, two per piece; with two or more blocks per chunk the
    // blocks' MMA chains interleave two at a time
    constexpr int NBLK = kGvChunk / 32 / PB > 0 ? kGvChunk / 32 / PB : 1;  // blocks touched per chunk
    constexpr int IW = NBLK < 2 ? 1 : 2;
    // the order of the 8 pieces: block-pair group, then piece in block, then block
    auto piece_of = [](int i) {
      return (i / (IW * PB)) * IW * PB + (i % IW) * PB + (i / IW) % PB;
    };
    // activation offsets past K (a ragged last chunk, whose weights the copy
    // zero-filled) are clamped into the row: finite values times zero
    // this chunk's first block inside the c~ window, as a buffer offset
    const int bwc = (cq % WC) * (kGvChunk / B > 0 ? kGvChunk / B : 1);
    uint32_t coff;
    if constexpr (GAPS) coff = (uint32_t)((bwc >> 1) * 256 + (bwc & 1) * 64);
    else coff = (uint32_t)(bwc * 16 * SV);
    const bool ktail = kb + kGvChunk > cK;
    const int klim = cK - 8 - 8 * tig;
    const uint16_t *apc[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) apc[nt] = ap[nt] + kb;
    auto act_load = [&](int j, uint4 (&av)[NT]) {
      if (!ktail) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) av[nt] = gv_ldg_act(apc[nt] + 32 * j);
      } else {
        const int off = min(kb + 32 * j, klim) - kb;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) av[nt] = gv_ldg_act(apc[nt] + off);
      }
    };
    uint4 av[2][NT];
    act_load(piece_of(0), av[0]);
    float part[IW][R][NT][4];
    float ones[IW][NT][4];
    float2 cs[IW][R];  // c~ of rows (g, g + 8) for the blocks in flight
    float4 cz[IW][R];  // INT4 asymmetric: (s_g, s_g z_g, s_g8, s_g8 z_g8), z instead of s z for bf16
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int j = piece_of(i);
      if (i < 7) act_load(piece_of(i + 1), av[(i + 1) & 1]);
      const int blk = j / PB, pib = j % PB, si = (j / PB) % IW;  // block in chunk, piece in block, chain slot
      if (pib == 0) {
        // block bw = bwc + jb of the window: rows (g, g + 8) at byte
        // (bw * 8 + g) * 2 * SV of the buffer (see caddr)
        const int jb = j / PB;
        uint32_t off;
        if constexpr (GAPS) {
          // o >> 7 = bw >> 1 and o & 127 = (bw & 1) * 64 + 8 g; bwc is even for B <= 128
          off = B <= 128 ? coff + (uint32_t)((jb >> 1) * 256 + (jb & 1) * 64) : coff;
        } else {
          off = coff + (uint32_t)(jb * 16 * SV);
        }
#pragma unroll
        for (int rt = 0; rt < R; ++rt) {
          const uint32_t cra = cbs[rt][crd] + off;
          if constexpr (ASYM) cz[si][rt] = gv_lds128f(cra);
          else cs[si][rt] = gv_lds64f(cra);
        }
      }
      (void)blk;
#pragma unroll
      for (int e = 0; e < 2; ++e) {  // the two k-steps of piece j
#pragma unroll
        for (int rt = 0; rt < R; ++rt) {
          const uint32_t w0 = wq[rt][j >> 1][2 * (j & 1)], w1 = wq[rt][j >> 1][2 * (j & 1) + 1];
          const int j0 = 2 * e, j1 = j0 + 1;
          if constexpr (EXACT) {
            uint32_t a0, a1, a2, a3;
            const float2 e0 = gv_lut64f(gv_lut_addr(w0, j0, lb));
            const float2 e1 = gv_lut64f(gv_lut_addr(w1, j0, lb));
            const float2 e2 = gv_lut64f(gv_lut_addr(w0, j1, lb));
            const float2 e3 = gv_lut64f(gv_lut_addr(w1, j1, lb));
            if constexpr (ASYM) {
              // w^ = bf16((q - z) s): the integer difference is exact
              const float sx = cz[si][rt].x, zx = cz[si][rt].y, sy = cz[si][rt].z, zy = cz[si][rt].w;
              a0 = Dt<DA>::pack2(__fmul_rn(e0.x - zx, sx), __fmul_rn(e0.y - zx, sx));
              a1 = Dt<DA>::pack2(__fmul_rn(e1.x - zy, sy), __fmul_rn(e1.y - zy, sy));
              a2 = Dt<DA>::pack2(__fmul_rn(e2.x - zx, sx), __fmul_rn(e2.y - zx, sx));
              a3 = Dt<DA>::pack2(__fmul_rn(e3.x - zy, sy), __fmul_rn(e3.y - zy, sy));
            } else {
              const float2 c = cs[si][rt];
              a0 = Dt<DA>::pack2(__fmul_rn(c.x, e0.x), __fmul_rn(c.x, e0.y));
              a1 = Dt<DA>::pack2(__fmul_rn(c.y, e1.x), __fmul_rn(c.y, e1.y));
              a2 = Dt<DA>::pack2(__fmul_rn(c.x, e2.x), __fmul_rn(c.x, e2.y));
              a3 = Dt<DA>::pack2(__fmul_rn(c.y, e3.x), __fmul_rn(c.y, e3.y));
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              const uint4 &b = av[i & 1][nt];
              GvMma<DA>::run(acc[rt][nt], a0, a1, a2, a3, e ? b.z : b.x, e ? b.w : b.y);
            }
          } else {
            // fp16: the four lookups and the NT MMAs in one asm block
            uint32_t bb[NT][2];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              const uint4 &b = av[i & 1][nt];
              bb[nt][0] = e ? b.z : b.x;
              bb[nt][1] = e ? b.w : b.y;
            }
            const uint32_t x0 = gv_lut_addr(w0, j0, lb), x1 = gv_lut_addr(w1, j0, lb);
            const uint32_t x2 = gv_lut_addr(w0, j1, lb), x3 = gv_lut_addr(w1, j1, lb);
            if (pib == 0 && e == 0) GvLutMma<NT, false>::run(part[si][rt], x0, x1, x2, x3, bb);
            else GvLutMma<NT, true>::run(part[si][rt], x0, x1, x2, x3, bb);
          }
        }
        if constexpr (ASYM && !EXACT) {
          constexpr uint32_t O = GvMma<DA>::kOnes;
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const uint4 &b = av[i & 1][nt];
            if (pib == 0 && e == 0) GvMma<DA>::run0(ones[si][nt], O, O, O, O, e ? b.z : b.x, e ? b.w : b.y);
            else GvMma<DA>::run(ones[si][nt], O, O, O, O, e ? b.z : b.x, e ? b.w : b.y);
          }
        }
      }
      if (!EXACT && (pib == PB - 1 || (B > kGvChunk && j == 7))) {
        // the block (or, for blocks longer than a chunk, this chunk's part
        // of it) is complete: scale its partial by c~ (pieces past K have a
        // zero partial and a zero c~)
#pragma unroll
        for (int rt = 0; rt < R; ++rt)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
              if constexpr (ASYM) {
                const float4 c = cz[si][rt];
                const float sc = jj < 2 ? c.x : c.z, sz = jj < 2 ? c.y : c.w;
                acc[rt][nt][jj] = fmaf(sc, part[si][rt][nt][jj], acc[rt][nt][jj]);
                acc[rt][nt][jj] = fmaf(-sz, ones[si][nt][jj], acc[rt][nt][jj]);
              } else {
                const float2 c = cs[si][rt];
                acc[rt][nt][jj] = fmaf(jj < 2 ? c.x : c.y, part[si][rt][nt][jj], acc[rt][nt][jj]);
              }
            }
      }
    }
    // Release the stage after the MMAs, which consumed every value read from
    // it; __syncwarp orders all lanes' reads before lane 0's arrive.
    __syncwarp();
    gv_arrive_lane0(sempty(s), lane);
    if (++s == S) {
      s = 0;
      ph ^= 1u;
    }
    ++cq;
    if (cq < cpc.q1) continue;

    // ---- end of a tile piece: write its rows out, move to the next piece
    {
      const GvInfo &mt = info[cpc.mi];
      const int N = mt.N, nc = mt.n_chunks;
      const int r_tile = cpc.tile * TR + wrow;
      const int len = cpc.q1 - cpc.q0;
      if (len == nc) {
#pragma unroll
        for (int rt = 0; rt < R; ++rt)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int row = r_tile + rt * 16 + (j >> 1) * 8 + g;
              const int m = nt * 8 + 2 * tig + (j & 1);
              if (m < M && row < N) gv_store(mt.Y, p.y_dtype, (int64_t)m * N + row, acc[rt][nt][j]);
            }
      } else {
        // a partial tile: its rows go to this CTA's slot, then each 16-row
        // group is counted; the contributor that completes a group sums
        // every contributor's slot in CTA order and zeroes them
        const int role = cpc.u == wk.u0 ? 0 : 1;
        float *slot = p.slots + ((int64_t)(blockIdx.x * 2 + role) * TR + wrow + g) * MW + 2 * tig;
#pragma unroll
        for (int rt = 0; rt < R; ++rt) {
          if (r_tile + rt * 16 >= N) continue;  // no finisher reads (and zeroes) rows past N
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h)
              __stcg(reinterpret_cast<float2 *>(slot + (rt * 16 + h * 8) * MW + nt * 8),
                     make_float2(acc[rt][nt][2 * h], acc[rt][nt][2 * h + 1]));
        }
        gv_fence_acq_rel_gpu();
        __syncwarp();
        const uint32_t tile_u0 = mt.unit_begin + (uint32_t)cpc.tile * (uint32_t)nc;
#pragma unroll
        for (int rt = 0; rt < R; ++rt) {
          const int r_base = r_tile + rt * 16;
          if (r_base >= N) continue;
          unsigned old = 0;
          if (lane == 0) old = atomicAdd(mt.cnt + (r_base >> 4), (unsigned)len);
          old = __shfl_sync(0xffffffffu, old, 0);
          if (old + (unsigned)len != (unsigned)nc) continue;
          __syncwarp();
          gv_fence_acq_rel_gpu();
          const int c0 = gv_cta_of(tile_u0, T, G), c1 = gv_cta_of(tile_u0 + (uint32_t)nc - 1, T, G);
          float sum[NT][4];
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 4; ++j) sum[nt][j] = 0.0f;
#pragma unroll 1
          for (int c = c0; c <= c1; ++c) {
            const int rl = gv_begin((uint32_t)c, T, G) >= tile_u0 ? 0 : 1;
            float *sl = p.slots + ((int64_t)(c * 2 + rl) * TR + wrow + rt * 16 + g) * MW + 2 * tig;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                float2 *q = reinterpret_cast<float2 *>(sl + (h * 8) * MW + nt * 8);
                const float2 v = __ldcg(q);
                __stcg(q, make_float2(0.0f, 0.0f));  // the workspace is left zeroed
                sum[nt][2 * h] += v.x;
                sum[nt][2 * h + 1] += v.y;
              }
          }
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int row = r_base + (j >> 1) * 8 + g;
              const int m = nt * 8 + 2 * tig + (j & 1);
              if (m < M && row < N) gv_store(mt.Y, p.y_dtype, (int64_t)m * N + row, sum[nt][j]);
            }
          if (lane == 0) mt.cnt[r_base >> 4] = 0u;
        }
      }
#pragma unroll
      for (int rt = 0; rt < R; ++rt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[rt][nt][j] = 0.0f;
      if (left > 1) {
        GvPiece nx;
        gv_piece_next(info, count, wk, cpc, nx);
        cpc = nx;
        cq = nx.q0;
        c_setup();
      }
    }
  }
  (void)ok;
}

}  // namespace q4
