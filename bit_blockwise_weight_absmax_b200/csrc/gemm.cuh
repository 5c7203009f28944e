// gemm.cuh -- W4A16 GEMM for prefill on tcgen05 tensor cores (sm_100a):
// Y[M,N] = A[M,K] . W^[N,K]^T with W^ the 16-bit dequantized NF4 weights.
//
// What it computes: learn.pranaymahendrakar.com, "Loading a model in 4-bit",
// "Where the accuracy goes" (Linear4bit dequantises the weights to the compute
// dtype and runs a standard 16-bit GEMM) and mbrenndoerfer.com, "INT4
// Quantization > Practical Implementation with bitsandbytes" (weights stored
// in 4 bits, dequantized to 16 bits before the matmul).  Each weight tile is
// dequantized exactly as q4_dequantize does (bit-exact w^ = cvt(c~ * level))
// into shared memory and consumed there by the tensor cores, so the 16-bit
// weight matrix never exists in HBM.
//
// Design (one CTA per SM, persistent over output tiles of 128 weight rows
// by 512 tokens -- or 256 tokens for launches of few tiles, a template
// parameter the host picks -- m-tiles fastest so that neighbouring CTAs
// share a weight tile in L2):
//   warp 0      TMA producer: the raw packed tile [128 rows x 32 bytes] of
//               each 64-k block into a ring of 4 dequant stages, and the
//               activation tile in 256-token halves [256 x 64] (128B-
//               swizzled, K-major) into a ring of 4 slots; the raw codes
//               run two k-blocks ahead of the activations (tall tiles).
//   warp 1      TMEM allocator and MMA issuer: per k-block and token half
//               4 tcgen05.mma kind::f16 (M=128 weight rows, N=256 tokens,
//               K=16), both halves reading the same dequantized weight
//               stage, into a 512-column fp32 accumulator (a TMEM lane per
//               weight row, a column per token).  256-token tiles use two
//               256-column accumulators that alternate between tiles, so an
//               epilogue overlaps the next tile's MMAs.  With the weight
//               tile on the M side each MMA reads 12 KB of shared memory
//               for 128 tensor cycles (two N=128 MMAs over token halves
//               would read 16 KB), and shared-memory bandwidth is what the
//               MMAs, the copies and the dequant stores share; a tall tile
//               also halves the dequant work per flop.
//   warps 2..17 dequant: four threads per weight row, 16 codes each, scaled
//               by the row's block scale into bf16/fp16 and written in the
//               128B-swizzled K-major layout the UMMA descriptor reads; the
//               block scales come 16 blocks per load.  Then the epilogue:
//               tcgen05.ld of the accumulator (a lane per weight row, 16
//               tokens at a time), convert, store one token row's 32
//               consecutive outputs per warp instruction.
// Every mbarrier wait is bounded in time; a timeout sets Q4_STATUS_TIMEOUT,
// stops the pipeline, waits for issued copies and for the issued MMAs, and
// frees TMEM.
#pragma once
#include <cuda.h>

#include "q4_common.cuh"

namespace q4 {

constexpr int kGemmBM = 512;      // tokens per tile (at most; a launch may use tiles of kGemmHalfM)
constexpr int kGemmHalfM = 256;   // tokens per MMA (UMMA N) and per activation slot
constexpr int kGemmBN = 128;      // weight rows per tile (UMMA M)
constexpr int kGemmBK = 64;
constexpr int kGemmStages = 4;    // ring of dequant stages (raw codes in, 16-bit weight tile out)
constexpr int kGemmASlots = 4;    // ring of activation half tiles (two per k-block)
constexpr int kGemmDqWarps = 16;                          // dequant + epilogue warps (2..17)
constexpr int kGemmThreads = (2 + kGemmDqWarps) * 32;
constexpr int kGemmATile = kGemmHalfM * kGemmBK * 2;  // 32 KB: one activation half tile
constexpr int kGemmBTile = kGemmBN * kGemmBK * 2;     // 16 KB
constexpr int kGemmRawTile = kGemmBN * kGemmBK / 2;   // 4 KB
constexpr int kGemmScBytes = kGemmBN * 16 * 4;       // c~ of 16 blocks per weight row
constexpr int kGemmTpr = kGemmDqWarps * 32 / kGemmBN;  // dequant threads per weight row
constexpr int kGemmCodes = kGemmBK / kGemmTpr;      // codes per thread and stage
// Per tile height (TALL: kGemmBM tokens, else kGemmHalfM):
//  - accumulators in TMEM's 512 columns: one, or two that alternate so that
//    an epilogue overlaps the next tile's MMAs;
//  - the epilogue of a tile runs after this many dequant stages of the
//    next: with two accumulators a ring's worth (its stores overlap the
//    MMAs of those stages); with one two stages, about when the MMAs of its
//    tile end, so that they find the next stages ready;
//  - raw codes are issued this many k-blocks ahead of the activations: the
//    activation ring holds two k-blocks of tall tiles and four of low ones,
//    the raw ring four, so the lead evens the two rings' look-ahead.
template <bool TALL> struct GemmShape {
  static constexpr int kTileM = TALL ? kGemmBM : kGemmHalfM;
  static constexpr int kSets = TALL ? 1 : 2;
  static constexpr int kEpiAfter = TALL ? 2 : kGemmStages;
  static constexpr int kRawLead = TALL ? 2 : 0;
  static_assert(kSets * kTileM <= 512 && kRawLead < kGemmStages, "TMEM columns, raw ring");
};
static_assert(kGemmBN == 128 && kGemmHalfM % 16 == 0 && kGemmHalfM <= 256, "UMMA M = 128 (weight rows), N = tokens");
static_assert(kGemmBM == 2 * kGemmHalfM && kGemmBM <= 512, "one accumulator of kGemmBM (or two of kGemmHalfM) TMEM columns");
static_assert(kGemmCodes == 16 || kGemmCodes == 32, "8 or 16 packed bytes per thread");
constexpr int kGemmSmem = kGemmASlots * kGemmATile + kGemmStages * (kGemmBTile + kGemmRawTile) + kGemmScBytes +
                          1024 /*align*/ + 256 /*barriers*/;

struct alignas(64) GemmMat {
  CUtensorMap tmA;  // A [M, K] 16-bit, box {64, 256}, 128B swizzle
  CUtensorMap tmW;  // packed [N, K/2] bytes, box {32, 128}
  const uint8_t *zero;  // INT4 asymmetric zero-points, two per byte
  const int8_t *absmax_q;
  const float *absmax_scale;
  const float *absmax_mean;
  const float *absmax;
  void *Y;
  int64_t tile_begin;
  int32_t M, N, K;
  int32_t tiles_m, tiles_n;
  int32_t pad;
};

// Up to this many work items a launch carries an explicit item list per
// CTA, balanced on the host by the k-blocks of each item (longest first onto
// the least loaded CTA); above it whole tiles are dealt round robin, which
// is then within a few percent of even.  An item is a whole tile or one
// half of a tile's k range (split-K): both halves write their fp32
// partials to the workspace and the second to finish adds the other's and
// writes Y.  Item encoding: bits 0-15 tile, 16-17 half (0 whole, 1 first,
// 2 second), 18-31 split slot.
constexpr int kGemmListTiles = 2048;
constexpr int kGemmGroupM = 4;  // m-tiles per group of a round-robin launch
constexpr int kGemmListCtas = 256;  // grid bound of a listed launch
constexpr int kGemmSplitWarpFloats = kGemmBM / 4 * 32;  // one epilogue warp's partial: its columns x lanes
constexpr size_t kGemmSplitSlotBytes = 2 * 16 * kGemmSplitWarpFloats * sizeof(float);  // two halves x 16 warps
// The arrival counters sit at the start of the workspace in a region of a
// fixed size (every slot a listed launch can have), so that whatever slot
// count the previous call used, they are the zeroed words it left.
constexpr size_t kGemmSplitCntBytes = (size_t)(kGemmListTiles / 2) * 16 * sizeof(unsigned);

struct GemmParams {
  GemmMat mat[16];
  int32_t count;
  int32_t y_dtype;
  int32_t dq;
  int32_t stall_copies;  // test hook: the producer issues no copies
  int32_t log2_bs;       // blocksize B = 2^log2_bs (32 .. 256)
  int32_t scale_f16;     // INT4: binary16 scales
  int64_t total_tiles;
  uint64_t wait_ns;      // bound of every mbarrier wait
  int *status;
  float levels[16];
  int32_t listed;        // items come from tile_list (else whole tiles round robin)
  int32_t tile_m;        // tokens per tile: kGemmBM (one accumulator) or kGemmHalfM (two, alternating); picks the instance
  int32_t grid;          // CTAs of the launch
  unsigned *split_cnt;   // split-K: [slot][epilogue warp] arrivals (zero between calls), at the workspace start
  float *partials;       // split-K: [slot][half][epilogue warp][kGemmSplitWarpFloats] fp32, after the counters
  uint16_t cta_off[kGemmListCtas + 1];  // CTA c runs tile_list[cta_off[c] .. cta_off[c + 1])
  uint32_t tile_list[kGemmListTiles];
};

// ---- PTX wrappers ------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("{ .reg .b64 st; mbarrier.arrive.shared::cta.b64 st, [%0]; }" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("{ .reg .b64 st; mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1; }" ::"r"(bar),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Bounded wait: gives up after `limit_ns` (2 s unless the launch sets a
// limit), raises Q4_STATUS_TIMEOUT and sets *abort.  The first probe is
// inlined; only a phase that is not yet complete pays the call into the
// polling loop.  A warp that waits for long (a copy warp ahead of its
// consumers, a reducer between chunks) passes `sleep_ns` > 0: it sleeps
// between probes instead of taking issue slots from the working warps of
// its scheduler.
constexpr uint64_t kWaitLimitNs = 2000000000ull;
static __device__ __noinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity, int *status,
                                                   volatile int *abort, uint64_t limit_ns, uint32_t sleep_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try(bar, parity)) return true;
    if (*abort) return false;
    if (globaltimer_ns() - t0 > limit_ns) {
      raise_status(status, Q4_STATUS_TIMEOUT);
      *abort = 1;
      return false;
    }
    if (sleep_ns) __nanosleep(sleep_ns);
  }
}
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, int *status, volatile int *abort,
                                          uint64_t limit_ns = kWaitLimitNs, uint32_t sleep_ns = 0) {
  if (mbar_try(bar, parity)) return true;
  return mbar_wait_slow(bar, parity, status, abort, limit_ns, sleep_ns);
}

// Wait by a whole warp: only lane 0 polls the barrier (many polling lanes
// would queue their try_waits ahead of the single-thread producers), then
// the result is broadcast.  Must be called by all 32 lanes.
// After lane 0 has seen the phase complete, each other lane queries it once
// (returns at once) so that it acquires the data the phase published itself.
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity, int *status, volatile int *abort,
                                               uint64_t limit_ns = kWaitLimitNs, uint32_t sleep_ns = 0) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, status, abort, limit_ns, sleep_ns);
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  if (ok && (threadIdx.x & 31) != 0) (void)mbar_try(bar, parity);
  return ok;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, uint32_t bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(map), "r"(bar), "r"(x), "r"(y)
      : "memory");
}

// Fetches a tensor map (a kernel parameter) into the descriptor cache ahead
// of its first copy.
__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(m) : "memory");
}

__device__ __forceinline__ float lds_f32(uint32_t addr) {
  float v;
  asm("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// K-major operand tile with 128-byte swizzle: 8-row atoms of 1024 bytes
// (stride byte offset 1024), leading byte offset unused (1), descriptor
// version 1, layout type 2 (SWIZZLE_128B).  `addr` is the shared-memory byte
// address of the first row, advanced by 32 bytes per 16-element k-step.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;                 // leading byte offset (ignored for swizzled K-major)
  d |= (uint64_t)(1024u >> 4) << 32;       // stride byte offset
  d |= (uint64_t)1u << 46;                 // descriptor version (sm100)
  d |= (uint64_t)2u << 61;                 // SWIZZLE_128B
  return d;
}

// Instruction descriptor, kind::f16: D fp32, A/B = fp16 (0) or bf16 (1),
// both K-major, N >> 3 at bit 17, M >> 4 at bit 24.
__host__ __device__ constexpr uint32_t umma_idesc_f16(int ab_bf16, int M, int N) {
  return (1u << 4) | ((uint32_t)ab_bf16 << 7) | ((uint32_t)ab_bf16 << 10) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %4, 0; "
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }" ::"r"(tmem_d),
      "l"(da), "l"(db), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// 32 lanes x 32 consecutive fp32 columns of TMEM -> 32 registers per thread.
// 16 fp32 accumulator columns of this warp's 32 TMEM lanes (one lane per
// thread); 16 at a time keeps the epilogue within the kernel's registers.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

struct TileCoord {
  int mi, tm, tn;
  int kb0, kb1;  // the k-blocks of this item
  int slot;      // split-K slot (-1: a whole tile)
  int half;      // split-K half (0, 1)
};
// Work item v: an encoded list item when the launch is listed, else a
// whole tile index.
__device__ __forceinline__ TileCoord gemm_tile(const GemmParams &p, int64_t v) {
  const int64_t t = p.listed ? (int64_t)(v & 0xFFFF) : v;
  const int hc = p.listed ? (int)((v >> 16) & 3) : 0;
  int mi = 0;
  while (mi + 1 < p.count && t >= p.mat[mi + 1].tile_begin) ++mi;
  const int64_t local = t - p.mat[mi].tile_begin;
  const int tm_count = p.mat[mi].tiles_m;
  const int nk = p.mat[mi].K / kGemmBK;
  // m-tiles fastest: consecutive CTAs share one weight tile (read once from
  // HBM).  Launches dealt round robin (too many tiles for a list: large M)
  // go through the m-tiles kGemmGroupM at a time, so that the CTAs running
  // at once share a few activation m-tiles in L2 instead of streaming all
  // of them (at M = 8192 the down projection's activations are 180 MB).
  int tm = (int)(local % tm_count), tn = (int)(local / tm_count);
  if (!p.listed && tm_count > kGemmGroupM) {
    const int64_t per_group = (int64_t)kGemmGroupM * p.mat[mi].tiles_n;
    const int64_t g = local / per_group, r = local % per_group;
    const int gm = min(kGemmGroupM, tm_count - (int)g * kGemmGroupM);
    tm = (int)g * kGemmGroupM + (int)(r % gm);
    tn = (int)(r / gm);
  }
  TileCoord tc{mi, tm, tn, 0, nk, -1, 0};
  if (hc != 0) {
    tc.half = hc - 1;
    tc.slot = (int)(v >> 18);
    tc.kb0 = tc.half == 0 ? 0 : nk / 2;
    tc.kb1 = tc.half == 0 ? nk / 2 : nk;
  }
  return tc;
}

// Epilogue helpers.  A dequant warp's share of a tile of TM tokens: TMEM
// lanes q * 32 .. + 31 (its quadrant: weight rows q * 32 .. + 31 of the
// tile) and the accumulator's token columns cc * TM / 4 .. + TM / 4 - 1, in
// TM / 64 chunks of 16.
template <int TM>
__device__ __forceinline__ uint32_t gemm_chunk(uint32_t tmem, int ab, int ch, int q, int cc, int &t16) {
  t16 = cc * (TM / 4) + 16 * ch;
  return tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(ab * TM + t16);
}
static_assert(kGemmBM / 64 * 32 * 16 == kGemmSplitWarpFloats, "split-K partial layout");
// Token halves of tile tm that hold any of the M tokens (the second half of
// the last tall tile may lie wholly past M: it is neither loaded nor
// multiplied).
template <bool TALL> __device__ __forceinline__ int gemm_halves(const GemmMat &m, int tm) {
  return TALL && tm * kGemmBM + kGemmHalfM < m.M ? 2 : 1;
}
// Y[t0 .. t0 + 15, n] of one lane (its weight row n) from 16 fp32
// accumulators; the warp's 32 lanes are 32 consecutive n, so each store
// instruction writes one contiguous run of a Y row.
__device__ __forceinline__ void gemm_store_y(const GemmMat &m, int y_dtype, int n, int t0, const uint32_t (&r)[16]) {
  if (n >= m.N || t0 >= m.M) return;
  const int nt = min(16, m.M - t0);
  if (y_dtype == Q4_F32) {
    float *y = reinterpret_cast<float *>(m.Y) + (int64_t)t0 * m.N + n;
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (j < nt) y[(int64_t)j * m.N] = __uint_as_float(r[j]);
  } else {
    uint16_t *y = reinterpret_cast<uint16_t *>(m.Y) + (int64_t)t0 * m.N + n;
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (j < nt)
        y[(int64_t)j * m.N] = (y_dtype == Q4_BF16) ? Dt<Q4_BF16>::from_f(__uint_as_float(r[j]))
                                                   : Dt<Q4_F16>::from_f(__uint_as_float(r[j]));
  }
}
// Split-K epilogue of one warp's share of a cut tile.  The half's fp32 partial is published, then counted; the warp that
// completes the count adds the other half's partial (a + b: the same bits
// whichever half finishes second), writes Y and zeroes the counter.
template <bool TALL>
static __device__ __forceinline__ void gemm_split_epilogue(const GemmParams *pp, uint32_t tmem, int ab, int mi, int tm,
                                                        int tn, int slot, int half, int q, int cc, int lane, int wp) {
  const GemmParams &p = *pp;
  const GemmMat &m = p.mat[mi];
  float *mine = p.partials + ((int64_t)(slot * 2 + half) * 16 + wp) * kGemmSplitWarpFloats;
  constexpr int TM = GemmShape<TALL>::kTileM, nch = TM / 64;
  const int ncols = gemm_halves<TALL>(m, tm) * kGemmHalfM;  // accumulator columns the tile filled
#pragma unroll 1
  for (int ch = 0; ch < nch; ++ch) {
    int t16;
    uint32_t r[16];
    const uint32_t ta = gemm_chunk<TM>(tmem, ab, ch, q, cc, t16);
    if (t16 >= ncols) break;
    tmem_ld16(ta, r);
    float4 *dst = reinterpret_cast<float4 *>(mine + (ch * 32 + lane) * 16);
#pragma unroll
    for (int v = 0; v < 4; ++v)
      __stcg(dst + v, make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                                  __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3])));
  }
  __threadfence();  // this lane's partial is visible before its count
  __syncwarp();
  unsigned old = 0;
  if (lane == 0) old = atomicAdd(p.split_cnt + slot * 16 + wp, 1u);
  old = __shfl_sync(0xffffffffu, old, 0);
  if (old != 1) return;  // the other half will finish the tile
  __threadfence();
  const float *other = p.partials + ((int64_t)(slot * 2 + (1 - half)) * 16 + wp) * kGemmSplitWarpFloats;
#pragma unroll 1
  for (int ch = 0; ch < nch; ++ch) {
    int t16;
    uint32_t r[16];
    const uint32_t ta = gemm_chunk<TM>(tmem, ab, ch, q, cc, t16);
    if (t16 >= ncols) break;
    tmem_ld16(ta, r);
    const float4 *src = reinterpret_cast<const float4 *>(other + (ch * 32 + lane) * 16);
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const float4 o = __ldcg(src + v);
      r[4 * v] = __float_as_uint(__uint_as_float(r[4 * v]) + o.x);
      r[4 * v + 1] = __float_as_uint(__uint_as_float(r[4 * v + 1]) + o.y);
      r[4 * v + 2] = __float_as_uint(__uint_as_float(r[4 * v + 2]) + o.z);
      r[4 * v + 3] = __float_as_uint(__uint_as_float(r[4 * v + 3]) + o.w);
    }
    gemm_store_y(m, p.y_dtype, tn * kGemmBN + q * 32 + lane, tm * TM + t16, r);
  }
  if (lane == 0) p.split_cnt[slot * 16 + wp] = 0u;  // the workspace is left zeroed
}

// Block-scale modes of the GEMM: absmax as stored (NF4, INT4 symmetric),
// double-quantized (NF4), or scale plus zero-point (INT4 asymmetric).
constexpr int kGemmPlain = 0, kGemmDq = 1, kGemmAsym = 2;

// DA: activation dtype; MODE: block-scale mode; SPLIT: the launch has cut
// tiles (the instance without them carries no split-K code, so its
// registers do not spill).  The blocksize is a launch parameter: it only
// decides which block scale a thread's 16 codes take.
template <int DA, int MODE, bool SPLIT, bool TALL>
__global__ void __launch_bounds__(kGemmThreads, 1) gemm_kernel(const __grid_constant__ GemmParams p) {
  constexpr bool DQ = MODE == kGemmDq, ASYM = MODE == kGemmAsym;
  using Sh = GemmShape<TALL>;
  pdl_launch_dependents();  // set-up (barriers, TMEM, level table) overlaps the previous kernel
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t *sA = smem;                                        // [activation slots][32 KB]
  uint8_t *sB = smem + kGemmASlots * kGemmATile;             // [stages][16 KB]
  uint8_t *sR = sB + kGemmStages * kGemmBTile;               // [stages][4 KB]
  float *sSc = reinterpret_cast<float *>(sR + kGemmStages * kGemmRawTile);  // [128 rows][16]
  uint64_t *bars = reinterpret_cast<uint64_t *>(reinterpret_cast<uint8_t *>(sSc) + kGemmScBytes);
  // bars: full[S], bfull[S], empty[S], accfull[2], accempty[2], afull[AS], aempty[AS]
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ float s_lv[16 * 32];
  __shared__ __align__(16) uint8_t s_z[ASYM ? kGemmBN * 16 : 4];  // zero-points of each row's window

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto bfull_bar = [&](int s) { return bar0 + 8u * (kGemmStages + s); };
  auto empty_bar = [&](int s) { return bar0 + 8u * (2 * kGemmStages + s); };
  auto accfull_bar = [&](int b) { return bar0 + 8u * (3 * kGemmStages + b); };
  auto accempty_bar = [&](int b) { return bar0 + 8u * (3 * kGemmStages + 2 + b); };
  auto afull_bar = [&](int a) { return bar0 + 8u * (3 * kGemmStages + 4 + a); };
  auto aempty_bar = [&](int a) { return bar0 + 8u * (3 * kGemmStages + 4 + kGemmASlots + a); };
  static_assert(8 * (3 * kGemmStages + 4 + 2 * kGemmASlots) <= 256, "barrier area");

  if (tid == 0) {
    for (int s = 0; s < kGemmStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(bfull_bar(s), kGemmDqWarps);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accfull_bar(b), 1);
      mbar_init(accempty_bar(b), kGemmDqWarps);
    }
    for (int a = 0; a < kGemmASlots; ++a) {
      mbar_init(afull_bar(a), 1);
      mbar_init(aempty_bar(a), 1);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    s_abort = 0;
  }
  for (int i = tid; i < 16 * 32; i += kGemmThreads) s_lv[i] = p.levels[i >> 5];
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (warp == 0 && lane < p.count) {
    prefetch_tensormap(&p.mat[lane].tmA);
    prefetch_tensormap(&p.mat[lane].tmW);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();
  const uint32_t tmem = s_tmem;
  volatile int *abort = &s_abort;
  // this CTA's tiles: a host-balanced list, or every gridDim.x-th tile
  const int64_t n_my = p.listed ? (int64_t)(p.cta_off[blockIdx.x + 1] - p.cta_off[blockIdx.x])
                                : (p.total_tiles - blockIdx.x + gridDim.x - 1) / gridDim.x;
  auto my_tile = [&](int64_t k) -> int64_t {
    return p.listed ? (int64_t)p.tile_list[p.cta_off[blockIdx.x] + k] : (int64_t)blockIdx.x + k * gridDim.x;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      // Two cursors over this CTA's (item, k-block) sequence: the raw codes
      // run kGemmRawLead k-blocks ahead of the activation halves, so that a
      // stage's codes land and are dequantized while the MMAs still work on
      // earlier k-blocks (the activation ring holds two k-blocks).
      struct Cur {
        int64_t k;  // item index; n_my when the sequence is exhausted
        int kb;
        TileCoord tc;
      };
      auto cur_init = [&](Cur &c) {
        c.k = 0;
        c.kb = 0;
        if (n_my > 0) {
          c.tc = gemm_tile(p, my_tile(0));
          c.kb = c.tc.kb0;
        }
      };
      auto cur_next = [&](Cur &c) {
        if (++c.kb == c.tc.kb1 && ++c.k < n_my) {
          c.tc = gemm_tile(p, my_tile(c.k));
          c.kb = c.tc.kb0;
        }
      };
      Cur cr, ca;
      cur_init(cr);
      cur_init(ca);
      uint32_t it = 0, ia = 0;  // dequant stages and activation half tiles issued
      auto issue_raw = [&]() -> bool {
        const int s = it % kGemmStages;
        if (!mbar_wait(empty_bar(s), ((it / kGemmStages) & 1) ^ 1, p.status, abort, p.wait_ns)) return false;
        if (!p.stall_copies) {  // test hook: no stage is ever filled
          mbar_arrive_expect_tx(full_bar(s), kGemmRawTile);
          tma_load_2d(smem_u32(sR + s * kGemmRawTile), &p.mat[cr.tc.mi].tmW, full_bar(s), cr.kb * (kGemmBK / 2),
                      cr.tc.tn * kGemmBN);
        }
        ++it;
        cur_next(cr);
        return true;
      };
      bool ok = true;
      for (int j = 0; j < Sh::kRawLead && cr.k < n_my && ok; ++j) ok = issue_raw();
      while (ok && ca.k < n_my && !*abort) {
        if (cr.k < n_my && !(ok = issue_raw())) break;
        const GemmMat &m = p.mat[ca.tc.mi];
        const int nh = gemm_halves<TALL>(m, ca.tc.tm);
        for (int h = 0; h < nh; ++h) {
          const int a = ia % kGemmASlots;
          if (!mbar_wait(aempty_bar(a), ((ia / kGemmASlots) & 1) ^ 1, p.status, abort, p.wait_ns)) {
            ok = false;
            break;
          }
          if (!p.stall_copies) {
            mbar_arrive_expect_tx(afull_bar(a), kGemmATile);
            tma_load_2d(smem_u32(sA + a * kGemmATile), &m.tmA, afull_bar(a), ca.kb * kGemmBK,
                        ca.tc.tm * Sh::kTileM + h * kGemmHalfM);
          }
          ++ia;
        }
        cur_next(ca);
      }
      // every issued copy completes before the CTA may exit (only the last
      // use of each ring slot can still be in flight)
      for (uint32_t j = (it > kGemmStages ? it - kGemmStages : 0); j < it && !p.stall_copies; ++j) {
        int dummy = 0;
        volatile int no_abort = 0;
        mbar_wait(full_bar(j % kGemmStages), (j / kGemmStages) & 1, &dummy, &no_abort);
      }
      for (uint32_t j = (ia > kGemmASlots ? ia - kGemmASlots : 0); j < ia && !p.stall_copies; ++j) {
        int dummy = 0;
        volatile int no_abort = 0;
        mbar_wait(afull_bar(j % kGemmASlots), (j / kGemmASlots) & 1, &dummy, &no_abort);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // M = 128 weight rows (the dequantized tile), N = kGemmHalfM tokens;
      // both token halves of a k-block multiply the same weight stage
      const uint32_t idesc = umma_idesc_f16(DA == Q4_BF16 ? 1 : 0, kGemmBN, kGemmHalfM);
      uint32_t it = 0, ia = 0, tcount = 0;
      uint32_t last_bar = 0, last_par = 0;  // the barrier and phase of the last commit issued
      bool committed = false, ok = true;
      for (int64_t k = 0; k < n_my && ok && !*abort; ++k, ++tcount) {
        const TileCoord tc = gemm_tile(p, my_tile(k));
        const int nh = gemm_halves<TALL>(p.mat[tc.mi], tc.tm);
        const int ab = tcount % Sh::kSets;  // accumulator of this tile
        const uint32_t aph = (tcount / Sh::kSets) & 1;
        if (!mbar_wait(accempty_bar(ab), aph ^ 1, p.status, abort, p.wait_ns)) break;
        tc_fence_after();
        for (int kb = tc.kb0; kb < tc.kb1 && ok; ++kb) {
          const int s = it % kGemmStages;
          const uint32_t use = it / kGemmStages;
          if (!mbar_wait(bfull_bar(s), use & 1, p.status, abort, p.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t b0 = smem_u32(sB + s * kGemmBTile);
          for (int h = 0; h < nh; ++h) {
            const int a = ia % kGemmASlots;
            const uint32_t ause = ia / kGemmASlots;
            if (!mbar_wait(afull_bar(a), ause & 1, p.status, abort, p.wait_ns)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t a0 = smem_u32(sA + a * kGemmATile);
            const uint32_t d = tmem + (uint32_t)(ab * Sh::kTileM + h * kGemmHalfM);
#pragma unroll
            for (int k16 = 0; k16 < kGemmBK / 16; ++k16)
              umma_f16(d, umma_desc_sw128(b0 + 32 * k16), umma_desc_sw128(a0 + 32 * k16), idesc,
                       kb != tc.kb0 || k16 != 0);
            umma_commit(aempty_bar(a));
            last_bar = aempty_bar(a), last_par = ause & 1, committed = true;
            ++ia;
          }
          if (!ok) break;
          umma_commit(empty_bar(s));
          last_bar = empty_bar(s), last_par = use & 1, committed = true;
          ++it;
        }
        if (!ok) break;
        umma_commit(accfull_bar(ab));
        last_bar = accfull_bar(ab), last_par = aph, committed = true;
      }
      // Every MMA issued completes before the CTA may free its TMEM, also
      // after a timeout: a commit's arrival covers all earlier MMAs of this
      // thread, so waiting for the last one is enough (nothing else arrives
      // on that barrier phase, so it completes).
      if (committed) {
        int dummy = 0;
        volatile int no_abort = 0;
        mbar_wait(last_bar, last_par, &dummy, &no_abort);
      }
    }
  } else {
    // ------------------------------------------------------------ dequant + epilogue
    const int dt = tid - 64;           // 0..511
    const int d = dt / kGemmTpr;       // weight row within the tile
    const int qk = dt % kGemmTpr;      // part of the 64-k block: codes kGemmCodes qk .. + kGemmCodes - 1
    const int q = warp & 3;            // TMEM lane quadrant of this warp
    const int cc = (warp - 2) >> 2;    // quarter of the accumulator columns handled in the epilogue
    const uint32_t lvb = smem_u32(s_lv) + 4u * lane;
    // epilogue of a finished item: its accumulator set -> Y
    // (the MMAs of the next item go to the other accumulator set meanwhile)
    const int wp = warp - 2;  // this warp's share of a tile's accumulators: 0..15
    auto epilogue = [&](int64_t item, uint32_t tcount) -> bool {
      const TileCoord tc = gemm_tile(p, item);  // decoded again: one word stays live across the loop
      const int ab = tcount % Sh::kSets;
      if (!mbar_wait_warp(accfull_bar(ab), (tcount / Sh::kSets) & 1, p.status, abort, p.wait_ns)) return false;
      tc_fence_after();
      if (SPLIT && tc.slot >= 0) {
        if constexpr (SPLIT) gemm_split_epilogue<TALL>(&p, tmem, ab, tc.mi, tc.tm, tc.tn, tc.slot, tc.half, q, cc, lane, wp);
      } else {
        const GemmMat &m = p.mat[tc.mi];
        constexpr int TM = Sh::kTileM, nch = TM / 64;
        const int ncols = gemm_halves<TALL>(m, tc.tm) * kGemmHalfM;
#pragma unroll 1
        for (int ch = 0; ch < nch; ++ch) {
          int t16;
          uint32_t r[16];
          const uint32_t ta = gemm_chunk<TM>(tmem, ab, ch, q, cc, t16);
          if (t16 >= ncols) break;
          tmem_ld16(ta, r);
          gemm_store_y(m, p.y_dtype, tc.tn * kGemmBN + q * 32 + lane, tc.tm * TM + t16, r);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(accempty_bar(ab));
      return true;
    };
    bool have_prev = false;
    int64_t prev_item = 0;
    uint32_t prev_count = 0;
    uint32_t it = 0, tcount = 0;
    for (int64_t k = 0; k < n_my && !*abort; ++k, ++tcount) {
      const int64_t item = my_tile(k);
      const TileCoord tc = gemm_tile(p, item);
      const GemmMat &m = p.mat[tc.mi];
      const int lbs = p.log2_bs;
      const int nblk = m.K >> lbs;  // blocks per weight row
      const int row = tc.tn * kGemmBN + d;
      const bool row_ok = row < m.N;
      const float mu = (DQ && row_ok) ? __ldg(m.absmax_mean) : 0.0f;
      const int64_t bi0 = (int64_t)min(row, m.N - 1) * nblk;
      // block scales: the c~ (and zero-points) of a window of 16 blocks of
      // the row at a time, computed by the row's four threads (four blocks
      // each) from inputs requested a window ahead, kept in shared memory
      // for the row
      struct In4 {
        uint32_t cw;     // int8 codes of four blocks (double quant) / their zero-points (asymmetric)
        float s2a, s2b;  // second-level scales of their (at most two) 256-groups
        int bsplit;
        float f[4];      // fp32 absmax (no double quant)
      };
      auto load4 = [&](int b0, In4 &o) {  // blocks b0 .. b0 + 3 of the row
        const int nv = max(0, min(4, nblk - b0));
        const int64_t bi = bi0 + b0;
        o.cw = 0;
        o.s2a = o.s2b = 0.0f;
        o.bsplit = 4;
        o.f[0] = o.f[1] = o.f[2] = o.f[3] = 0.0f;
        if (nv == 0) return;
        if constexpr (DQ) {
          o.s2a = __ldg(m.absmax_scale + (bi >> 8));
          o.s2b = __ldg(m.absmax_scale + ((bi + nv - 1) >> 8));
          o.bsplit = (int)min((int64_t)4, (((bi >> 8) + 1) << 8) - bi);
          if (nv == 4 && (bi & 3) == 0) {
            o.cw = __ldg(reinterpret_cast<const unsigned *>(m.absmax_q + bi));
          } else {
            uint32_t w = 0;
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (e < nv) w |= (uint32_t)(uint8_t)__ldg(m.absmax_q + bi + e) << (8 * e);
            o.cw = w;
          }
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) o.f[e] = e < nv ? ld_scale(m.absmax, bi + e, p.scale_f16 != 0) : 0.0f;
          if constexpr (ASYM) {
            uint32_t w = 0;
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (e < nv) w |= ((uint32_t)(__ldg(m.zero + ((bi + e) >> 1)) >> (((bi + e) & 1) * 4)) & 15u) << (8 * e);
            o.cw = w;
          }
        }
      };
      float *scrow = sSc + d * 16;
      uint8_t *zrow = s_z + (ASYM ? d * 16 : 0);
      auto store4 = [&](const In4 &o) {  // this thread's four blocks of the window
        float v[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if constexpr (DQ) {
            const int code = (int)(int8_t)((o.cw >> (8 * e)) & 0xFFu);
            v[e] = __fadd_rn(__fmul_rn((float)code, e < o.bsplit ? o.s2a : o.s2b), mu);
          } else {
            v[e] = o.f[e];
          }
          if (!row_ok) v[e] = 0.0f;
        }
        *reinterpret_cast<float4 *>(scrow + 4 * qk) = make_float4(v[0], v[1], v[2], v[3]);
        if constexpr (ASYM) *reinterpret_cast<uint32_t *>(zrow + 4 * qk) = o.cw;
      };
      // the window of 16 blocks holding the item's first k-block
      const int w0 = ((tc.kb0 * kGemmBK) >> lbs) & ~15;
      In4 nin;
      {
        In4 cin;
        load4(w0 + 4 * qk, cin);
        load4(w0 + 16 + 4 * qk, nin);  // zeros past the row's end
        __syncwarp();  // the row's previous c~ have been read
        store4(cin);
        __syncwarp();
      }
      int wnext = w0 + 16;  // first block of the window held in nin
      bool ok = true;
      for (int kb = tc.kb0; kb < tc.kb1; ++kb, ++it) {
        const int s = it % kGemmStages;
        const uint32_t use = it / kGemmStages;
        const int kk = kb * kGemmBK;
        if (kb > tc.kb0 && (kk & ((16 << lbs) - 1)) == 0) {
          // a new window of 16 blocks starts at this k-block
          __syncwarp();  // the row's c~ of the previous window have been read
          store4(nin);
          __syncwarp();
          wnext += 16;
          load4(wnext + 4 * qk, nin);
        }
        const int blk = ((kk + kGemmCodes * qk) >> lbs) & 15;  // this thread's block in the window
        const float sc = scrow[blk];
        const uint64_t sc2 = f2_pack(sc, sc);
        const float nz = ASYM ? -(float)zrow[blk] : 0.0f;
        const uint64_t nz2 = f2_pack(nz, nz);
        // lane 0 waits for the copy (acquire); the shuffle keeps the other
        // lanes' reads of the stage after it
        {
          bool ready = true;
          if (lane == 0) ready = mbar_wait(full_bar(s), use & 1, p.status, abort, p.wait_ns);
          if (!__shfl_sync(0xffffffffu, ready ? 1 : 0, 0)) {
            ok = false;
            break;
          }
        }
        // kGemmCodes / 2 packed bytes = codes kGemmCodes qk .. + kGemmCodes - 1 of row d
        uint32_t rw[kGemmCodes / 8];
        if constexpr (kGemmCodes == 16) {
          const uint2 v = *reinterpret_cast<const uint2 *>(sR + s * kGemmRawTile + d * 32 + qk * 8);
          rw[0] = v.x;
          rw[1] = v.y;
        } else {
          const uint4 v = *reinterpret_cast<const uint4 *>(sR + s * kGemmRawTile + d * 32 + qk * 16);
          rw[0] = v.x;
          rw[1] = v.y;
          rw[2] = v.z;
          rw[3] = v.w;
        }
        uint8_t *brow = sB + s * kGemmBTile + (d >> 3) * 1024 + (d & 7) * 128;
#pragma unroll
        for (int c2 = 0; c2 < kGemmCodes / 8; ++c2) {  // 16-byte chunk (kGemmCodes / 8) qk + c2
          const uint32_t w = rw[c2];
          const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;  // codes 2j, 2j+1
          uint32_t o[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            // level table: entry e of this lane at lvb + e * 128
            const float l0 = lds_f32((__byte_perm(lo, 0u, 0x4440u | j) << 7) + lvb);
            const float l1 = lds_f32((__byte_perm(hi, 0u, 0x4440u | j) << 7) + lvb);
            uint64_t l2 = f2_pack(l0, l1);
            if constexpr (ASYM) l2 = f2_add(l2, nz2);  // q - z, exact
            float p0, p1;  // one rounding each, as the scalar multiply
            f2_unpack(f2_mul(sc2, l2), p0, p1);
            o[j] = Dt<DA>::pack2(p0, p1);
          }
          const int c = (kGemmCodes / 8) * qk + c2;
          *reinterpret_cast<uint4 *>(brow + ((c ^ (d & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bfull_bar(s));
        // the previous tile's epilogue once this tile's first stages are
        // queued (GemmShape::kEpiAfter)
        if (have_prev && kb - tc.kb0 == min(Sh::kEpiAfter, tc.kb1 - tc.kb0) - 1) {
          if (!epilogue(prev_item, prev_count)) {
            ok = false;
            break;
          }
          have_prev = false;
        }
      }
      if (!ok) break;
      have_prev = true;
      prev_item = item;
      prev_count = tcount;
    }
    if (have_prev && !*abort) epilogue(prev_item, prev_count);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
}

}  // namespace q4
