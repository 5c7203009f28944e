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
// Design (one CTA per SM, persistent over output tiles of 256 x 256):
//   warp 0      TMA producer: the A tile [256 x 64] (128B-swizzled, K-major)
//               and the raw packed tile [256 rows x 32 bytes] per k-block.
//   warp 1      TMEM allocator and MMA issuer: per k-block 2 x 4
//               tcgen05.mma kind::f16 (M=128, N=256, K=16) into two fp32
//               accumulators (512 TMEM columns), committed to the stage's
//               "empty" barrier.
//   warps 4..11 dequant: thread d expands weight row d of the tile (64 codes)
//               with its block scale into bf16/fp16 and writes it in the
//               128B-swizzled K-major layout the UMMA descriptor reads; then
//               the epilogue: tcgen05.ld of the accumulators, convert, store.
// Every mbarrier wait is bounded in time; a timeout sets Q4_STATUS_TIMEOUT,
// stops the pipeline, waits for issued copies and frees TMEM.
#pragma once
#include <cuda.h>

#include "q4_common.cuh"

namespace q4 {

constexpr int kGemmBM = 256;
constexpr int kGemmBN = 256;
constexpr int kGemmBK = 64;
constexpr int kGemmStages = 3;
constexpr int kGemmThreads = 384;
constexpr int kGemmATile = kGemmBM * kGemmBK * 2;   // 32 KB
constexpr int kGemmBTile = kGemmBN * kGemmBK * 2;   // 32 KB
constexpr int kGemmRawTile = kGemmBN * kGemmBK / 2; // 8 KB
constexpr int kGemmStageBytes = kGemmATile + kGemmBTile + kGemmRawTile;
constexpr int kGemmSmem = kGemmStages * kGemmStageBytes + 1024 /*align*/ + 256 /*barriers*/;

struct alignas(64) GemmMat {
  CUtensorMap tmA;  // A [M, K] 16-bit, box {64, 256}, 128B swizzle
  CUtensorMap tmW;  // packed [N, K/2] bytes, box {32, 256}
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

struct GemmParams {
  GemmMat mat[16];
  int32_t count;
  int32_t y_dtype;
  int32_t dq;
  int32_t pad;
  int64_t total_tiles;
  int *status;
  float levels[16];
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
// Bounded wait: gives up after ~2 s, raises Q4_STATUS_TIMEOUT and sets *abort.
// The first probe is inlined; only a phase that is not yet complete pays the
// call into the polling loop.
static __device__ __noinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity, int *status,
                                                   volatile int *abort) {
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try(bar, parity)) return true;
    if (*abort) return false;
    if (globaltimer_ns() - t0 > 2000000000ull) {
      raise_status(status, Q4_STATUS_TIMEOUT);
      *abort = 1;
      return false;
    }
  }
}
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, int *status, volatile int *abort) {
  if (mbar_try(bar, parity)) return true;
  return mbar_wait_slow(bar, parity, status, abort);
}

// Wait by a whole warp: only lane 0 polls the barrier (many polling lanes
// would queue their try_waits ahead of the single-thread producers), then
// the result is broadcast.  Must be called by all 32 lanes.
// After lane 0 has seen the phase complete, each other lane queries it once
// (returns at once) so that it acquires the data the phase published itself.
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity, int *status, volatile int *abort) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, status, abort);
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
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

struct TileCoord {
  int mi, tm, tn;
};
__device__ __forceinline__ TileCoord gemm_tile(const GemmParams &p, int64_t t) {
  int mi = 0;
  while (mi + 1 < p.count && t >= p.mat[mi + 1].tile_begin) ++mi;
  const int64_t local = t - p.mat[mi].tile_begin;
  const int tm_count = p.mat[mi].tiles_m;
  // m-tiles fastest: consecutive CTAs share one weight tile (read once from HBM)
  return TileCoord{mi, (int)(local % tm_count), (int)(local / tm_count)};
}

template <int DA>
__global__ void __launch_bounds__(kGemmThreads, 1) gemm_kernel(const __grid_constant__ GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t *sA = smem;                                        // [stages][32 KB]
  uint8_t *sB = smem + kGemmStages * kGemmATile;             // [stages][32 KB]
  uint8_t *sR = sB + kGemmStages * kGemmBTile;               // [stages][8 KB]
  uint64_t *bars = reinterpret_cast<uint64_t *>(sR + kGemmStages * kGemmRawTile);
  // bars: full[S], bfull[S], empty[S], accfull, accempty
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ float s_lv[16 * 32];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto bfull_bar = [&](int s) { return bar0 + 8u * (kGemmStages + s); };
  auto empty_bar = [&](int s) { return bar0 + 8u * (2 * kGemmStages + s); };
  const uint32_t accfull_bar = bar0 + 8u * (3 * kGemmStages);
  const uint32_t accempty_bar = bar0 + 8u * (3 * kGemmStages + 1);

  if (tid == 0) {
    for (int s = 0; s < kGemmStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(bfull_bar(s), 8);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(accfull_bar, 1);
    mbar_init(accempty_bar, 8);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    s_abort = 0;
  }
  for (int i = tid; i < 16 * 32; i += kGemmThreads) s_lv[i] = p.levels[i >> 5];
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  volatile int *abort = &s_abort;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t it = 0;
      for (int64_t t = blockIdx.x; t < p.total_tiles && !*abort; t += gridDim.x) {
        const TileCoord tc = gemm_tile(p, t);
        const GemmMat &m = p.mat[tc.mi];
        const int nk = m.K / kGemmBK;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % kGemmStages;
          const uint32_t use = it / kGemmStages;
          if (!mbar_wait(empty_bar(s), (use & 1) ^ 1, p.status, abort)) break;
          mbar_arrive_expect_tx(full_bar(s), kGemmATile + kGemmRawTile);
          tma_load_2d(smem_u32(sA + s * kGemmATile), &m.tmA, full_bar(s), kb * kGemmBK, tc.tm * kGemmBM);
          tma_load_2d(smem_u32(sR + s * kGemmRawTile), &m.tmW, full_bar(s), kb * (kGemmBK / 2), tc.tn * kGemmBN);
        }
      }
      // every issued copy completes before the CTA may exit
      for (uint32_t j = (it > kGemmStages ? it - kGemmStages : 0); j < it; ++j) {
        int dummy = 0;
        volatile int no_abort = 0;
        mbar_wait(full_bar(j % kGemmStages), (j / kGemmStages) & 1, &dummy, &no_abort);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_f16(DA == Q4_BF16 ? 1 : 0, 128, kGemmBN);
      uint32_t it = 0, tcount = 0;
      for (int64_t t = blockIdx.x; t < p.total_tiles && !*abort; t += gridDim.x, ++tcount) {
        const TileCoord tc = gemm_tile(p, t);
        const int nk = p.mat[tc.mi].K / kGemmBK;
        if (!mbar_wait(accempty_bar, (tcount & 1) ^ 1, p.status, abort)) break;
        tc_fence_after();
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % kGemmStages;
          const uint32_t use = it / kGemmStages;
          if (!mbar_wait(full_bar(s), use & 1, p.status, abort) ||
              !mbar_wait(bfull_bar(s), use & 1, p.status, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + s * kGemmATile);
          const uint32_t b0 = smem_u32(sB + s * kGemmBTile);
#pragma unroll
          for (int k16 = 0; k16 < kGemmBK / 16; ++k16) {
            const uint64_t db = umma_desc_sw128(b0 + 32 * k16);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint64_t da = umma_desc_sw128(a0 + h * (kGemmATile / 2) + 32 * k16);
              umma_f16(tmem + h * kGemmBN, da, db, idesc, (kb | k16) != 0);
            }
          }
          umma_commit(empty_bar(s));
        }
        if (!ok) break;
        umma_commit(accfull_bar);
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ dequant + epilogue
    const int d = tid - 128;  // weight row within the tile, 0..255
    const int q = warp & 3;   // TMEM lane quadrant of this warp
    const int ch = (warp - 4) >> 2;  // column half handled in the epilogue
    const bool dq = p.dq != 0;
    uint32_t it = 0, tcount = 0;
    for (int64_t t = blockIdx.x; t < p.total_tiles && !*abort; t += gridDim.x, ++tcount) {
      const TileCoord tc = gemm_tile(p, t);
      const GemmMat &m = p.mat[tc.mi];
      const int nk = m.K / kGemmBK;
      const int row = tc.tn * kGemmBN + d;
      const bool row_ok = row < m.N;
      const float mu = (dq && row_ok) ? __ldg(m.absmax_mean) : 0.0f;
      const int64_t bi0 = (int64_t)row * nk;
      auto scale_of = [&](int kb) -> float {
        if (!row_ok || kb >= nk) return 0.0f;
        const int64_t bi = bi0 + kb;
        if (dq) return __fadd_rn(__fmul_rn((float)__ldg(m.absmax_q + bi), __ldg(m.absmax_scale + (bi >> 8))), mu);
        return __ldg(m.absmax + bi);
      };
      float sc_next = scale_of(0);
      bool ok = true;
      for (int kb = 0; kb < nk; ++kb, ++it) {
        const int s = it % kGemmStages;
        const uint32_t use = it / kGemmStages;
        const float sc = sc_next;
        sc_next = scale_of(kb + 1);
        if (!mbar_wait_warp(full_bar(s), use & 1, p.status, abort)) {
          ok = false;
          break;
        }
        const uint4 *raw = reinterpret_cast<const uint4 *>(sR + s * kGemmRawTile + d * 32);
        const uint4 r0 = raw[0], r1 = raw[1];
        const uint32_t words[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
        uint8_t *brow = sB + s * kGemmBTile + (d >> 3) * 1024 + (d & 7) * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {  // 16-byte chunk c = k 8c..8c+7 = packed word c
          const uint32_t w = words[c];
          uint32_t o[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float l0 = s_lv[((w >> (8 * j)) & 15) * 32 + lane];
            const float l1 = s_lv[((w >> (8 * j + 4)) & 15) * 32 + lane];
            o[j] = Dt<DA>::pack2(__fmul_rn(sc, l0), __fmul_rn(sc, l1));
          }
          *reinterpret_cast<uint4 *>(brow + ((c ^ (d & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bfull_bar(s));
      }
      if (!ok) break;
      // ---- epilogue
      if (!mbar_wait_warp(accfull_bar, tcount & 1, p.status, abort)) break;
      tc_fence_after();
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        const int mrow = tc.tm * kGemmBM + h * 128 + q * 32 + lane;
#pragma unroll 1
        for (int j = 0; j < 4; ++j) {
          const int col0 = ch * 128 + j * 32;
          uint32_t r[32];
          tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(h * kGemmBN + col0), r);
          const int n0 = tc.tn * kGemmBN + col0;
          if (mrow < m.M && n0 < m.N) {
            if (p.y_dtype == Q4_F32) {
              float *y = reinterpret_cast<float *>(m.Y) + (int64_t)mrow * m.N + n0;
#pragma unroll
              for (int v = 0; v < 8; ++v)
                if (n0 + 4 * v < m.N)
                  *reinterpret_cast<uint4 *>(y + 4 * v) = make_uint4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
            } else {
              uint16_t *y = reinterpret_cast<uint16_t *>(m.Y) + (int64_t)mrow * m.N + n0;
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                if (n0 + 8 * v < m.N) {
                  uint32_t o[4];
#pragma unroll
                  for (int e = 0; e < 4; ++e) {
                    const float f0 = __uint_as_float(r[8 * v + 2 * e]), f1 = __uint_as_float(r[8 * v + 2 * e + 1]);
                    o[e] = (p.y_dtype == Q4_BF16) ? Dt<Q4_BF16>::pack2(f0, f1) : Dt<Q4_F16>::pack2(f0, f1);
                  }
                  *reinterpret_cast<uint4 *>(y + 8 * v) = make_uint4(o[0], o[1], o[2], o[3]);
                }
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(accempty_bar);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
}

}  // namespace q4
