// quantize_grouped.cuh -- the blockwise 4-bit quantize of every matrix of a
// layer in one persistent, warp-specialized launch (sm_100a).
//
// What it computes is quantize_kernel's (learn.pranaymahendrakar.com,
// "Loading a model in 4-bit", "Block-wise quantisation, stated exactly";
// n4n.ai "INT4 symmetric"; robotsatlas.com "INT4", "How it works"): per block
// of B contiguous weights the scale, the 16 codes packed two per byte, and
// with double quantization the fp64 pairwise mean of the block absmax values
// (learn.pranaymahendrakar.com, "Double quantisation") -- bit for bit.
//
// Design (one CTA of 32 warps per SM, persistent over the 256-block chunks
// of all matrices with a grid stride):
//   warp 30     producer: streams each chunk as pieces of 8192 weights
//               (16 KB) into a ring of kQgStages shared-memory stages with
//               cp.async.bulk (one copy per piece, completion counted on the
//               stage's mbarrier), so DRAM reads run ahead of the math;
//   warps 0..29 consumers: the pieces are cut into slices of 1024 weights
//               that the warps take in turn (slice i of the CTA's stream goes
//               to warp i mod 30); lane l quantizes weights 16l..16l+15 and
//               512+16l..512+16l+15 of the slice, writes the packed codes
//               and, per block, the scale (and zero-point; with double
//               quantization also into the chunk's buffer in shared memory),
//               then the warp releases the slice; a stage is free again once
//               its 8 slices are released;
//   warp 31     reducer (double quantization): when the producer reclaims
//               the last stage of a chunk it posts the chunk as done (every
//               scale of it is in the chunk buffer); the reducer forms the
//               fp64 pairwise sum of the chunk's 256 block scales, stored
//               per chunk, and frees the buffer (the producer issues a
//               chunk's first piece only once the reducer has freed the
//               buffer the chunk will use); when the CTA has done its last chunk
//               of a matrix it adds its chunk count to the matrix's counter,
//               and the CTA that completes the count forms the mean at its
//               end, with all its threads, in the tree order of the
//               definition.
// The consumers carry no double-quant work and meet no CTA-wide barrier;
// every wait is bounded in time (a timeout sets Q4_STATUS_TIMEOUT, stops the
// CTA and waits for the copies in flight).
#pragma once
#include "gemm.cuh"  // mbarrier wrappers, bounded waits
#include "quantize.cuh"

namespace q4 {

constexpr int kQgWarps = 30;                         // consumer warps
constexpr int kQgThreads = (kQgWarps + 2) * 32;      // + producer + reducer
constexpr int kQgSlice = 1024;                       // weights per consumer step (2 x 16 per lane)
constexpr int kQgSlices = 8;                         // slices per piece
constexpr int kQgPiece = kQgSlices * kQgSlice;       // weights per ring stage (8192)
constexpr int kQgPieceBytes = kQgPiece * 2;          // 16 KB
constexpr int kQgStages = 8;
constexpr int kQgBufs = 16;                          // chunk buffers of block scales (reducer input)
constexpr int kQgRing = kQgStages * kQgPieceBytes;
constexpr uint32_t kQgSleepNs = 200;      // producer / reducer back-off between probes
constexpr int64_t kQgMaxChunks = 65536;  // chunk sums one matrix's mean is formed from
static_assert(kQgBufs >= kQgStages, "the producer never waits on a chunk buffer whose chunk it has not reclaimed");
constexpr int kQgSmem = kQgRing + 32 * 32 * 8 /*bin tables*/ + kQgBufs * kChunkBlocks * 4 +
                        (2 * kQgStages + 2 * kQgBufs) * 8 + 64;

__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ uint4 lds_v4(uint32_t addr) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(addr));
  return r;
}

// The fp64 pairwise sum (level by level, adjacent pairs, odd last carried
// up) of the n <= 65536 chunk sums at src, by all NT threads of the CTA.
// Padding the values with zeros to a power of two P >= 256 leaves that sum
// unchanged (x + 0 == x), so it is the aligned binary tree over P leaves:
// each warp forms aligned subtrees of 256 leaves (8 per lane, then xor
// shuffles pairing adjacent subtrees), and warp 0 the tree over the P / 256
// subtree sums, padded to 256 in turn.  Returns the sum in warp 0.
template <int NT>
__device__ __forceinline__ double qg_matrix_sum(const double *src, int64_t n, double *s_red, int tid) {
  const int lane = tid & 31, warp = tid >> 5;
  int64_t P = 256;
  while (P < n) P <<= 1;
  const int nsub = (int)(P / 256);
  for (int j = warp; j < nsub; j += NT / 32) {
    const int64_t b = (int64_t)j * 256 + 8 * lane;
    double x[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) x[t] = (b + t < n) ? __ldcg(src + b + t) : 0.0;
    double sm = ((x[0] + x[1]) + (x[2] + x[3])) + ((x[4] + x[5]) + (x[6] + x[7]));
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) sm = sm + __shfl_xor_sync(0xffffffffu, sm, o);
    if (lane == 0) s_red[j] = sm;
  }
  __syncthreads();
  double r = 0.0;
  if (warp == 0) {
    double x[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) x[t] = (8 * lane + t < nsub) ? s_red[8 * lane + t] : 0.0;
    r = ((x[0] + x[1]) + (x[2] + x[3])) + ((x[4] + x[5]) + (x[6] + x[7]));
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) r = r + __shfl_xor_sync(0xffffffffu, r, o);
  }
  __syncthreads();
  return r;
}

template <int DT, int QT, int B, bool DQ>
__global__ void __launch_bounds__(kQgThreads, 1) quantize_grouped_kernel(const __grid_constant__ QuantGroupParams p) {
  pdl_launch_dependents();  // the set-up below overlaps the previous kernel
  static_assert(B % 32 == 0 && B <= 256, "half a slice covers an even number of whole blocks");
  constexpr int LPB = B / 16;                                  // lanes per block
  constexpr int64_t CHUNK = (int64_t)kChunkBlocks * B;         // weights per chunk
  constexpr int NP = (int)(CHUNK / kQgPiece);                  // pieces per chunk
  constexpr int SPC = kQgSlices * NP;                          // slices per chunk
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t *ring = smem;
  float2 *s_tab = reinterpret_cast<float2 *>(smem + kQgRing);
  float *s_blk = reinterpret_cast<float *>(smem + kQgRing + 32 * 32 * 8);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kQgRing + 32 * 32 * 8 + kQgBufs * kChunkBlocks * 4);
  volatile int *abort = reinterpret_cast<volatile int *>(bars + 2 * kQgStages + 2 * kQgBufs);
  unsigned *combine = reinterpret_cast<unsigned *>(bars + 2 * kQgStages + 2 * kQgBufs) + 1;
  const uint32_t ring_u = smem_u32(ring);
  auto full = [&](int s) { return smem_u32(bars + s); };
  auto empty = [&](int s) { return smem_u32(bars + kQgStages + s); };
  auto done = [&](int b) { return smem_u32(bars + 2 * kQgStages + b); };
  auto dfree = [&](int b) { return smem_u32(bars + 2 * kQgStages + kQgBufs + b); };

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t G = gridDim.x;
  if (QT == Q4_NF4)
    for (int i = tid; i < 32 * 32; i += kQgThreads) {
      const int e = i >> 5;
      s_tab[i] = make_float2(p.tab.thr[e], __int_as_float(p.tab.base[e]));
    }
  if (tid == 0) {
    for (int s = 0; s < kQgStages; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), kQgSlices);  // one release per slice
    }
    for (int b = 0; b < kQgBufs; ++b) {
      mbar_init(done(b), 1);
      mbar_init(dfree(b), 1);
    }
    *abort = 0;
    *combine = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  pdl_wait();

  if (warp == kQgWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int64_t issued = 0, rel = 0;  // pieces issued / reclaimed (released by the consumers)
      int pc_rel = 0, k_rel = 0;    // piece of its chunk, and chunk ordinal, that `rel` is
      bool ok = true;
      // Reclaim the oldest piece's stage once its slices are released; the
      // last piece of a chunk makes the chunk done for the reducer (every
      // scale of it is in its chunk buffer).
      auto reclaim = [&]() -> bool {
        const int rs = (int)(rel % kQgStages);
        if (!mbar_wait(empty(rs), (uint32_t)((rel / kQgStages) & 1), p.status, abort, p.wait_ns, kQgSleepNs))
          return false;
        ++rel;
        if (++pc_rel == NP) {
          pc_rel = 0;
          if (DQ) mbar_arrive(done(k_rel % kQgBufs));
          ++k_rel;
        }
        return true;
      };
      int mi = 0, k = 0;
      for (int64_t gc = blockIdx.x; gc < p.total_chunks && ok; gc += G, ++k) {
        while (mi + 1 < p.count && gc >= p.mat[mi + 1].chunk_begin) ++mi;
        const QMat &m = p.mat[mi];
        const int64_t chunk = gc - m.chunk_begin;
        for (int pc = 0; pc < NP; ++pc) {
          if (issued - rel == kQgStages && !reclaim()) { ok = false; break; }
          // the chunk buffer that this chunk's scales go to was read by the
          // reducer for the chunk kQgBufs earlier
          if (DQ && pc == 0 && k >= kQgBufs &&
              !mbar_wait(dfree(k % kQgBufs), (uint32_t)(((k / kQgBufs) & 1) ^ 1), p.status, abort, p.wait_ns,
                         kQgSleepNs)) {
            ok = false;
            break;
          }
          const int s = (int)(issued % kQgStages);
          ++issued;
          if (p.stall_copies) continue;  // test hook: the stage is never filled
          const int64_t e0 = chunk * CHUNK + (int64_t)pc * kQgPiece;
          // whole 16-byte words of the piece (none past the matrix's end); the
          // last < 8 weights of a matrix are read by the consumers themselves
          const uint32_t bytes =
              e0 < m.n ? (uint32_t)min((int64_t)kQgPieceBytes, (m.n - e0) * 2) & ~15u : 0u;
          // the consumers' reads of this stage (generic proxy) come before
          // the copy that overwrites it (async proxy)
          fence_proxy_async_smem();
          mbar_arrive_expect_tx(full(s), bytes);
          if (bytes) bulk_load(ring_u + (uint32_t)s * kQgPieceBytes, m.W + e0, bytes, full(s));
        }
      }
      while (ok && rel < issued) ok = reclaim();  // the last chunks' releases
      if (!ok && !p.stall_copies) {
        // stopped early: let the copies still in flight land (pieces before
        // `rel` were consumed, so theirs are complete)
        for (int64_t g = rel; g < issued; ++g) {
          int dummy = 0;
          volatile int no_abort = 0;
          mbar_wait(full((int)(g % kQgStages)), (uint32_t)((g / kQgStages) & 1), &dummy, &no_abort);
        }
      }
    }
    __syncwarp();
  } else if (warp == kQgWarps + 1) {
    // ------------------------------------------------------------- reducer
    if (DQ) {
      int mi = 0, k = 0;
      unsigned cnt = 0;
      for (int64_t gc = blockIdx.x; gc < p.total_chunks; gc += G, ++k) {
        while (mi + 1 < p.count && gc >= p.mat[mi + 1].chunk_begin) ++mi;
        const QMat &m = p.mat[mi];
        const int64_t chunk = gc - m.chunk_begin;
        const int b = k % kQgBufs;
        if (!mbar_wait_warp(done(b), (uint32_t)((k / kQgBufs) & 1), p.status, abort, p.wait_ns, kQgSleepNs)) break;
        // Pairwise fp64 sum of the chunk's block scales in tree order: lane
        // l reduces blocks 8l..8l+7 as ((0+1)+(2+3))+((4+5)+(6+7)), then xor
        // shuffles at distance 1, 2, 4, 8, 16 pair adjacent subtrees; blocks
        // past the matrix's end count as 0.
        const int nbv = (int)min((int64_t)kChunkBlocks, m.nb - chunk * kChunkBlocks);
        const float4 a0 = *reinterpret_cast<const float4 *>(s_blk + b * kChunkBlocks + 8 * lane);
        const float4 a1 = *reinterpret_cast<const float4 *>(s_blk + b * kChunkBlocks + 8 * lane + 4);
        const float xs[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        double x[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) x[j] = (8 * lane + j < nbv) ? (double)xs[j] : 0.0;
        double sum = ((x[0] + x[1]) + (x[2] + x[3])) + ((x[4] + x[5]) + (x[6] + x[7]));
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) sum = sum + __shfl_xor_sync(0xffffffffu, sum, o);
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(dfree(b));
          m.partials[chunk] = sum;
          ++cnt;
          const int64_t nx = gc + G;
          if (nx >= p.total_chunks || nx >= m.chunk_begin + m.n_chunks) {
            // this CTA's last chunk of the matrix
            __threadfence();
            const unsigned old = atomicAdd(m.counter, cnt);
            if (old + cnt == (unsigned)m.n_chunks) *combine |= 1u << mi;
            cnt = 0;
          }
        }
      }
    }
  } else {
    // ----------------------------------------------------------- consumers
    const uint32_t tb = smem_u32(s_tab) + 8u * lane - 0x40000000u;
    int nonfinite = 0;
    int mi = 0, kc = -1;
    int left = 0;                  // weights of the current chunk (CHUNK when whole)
    const uint16_t *W = nullptr;   // the current chunk's weights, packed codes, scales, zero-points
    uint8_t *pk = nullptr, *zc = nullptr;
    float *am = nullptr, *sb = nullptr;  // am: the matrix's scales; block b of the chunk at ab0 + b
    int64_t ab0 = 0;
    const bool sf16 = p.scale_f16 != 0;
    // One 16-weight group of a slice: weights g0..g0+15 of the chunk, read
    // at shared address src.
    auto group = [&](int g0, uint32_t src, int pe0) {
      float scale = 0.0f;
      int z = 0;
      uint32_t codes[2];
      uint4 v[2];
      const int bl = g0 / B;  // block within the chunk
      if (left == (int)CHUNK) {
        v[0] = lds_v4(src);
        v[1] = lds_v4(src + 16);
        quant16<DT, QT, B>(v, scale, z, codes, lane, tb, s_tab, nonfinite, sf16);
        *reinterpret_cast<uint2 *>(pk + g0 / 2) = make_uint2(codes[0], codes[1]);
        if (QT == Q4_INT4_ASYM) {
          // the zero-points of blocks 2k, 2k+1 share a byte; 512 weights
          // cover an even number of whole blocks
          const int zn = __shfl_down_sync(0xffffffffu, z, LPB);
          if ((lane % (2 * LPB)) == 0) zc[bl >> 1] = (uint8_t)(z | (zn << 4));
        }
        if ((lane % LPB) == 0) {
          st_scale(am, ab0 + bl, scale, sf16);
          if (DQ) sb[bl] = scale;
        }
      } else {
        // the matrix's last chunk: weights up to the end; the copy holds the
        // piece's whole 16-byte words, the rest comes from global memory
        const int pvalid = min(kQgPiece, left - pe0);
        const int copied = pvalid & ~7;
        const int ip0 = g0 - pe0;  // within the piece
        if (ip0 + 16 <= copied) {
          v[0] = lds_v4(src);
          v[1] = lds_v4(src + 16);
        } else {
          uint32_t w[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            uint32_t h[2];
#pragma unroll
            for (int t = 0; t < 2; ++t) {
              const int ip = ip0 + 2 * j + t;
              uint16_t x = 0;
              if (ip < copied) {
                asm volatile("ld.shared.u16 %0, [%1];" : "=h"(x) : "r"(src + 2u * (2 * j + t)));
              } else if (ip < pvalid) {
                x = W[pe0 + ip];
              }
              h[t] = x;
            }
            w[j] = h[0] | (h[1] << 16);
          }
          v[0] = make_uint4(w[0], w[1], w[2], w[3]);
          v[1] = make_uint4(w[4], w[5], w[6], w[7]);
        }
        quant16<DT, QT, B>(v, scale, z, codes, lane, tb, s_tab, nonfinite, sf16);
        const int nv = min(16, left - g0);  // this lane's weights (<= 0: none)
        if (nv >= 16) {
          *reinterpret_cast<uint2 *>(pk + g0 / 2) = make_uint2(codes[0], codes[1]);
        } else if (nv > 0) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (2 * j < nv) {
              uint32_t byte = (codes[j >> 2] >> (8 * (j & 3))) & 0xFFu;
              if (2 * j + 1 >= nv) byte &= 0x0Fu;  // odd n: the high nibble is padding
              pk[g0 / 2 + j] = (uint8_t)byte;
            }
          }
        }
        if (QT == Q4_INT4_ASYM) {
          const int zn = __shfl_down_sync(0xffffffffu, z, LPB);
          if ((lane % (2 * LPB)) == 0 && nv > 0) zc[bl >> 1] = (uint8_t)(z | (zn << 4));
        }
        if ((lane % LPB) == 0 && nv > 0) {
          st_scale(am, ab0 + bl, scale, sf16);
          if (DQ) sb[bl] = scale;
        }
      }
    };
    // slice i of the CTA's walk: piece i / 8 (every chunk has NP pieces),
    // chunk ordinal i / (8 NP); warp w takes slices w, w + 30, ...
    for (int i = warp;; i += kQgWarps) {
      const int gp = i / kQgSlices;
      const int k = gp / NP;
      if (k != kc) {
        const int64_t gc = blockIdx.x + (int64_t)k * G;
        if (gc >= p.total_chunks) break;
        kc = k;
        while (mi + 1 < p.count && gc >= p.mat[mi + 1].chunk_begin) ++mi;
        const QMat &m = p.mat[mi];
        const int64_t chunk = gc - m.chunk_begin;
        const int64_t ce0 = chunk * CHUNK;
        left = (int)min(CHUNK, m.n - ce0);
        W = m.W + ce0;
        pk = m.packed + ce0 / 2;
        am = m.absmax;
        ab0 = chunk * kChunkBlocks;
        zc = QT == Q4_INT4_ASYM ? m.zero + chunk * (kChunkBlocks / 2) : nullptr;
        sb = s_blk + (k % kQgBufs) * kChunkBlocks;
      }
      const int sl = i % SPC;                         // slice of the chunk
      const int st = gp % kQgStages;
      if (!__all_sync(0xffffffffu, mbar_wait(full(st), (uint32_t)(gp / kQgStages) & 1u, p.status, abort,
                                             p.wait_ns)))
        break;
      const int s0 = sl * kQgSlice;                   // the slice's first weight within the chunk
      if (s0 < left) {
        const uint32_t src = ring_u + (uint32_t)st * kQgPieceBytes + (uint32_t)(i % kQgSlices) * (2 * kQgSlice) +
                             32u * lane;
        const int pe0 = (sl / kQgSlices) * kQgPiece;  // the piece's first weight
        group(s0 + 16 * lane, src, pe0);
        group(s0 + kQgSlice / 2 + 16 * lane, src + kQgSlice, pe0);
      }
      // release the slice once its results are written
      __syncwarp();
      if (lane == 0) mbar_arrive(empty(st));
    }
    if (nonfinite) raise_status(p.status, Q4_STATUS_NONFINITE);
  }

  if (DQ) {
    __syncthreads();  // every warp is done: the ring is free for the mean
    const unsigned mask = *combine;
    if (mask && !*abort) {
      double *s_red = reinterpret_cast<double *>(ring);
      for (int mi = 0; mi < p.count; ++mi) {
        if (!(mask & (1u << mi))) continue;
        const QMat &m = p.mat[mi];
        // this CTA completed the matrix's count: the pairwise tree over its
        // chunk sums
        __threadfence();
        const double S = qg_matrix_sum<kQgThreads>(m.partials, m.n_chunks, s_red, tid);
        for (int64_t i = tid; i < m.n_chunks; i += kQgThreads) __stcg(m.partials + i, 0.0);
        if (tid == 0) {
          m.absmax_mean[0] = __double2float_rn(__ddiv_rn(S, (double)m.nb));
          *m.counter = 0u;  // the workspace is left zeroed for the next call
        }
        __syncthreads();
      }
    }
  }
}

}  // namespace q4
