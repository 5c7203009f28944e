// gemv.cuh -- fused NF4 dequant-GEMV for decode, Y[M,N] = A[M,K] . W^[N,K]^T,
// 1 <= M <= 32 (sm_100a).
//
// What it computes: n4n.ai, "What is 4-bit quantization and why does it
// matter?", "Why it matters for deployment" (decode at batch < 32 reads every
// weight once per token and is bound by memory) and learn.pranaymahendrakar.com,
// "Loading a model in 4-bit", "Where the accuracy goes" (the weights are
// dequantized to the compute dtype and multiplied in 16-bit); here the
// dequantization happens in registers while the packed weights stream from
// HBM, and the products accumulate in fp32.
//
// Design (B200): the weights are the 16-row side of mma.sync m16n8k16
// (swap-AB), the activations the 8-column side (M padded to 8/16/32).  A lane
// of quad position tig owns B/8 consecutive bytes of one block row, so every
// MMA k-step stays inside one block: the MMA runs on the *unscaled* codebook
// values (a 256-entry byte -> two-level LUT in shared memory, one copy per
// lane so lookups never conflict) and the per-block scale c~ (double-dequant
// of the absmax) multiplies the fp32 partial once per block.  The k order
// inside a block is permuted identically on both operands.  Packed weights
// are prefetched into registers PF blocks ahead with 8-byte streaming loads.
// Work is split into units of (row tile, k-range) over all matrices of one
// grouped launch; partial sums of split rows are added with fp32 atomics into
// a workspace and the last unit to finish a row tile (arrival counter) writes
// Y and zeroes its workspace rows again.
#pragma once
#include "q4_common.cuh"

namespace q4 {

constexpr int kMaxGroup = 16;
constexpr int kGemvWarps = 8;

struct GemvMat {
  const uint8_t *packed;
  const float *absmax;
  const int8_t *absmax_q;
  const float *absmax_scale;
  const float *absmax_mean;
  const uint16_t *A;
  void *Y;
  float *acc;      // workspace [N][M] fp32 (n_splits > 1)
  unsigned *cnt;   // workspace [n_tiles] arrival counters (n_splits > 1)
  int64_t unit_begin;
  int32_t N, K;
  int32_t n_tiles, n_splits;
};

struct GemvParams {
  GemvMat mat[kMaxGroup];
  int32_t count;
  int32_t M;
  int32_t y_dtype;
  int32_t dq;
  int64_t total_units;
  float levels[16];
};

template <int DA> struct Mma;
template <> struct Mma<Q4_F16> {
  static __device__ __forceinline__ void run(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                             uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
};
template <> struct Mma<Q4_BF16> {
  static __device__ __forceinline__ void run(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                             uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
};

// Per-lane slice of one block row: B/8 bytes = NW 32-bit words.
template <int B> struct WRow {
  static constexpr int NW = B / 32;
  uint32_t w[NW];
  __device__ __forceinline__ void load(const uint8_t *p) {
    if constexpr (NW == 1) {
      w[0] = __ldg(reinterpret_cast<const unsigned int *>(p));
    } else if constexpr (NW == 2) {
      uint2 v = ldg_stream_v2(p);
      w[0] = v.x;
      w[1] = v.y;
    } else {
#pragma unroll
      for (int i = 0; i < NW; i += 4) {
        uint4 v = ldg_stream_v4(p + 4 * i);
        w[i] = v.x; w[i + 1] = v.y; w[i + 2] = v.z; w[i + 3] = v.w;
      }
    }
  }
  __device__ __forceinline__ void zero() {
#pragma unroll
    for (int i = 0; i < NW; ++i) w[i] = 0;
  }
  __device__ __forceinline__ uint32_t byte(int j) const { return (w[j >> 2] >> (8 * (j & 3))) & 0xFFu; }
};

// One prefetch stage: the lane's bytes of rows g and g+8 of R row tiles, and
// their block scales.
template <int B, int R> struct Stage {
  WRow<B> row[R][2];
  float sc[R][2];
};

// Y element store in the output dtype (uniform runtime switch).
__device__ __forceinline__ void store_y(void *Y, int ydt, int64_t idx, float v) {
  if (ydt == Q4_F32) reinterpret_cast<float *>(Y)[idx] = v;
  else if (ydt == Q4_F16) reinterpret_cast<uint16_t *>(Y)[idx] = Dt<Q4_F16>::from_f(v);
  else reinterpret_cast<uint16_t *>(Y)[idx] = Dt<Q4_BF16>::from_f(v);
}

template <int DA, int NT, int R, int B, int UB, int PF>
__global__ void __launch_bounds__(kGemvWarps * 32) gemv_kernel(GemvParams p) {
  constexpr int STEPS = B / 16;                  // MMA k-steps per block
  constexpr int ROWS = 16 * R;                   // rows per unit
  extern __shared__ uint32_t s_lut[];            // [256][32] (fp16 pairs or float2)

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tig = lane & 3;

  if constexpr (DA == Q4_BF16) {
    // bf16 activations: the reference dequantizes to bf16 first, so the MMA
    // must see the exact w^ = bf16(c~ * level); the LUT holds binary32 level
    // pairs and the scale is applied per weight before the rounding.
    float2 *lut2 = reinterpret_cast<float2 *>(s_lut);
    for (int i = tid; i < 256 * 32; i += blockDim.x) {
      const int b = i >> 5;
      lut2[i] = make_float2(p.levels[b & 15], p.levels[b >> 4]);
    }
  } else {
    // fp16 activations: byte -> (level(lo nibble), level(hi nibble)) as an
    // fp16 pair; the block scale multiplies the fp32 partial afterwards.
    for (int i = tid; i < 256 * 32; i += blockDim.x) {
      const int b = i >> 5;
      s_lut[i] = Dt<DA>::pack2(p.levels[b & 15], p.levels[b >> 4]);
    }
  }
  __syncthreads();

  const int M = p.M;
  for (int64_t u = (int64_t)blockIdx.x * kGemvWarps + warp; u < p.total_units;
       u += (int64_t)gridDim.x * kGemvWarps) {
    int mi = 0;
#pragma unroll 1
    while (mi + 1 < p.count && u >= p.mat[mi + 1].unit_begin) ++mi;
    const GemvMat &mt = p.mat[mi];
    const int64_t local = u - mt.unit_begin;
    const int tile = (int)(local % mt.n_tiles);
    const int split = (int)(local / mt.n_tiles);
    const int K = mt.K, N = mt.N;
    const int nbk = K / B;                     // blocks per row
    const int blk0 = split * UB;
    const int nblk = min(UB, nbk - blk0);
    const int r_base = tile * ROWS;
    const bool dq = p.dq != 0;
    const float mu = dq ? __ldg(mt.absmax_mean) : 0.0f;

    float acc[R][NT][4];
#pragma unroll
    for (int rt = 0; rt < R; ++rt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[rt][nt][i] = 0.0f;

    Stage<B, R> st[PF];
    auto load_stage = [&](Stage<B, R> &s, int i) {
      const int blk = blk0 + i;
#pragma unroll
      for (int rt = 0; rt < R; ++rt)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int row = r_base + rt * 16 + h * 8 + g;
          if (i < nblk && row < N) {
            const int64_t bi = (int64_t)row * nbk + blk;
            s.row[rt][h].load(mt.packed + (int64_t)row * (K / 2) + (int64_t)blk * (B / 2) + tig * (B / 8));
            if (dq) {
              s.sc[rt][h] = __fadd_rn(__fmul_rn((float)__ldg(mt.absmax_q + bi), __ldg(mt.absmax_scale + (bi >> 8))), mu);
            } else {
              s.sc[rt][h] = __ldg(mt.absmax + bi);
            }
          } else {
            s.row[rt][h].zero();
            s.sc[rt][h] = 0.0f;
          }
        }
    };

#pragma unroll
    for (int i = 0; i < PF; ++i) load_stage(st[i], i);

#pragma unroll
    for (int i = 0; i < UB; ++i) {
      Stage<B, R> cur = st[i % PF];
      if (i + PF < UB) load_stage(st[i % PF], i + PF);
      if (i < nblk) {
        const int k0 = (blk0 + i) * B + tig * (B / 4);
        // activations: lane (g, tig) holds A[nt*8+g][k0 .. k0 + B/4)
        uint32_t act[NT][B / 8];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int m = nt * 8 + g;
          if (m < M) {
            const uint16_t *ap = mt.A + (int64_t)m * K + k0;
#pragma unroll
            for (int v = 0; v < B / 32; ++v) {
              uint4 x = __ldg(reinterpret_cast<const uint4 *>(ap) + v);
              act[nt][4 * v] = x.x; act[nt][4 * v + 1] = x.y;
              act[nt][4 * v + 2] = x.z; act[nt][4 * v + 3] = x.w;
            }
          } else {
#pragma unroll
            for (int v = 0; v < B / 8; ++v) act[nt][v] = 0;
          }
        }
        if constexpr (DA == Q4_BF16) {
          const float2 *lut2 = reinterpret_cast<const float2 *>(s_lut) + lane;
#pragma unroll
          for (int s = 0; s < STEPS; ++s) {
#pragma unroll
            for (int rt = 0; rt < R; ++rt) {
              const float c0 = cur.sc[rt][0], c1 = cur.sc[rt][1];
              const float2 e0 = lut2[cur.row[rt][0].byte(2 * s) * 32];
              const float2 e1 = lut2[cur.row[rt][1].byte(2 * s) * 32];
              const float2 e2 = lut2[cur.row[rt][0].byte(2 * s + 1) * 32];
              const float2 e3 = lut2[cur.row[rt][1].byte(2 * s + 1) * 32];
              uint32_t a[4];
              a[0] = Dt<DA>::pack2(__fmul_rn(c0, e0.x), __fmul_rn(c0, e0.y));
              a[1] = Dt<DA>::pack2(__fmul_rn(c1, e1.x), __fmul_rn(c1, e1.y));
              a[2] = Dt<DA>::pack2(__fmul_rn(c0, e2.x), __fmul_rn(c0, e2.y));
              a[3] = Dt<DA>::pack2(__fmul_rn(c1, e3.x), __fmul_rn(c1, e3.y));
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) Mma<DA>::run(acc[rt][nt], a, act[nt][2 * s], act[nt][2 * s + 1]);
            }
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
          for (int s = 0; s < STEPS; ++s) {
#pragma unroll
            for (int rt = 0; rt < R; ++rt) {
              const uint32_t *lut = s_lut + lane;
              uint32_t a[4];
              a[0] = lut[cur.row[rt][0].byte(2 * s) * 32];
              a[1] = lut[cur.row[rt][1].byte(2 * s) * 32];
              a[2] = lut[cur.row[rt][0].byte(2 * s + 1) * 32];
              a[3] = lut[cur.row[rt][1].byte(2 * s + 1) * 32];
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) Mma<DA>::run(part[rt][nt], a, act[nt][2 * s], act[nt][2 * s + 1]);
            }
          }
#pragma unroll
          for (int rt = 0; rt < R; ++rt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              acc[rt][nt][0] = fmaf(cur.sc[rt][0], part[rt][nt][0], acc[rt][nt][0]);
              acc[rt][nt][1] = fmaf(cur.sc[rt][0], part[rt][nt][1], acc[rt][nt][1]);
              acc[rt][nt][2] = fmaf(cur.sc[rt][1], part[rt][nt][2], acc[rt][nt][2]);
              acc[rt][nt][3] = fmaf(cur.sc[rt][1], part[rt][nt][3], acc[rt][nt][3]);
            }
        }
      }
    }

    // ---- epilogue: D fragment (row g / g+8, column m = nt*8 + 2*tig + {0,1})
    if (mt.n_splits == 1) {
#pragma unroll
      for (int rt = 0; rt < R; ++rt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int row = r_base + rt * 16 + (j >> 1) * 8 + g;
            const int m = nt * 8 + 2 * tig + (j & 1);
            if (m < M && row < N) store_y(mt.Y, p.y_dtype, (int64_t)m * N + row, acc[rt][nt][j]);
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
          store_y(mt.Y, p.y_dtype, (int64_t)m * N + r_base + r, v);
        }
        if (lane == 0) mt.cnt[tile] = 0u;
      }
    }
  }
}

}  // namespace q4
