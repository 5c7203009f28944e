// q4_common.cuh -- shared device helpers for the sm_100a kernels of libq4.so.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/q4.h"

namespace q4 {

// Sticky status word (Q4_STATUS_* bits): kernels receive its device address.
// Programmatic dependent launch: every kernel of this library is launched
// with programmatic stream serialization, so it may become resident while
// the previous kernel of the stream drains.  It first lets the next kernel
// start launching, then waits until the previous one has completed and its
// memory operations are visible, before touching global memory.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_then_wait() {
  pdl_launch_dependents();
  pdl_wait();
}
// A kernel whose set-up reads neither global memory nor anything the
// previous kernel writes (shared-memory tables, barrier init, tensor-map
// prefetch) runs it between the two: it then overlaps the previous kernel's
// last CTAs, and each thread calls pdl_wait() before its first global access.

__device__ __forceinline__ void raise_status(int *status, int bit) {
  if (status) atomicOr(status, bit);
}

// ---- 16-bit loads/conversions ------------------------------------------------
template <int DT> struct Dt;
template <> struct Dt<Q4_F16> {
  using T = __half;
  using T2 = __half2;
  static __device__ __forceinline__ float to_f(uint16_t b) {
    return __half2float(__ushort_as_half(b));
  }
  static __device__ __forceinline__ uint16_t from_f(float f) {
    return __half_as_ushort(__float2half_rn(f));
  }
  static __device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
  }
};
template <> struct Dt<Q4_BF16> {
  using T = __nv_bfloat16;
  using T2 = __nv_bfloat162;
  static __device__ __forceinline__ float to_f(uint16_t b) {
    return __uint_as_float(((uint32_t)b) << 16);
  }
  static __device__ __forceinline__ uint16_t from_f(float f) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
  }
  static __device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
  }
};

// Lower / upper 16-bit float of a 32-bit word as binary32.
template <int DT> __device__ __forceinline__ float lo16(uint32_t w) {
  return Dt<DT>::to_f((uint16_t)(w & 0xFFFFu));
}
template <int DT> __device__ __forceinline__ float hi16(uint32_t w) {
  return Dt<DT>::to_f((uint16_t)(w >> 16));
}

// Streaming 128-bit global load that does not allocate in L1.
__device__ __forceinline__ uint4 ldg_stream_v4(const void *p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}
__device__ __forceinline__ uint32_t ldg_stream_u32(const void *p) {
  uint32_t r;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
  return r;
}

// Correctly rounded binary32 quotient a / b from y = RN(1/b) with one
// correction step (Markstein's theorem: q = RN(a*y) is within one ulp of a/b,
// the residual r = a - b*q is exact under FMA, and RN(q + r*y) = RN(a/b);
// the residual must not underflow: with the divisor in [2^-90, 2^125] the
// result is exact whenever |a/b| >= 2^-6 and otherwise stays below 2^-5 in
// magnitude, which decides every NF4 code and every INT4 rint the same way;
// callers use __fdiv_rn outside that divisor range).
__device__ __forceinline__ float div_markstein(float a, float b, float y) {
  float q = __fmul_rn(a, y);
  float r = __fmaf_rn(-q, b, a);
  return __fmaf_rn(r, y, q);
}

// The per-block scale buffer of a state (`absmax`): binary32, or binary16
// when the state's scales are stored as binary16 (INT4 with Q4_SCALE_F16).
__device__ __forceinline__ float ld_scale(const float *absmax, int64_t b, bool f16) {
  if (f16) return __half2float(__ushort_as_half(__ldg(reinterpret_cast<const unsigned short *>(absmax) + b)));
  return __ldg(absmax + b);
}
// Scales b0 .. b0 + 7 (all inside the buffer), vector loads when aligned.
__device__ __forceinline__ void ld_scales8(const float *absmax, int64_t b0, bool f16, float (&f)[8]) {
  if (f16) {
    const unsigned short *h = reinterpret_cast<const unsigned short *>(absmax) + b0;
    if (((uintptr_t)h & 15u) == 0) {
      const uint4 v = __ldg(reinterpret_cast<const uint4 *>(h));
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        f[2 * j] = __half2float(__ushort_as_half((unsigned short)(w[j] & 0xFFFFu)));
        f[2 * j + 1] = __half2float(__ushort_as_half((unsigned short)(w[j] >> 16)));
      }
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) f[j] = __half2float(__ushort_as_half(__ldg(h + j)));
    }
  } else if (((uintptr_t)(absmax + b0) & 15u) == 0) {
    const float4 x = __ldg(reinterpret_cast<const float4 *>(absmax + b0));
    const float4 y = __ldg(reinterpret_cast<const float4 *>(absmax + b0) + 1);
    f[0] = x.x, f[1] = x.y, f[2] = x.z, f[3] = x.w, f[4] = y.x, f[5] = y.y, f[6] = y.z, f[7] = y.w;
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) f[j] = __ldg(absmax + b0 + j);
  }
}
// Stores scale v (already a binary16 value when f16) of block b.
__device__ __forceinline__ void st_scale(float *absmax, int64_t b, float v, bool f16) {
  if (f16) reinterpret_cast<unsigned short *>(absmax)[b] = __half_as_ushort(__float2half_rn(v));
  else absmax[b] = v;
}

// Two binary32 values in one 64-bit register for the packed f32x2 ALU ops
// of sm_100 (each lane of a pair is computed and rounded exactly as the
// scalar instruction would).
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float &lo, float &hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
// div_markstein on a pair: yy = {y, y}, nb = {-b, -b}.
__device__ __forceinline__ uint64_t div_markstein2(uint64_t a, uint64_t nb, uint64_t yy) {
  const uint64_t q = f2_mul(a, yy);
  const uint64_t r = f2_fma(q, nb, a);
  return f2_fma(r, yy, q);
}

__device__ __forceinline__ bool markstein_ok(float b) {
  float ab = fabsf(b);
  return ab >= 8.0779356e-28f /* 2^-90 */ && ab <= 4.2535296e37f /* 2^125 */;
}

}  // namespace q4
