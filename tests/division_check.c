/*
 * division_check.c -- exhaustive CPU check of the quotient method the
 * quantize kernel uses in place of a full correctly rounded division.
 *
 * The kernel forms x = w / d as y = RN(1/d), q = RN(w*y), r = fma(-q, d, w),
 * x' = fma(r, y, q) (Markstein's method, "IA-64 and Elementary Functions",
 * Markstein, 2000, theorem 8.10: when RN(1/d) is correctly rounded and the
 * residual r is exact, x' = RN(w/d)).  It uses the method only for divisors
 * with 2^-90 <= |d| <= 2^125 and claims, for every 16-bit weight w with
 * |w| <= |the block maximum|:
 *   - |RN(w/d)| >= 2^-6  =>  x' == RN(w/d) bit for bit;
 *   - otherwise |x'| < 2^-5 and |RN(w/d)| < 2^-5, where every NF4 code
 *     (the level 0.0, decision points at -0.0455 and 0.0395) and every INT4
 *     rint (0) is the same.
 * This program checks the claim over every finite fp16 / bf16 pair (w, c)
 * with |w| <= c, for the NF4 divisor d = c and the INT4-symmetric divisor
 * d = RN(c / 7), and over a seeded random sample for the INT4-asymmetric
 * divisor d = RN(RN(mx - mn) / 15).  It prints the number of pairs checked
 * and of violations per case; exit status 1 on any violation.
 *
 * Build: gcc -O2 -std=c99 -ffp-contract=off [-fopenmp] division_check.c -lm
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

static float f32(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }

static float from16(uint16_t b, int bf16) {
  if (bf16) return f32((uint32_t)b << 16);
  /* binary16 -> binary32, exact */
  uint32_t s = (uint32_t)(b >> 15) << 31, e = (b >> 10) & 31, m = b & 1023;
  if (e == 0) {
    float v = (float)m * 5.9604644775390625e-08f; /* m * 2^-24, exact */
    return s ? -v : v;
  }
  return f32(s | ((e - 15 + 127) << 23) | (m << 13));
}

static int finite16(uint16_t b, int bf16) {
  return bf16 ? ((b & 0x7F80u) != 0x7F80u) : ((b & 0x7C00u) != 0x7C00u);
}

static int in_range(float d) {
  float a = fabsf(d);
  return a >= 8.0779356e-28f && a <= 4.2535296e37f;
}

static float markstein(float w, float d, float y) {
  volatile float q = w * y; /* RN(w * y), no contraction */
  float r = fmaf(-q, d, w);
  return fmaf(r, y, q);
}

/* 0 = ok, 1 = violation */
static int check(float w, float d) {
  const float y = 1.0f / d;
  const float x = w / d;
  const float xm = markstein(w, d, y);
  if (fabsf(x) >= 0.015625f) return memcmp(&x, &xm, 4) != 0;
  return !(fabsf(xm) < 0.03125f && fabsf(x) < 0.03125f);
}

static uint64_t rng_state = 0x243F6A8885A308D3ull;
static uint32_t rnd(void) {
  rng_state ^= rng_state << 13;
  rng_state ^= rng_state >> 7;
  rng_state ^= rng_state << 17;
  return (uint32_t)(rng_state >> 16);
}

int main(void) {
  int fail = 0;
  for (int bf16 = 0; bf16 < 2; ++bf16) {
    long long pairs[2] = {0, 0}, bad[2] = {0, 0};
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 64) reduction(+ : pairs[:2], bad[:2])
#endif
    for (int cb = 1; cb < 0x8000; ++cb) {
      if (!finite16((uint16_t)cb, bf16)) continue;
      const float c = from16((uint16_t)cb, bf16);
      const float s = c / 7.0f;
      const int ok_nf4 = in_range(c), ok_sym = in_range(s);
      /* every w with |w| <= c: magnitudes 0..cb, both signs */
      for (int wb = 0; wb <= cb; ++wb) {
        for (int sg = 0; sg < 2; ++sg) {
          const float w = from16((uint16_t)(wb | (sg << 15)), bf16);
          if (ok_nf4) { pairs[0]++; bad[0] += check(w, c); }
          if (ok_sym) { pairs[1]++; bad[1] += check(w, s); }
        }
      }
    }
    printf("%s nf4 pairs %lld violations %lld\n", bf16 ? "bf16" : "fp16", pairs[0], bad[0]);
    printf("%s int4_sym pairs %lld violations %lld\n", bf16 ? "bf16" : "fp16", pairs[1], bad[1]);
    fail |= bad[0] != 0 || bad[1] != 0;

    /* INT4 asymmetric: d = RN(RN(mx - mn) / 15) over random 16-bit group
     * ends (mn <= 0 <= mx), w between them */
    long long ap = 0, ab = 0;
    for (long long i = 0; i < 40000000LL; ++i) {
      uint16_t a = (uint16_t)(rnd() & 0x7FFF), b = (uint16_t)(rnd() & 0x7FFF);
      if (!finite16(a, bf16) || !finite16(b, bf16)) continue;
      const float mx = from16(a, bf16), mn = -from16(b, bf16);
      const float d = (mx - mn) / 15.0f;
      if (d == 0.0f || !in_range(d)) continue;
      uint16_t wb = (uint16_t)(rnd() & 0xFFFF);
      if (!finite16(wb, bf16)) continue;
      const float w = from16(wb, bf16);
      if (w < mn || w > mx) continue;
      ap++;
      ab += check(w, d);
    }
    printf("%s int4_asym sampled %lld violations %lld\n", bf16 ? "bf16" : "fp16", ap, ab);
    fail |= ab != 0;
  }
  return fail;
}
