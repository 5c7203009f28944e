/*
 * q4_oracle.c -- the CPU oracle for blockwise 4-bit weight quantization
 * (NF4 absmax, INT4 symmetric, INT4 asymmetric with zero-point, double
 * quantization of the absmax) and for the matmul that consumes it.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file: it is used by tests/, by __graft_entry__.smoke() and by the
 * cpu_baseline / --impl reference legs of bench.py.  It shares no code, no
 * header, no table and no constant with the CUDA library; the NF4 codebook
 * below is transcribed from the page, independently of the library's copy.
 *
 * Plain scalar C99.  Build: gcc -O2 -ffp-contract=off -fno-fast-math
 * (-fopenmp optional: the parallel loops touch disjoint outputs and do not
 * change any arithmetic or its order).  All floating point is IEEE binary32 /
 * binary64 with round-to-nearest-even, no contraction into FMA.
 *
 * Sources (web pages, cited by title and section):
 *  [BWQ]  learn.pranaymahendrakar.com, "Loading a model in 4-bit",
 *         section "Block-wise quantisation, stated exactly".
 *  [NF4]  n4n.ai, "What is 4-bit quantization and why does it matter?",
 *         code block "Conceptual NF4 dequantization" (levels and the
 *         dequantize_nf4 snippet) and the "INT4 symmetric" paragraph.
 *  [INT4] robotsatlas.com, "INT4", sections "How it works", "Key mechanisms"
 *         and "Components" (levels 0..15 / -8..7, per-group scale,
 *         integer zero-point).
 *  [BNB]  mbrenndoerfer.com, "INT4 Quantization > Practical Implementation
 *         with bitsandbytes" (dequantize to fp16, then a 16-bit matmul).
 *
 * Readings where the pages are silent:
 *  - ties in nearest-level coding go to the level of smaller magnitude;
 *  - an all-zero block has c = 0, every x = 0, and dequantizes to 0;
 *  - INT4 asymmetric widens [min, max] to include 0; scale and zero-point
 *    are s = (mx - mn) / 15 and z = clamp(rint(-mn / s), 0, 15);
 *  - double quantization is symmetric linear int8 (the INT4-symmetric rule
 *    with 127) of (c - mu) per group of 256 blocks, mu = mean of all c
 *    computed as a pairwise (level-by-level) fp64 sum rounded to fp32;
 *  - NF4 codes are computed from the original c; dequantization uses the
 *    double-dequantized c~.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { QT_NF4 = 0, QT_INT4_SYM = 1, QT_INT4_ASYM = 2 };

/* The 16 NF4 levels exactly as printed in [NF4] (three decimals), read as
 * binary32.  Index 7 is the exact zero; index 0 is -1 and index 15 is +1. */
static const float NF4_LEVELS[16] = {
    -1.0f,  -0.696f, -0.525f, -0.395f, -0.284f, -0.185f, -0.091f, 0.0f,
    0.079f, 0.161f,  0.246f,  0.338f,  0.441f,  0.562f,  0.720f,  1.0f};

#define DQ_GROUP 256 /* [BWQ]: the block scales are quantized in blocks of 256 */

/* ------------------------------------------------------------------------ */
/* 16-bit float formats, written out from the IEEE 754 definitions.          */
/* ------------------------------------------------------------------------ */

static float bits_to_f32(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t f32_to_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits. */
float oracle_half_to_float(uint16_t h) {
  int sign = (h >> 15) & 1, e = (h >> 10) & 31, m = h & 1023;
  double v;
  if (e == 31) return bits_to_f32((sign ? 0x80000000u : 0u) | 0x7F800000u | (m ? 0x400000u : 0u));
  if (e == 0) v = ldexp((double)m, -24);               /* subnormal: m * 2^-24 */
  else v = ldexp((double)(1024 + m), e - 25);          /* (1 + m/1024) * 2^(e-15) */
  return (float)(sign ? -v : v);                       /* exact: 11 bits fit */
}

/* bfloat16: the top 16 bits of a binary32. */
float oracle_bf16_to_float(uint16_t b) { return bits_to_f32((uint32_t)b << 16); }

/* Round a finite |v| (exact double) to a float format with p significand bits,
 * minimum normal exponent emin and maximum finite value maxv, ties to even.
 * Returns the rounded magnitude as a double (or INFINITY on overflow). */
static double round_to_format(double v, int p, int emin, double maxv) {
  if (v == 0.0) return 0.0;
  int e;
  frexp(v, &e);                                        /* v = f * 2^e, f in [0.5,1) */
  int exp_unbiased = e - 1;                            /* v in [2^(e-1), 2^e) */
  if (exp_unbiased < emin) exp_unbiased = emin;        /* subnormal quantum */
  double quantum = ldexp(1.0, exp_unbiased - (p - 1));
  double r = nearbyint(v / quantum);                   /* exact scaling; RNE */
  double out = r * quantum;
  /* overflow: anything that rounds above the largest finite value */
  if (out > maxv) return INFINITY;
  return out;
}

uint16_t oracle_float_to_half(float f) {
  uint32_t u = f32_to_bits(f);
  uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
  if ((u & 0x7F800000u) == 0x7F800000u)                /* inf / nan */
    return sign | 0x7C00u | ((u & 0x7FFFFFu) ? 0x200u : 0u);
  double a = fabs((double)f);
  double r = round_to_format(a, 11, -14, 65504.0);
  if (isinf(r)) return sign | 0x7C00u;
  if (r < ldexp(1.0, -14))                              /* subnormal or zero */
    return sign | (uint16_t)(r / ldexp(1.0, -24));
  int e; double fr = frexp(r, &e);                      /* r = fr * 2^e */
  uint16_t m = (uint16_t)((fr * 2.0 - 1.0) * 1024.0);
  return sign | (uint16_t)((e - 1 + 15) << 10) | m;
}

uint16_t oracle_float_to_bf16(float f) {
  uint32_t u = f32_to_bits(f);
  uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
  if ((u & 0x7F800000u) == 0x7F800000u)
    return sign | 0x7F80u | ((u & 0x7FFFFFu) ? 0x40u : 0u);
  double a = fabs((double)f);
  double maxv = ldexp(255.0, 127 - 7);                  /* (2 - 2^-7) * 2^127 */
  double r = round_to_format(a, 8, -126, maxv);
  if (isinf(r)) return sign | 0x7F80u;
  float rf = (float)r;                                  /* exact: 8 bits fit */
  return (uint16_t)(f32_to_bits(rf) >> 16) | sign;
}

static float to_f32(uint16_t v, int is_bf16) {
  return is_bf16 ? oracle_bf16_to_float(v) : oracle_half_to_float(v);
}
static uint16_t from_f32(float f, int is_bf16) {
  return is_bf16 ? oracle_float_to_bf16(f) : oracle_float_to_half(f);
}

/* ------------------------------------------------------------------------ */
/* Nearest-level coding ([BWQ]: "mapped to the nearest of 2^4 codebook      */
/* entries after dividing by c").                                           */
/* ------------------------------------------------------------------------ */

/* argmin_i |x - L_i| by brute force.  Distances are binary64: for |x| >=
 * 2^-30 the difference of two binary32 values in [-1, 1] needs at most 51
 * significant bits, so it is exact; for smaller |x| the nearest level is 0
 * by a margin of 0.079, far above any rounding.  Ties (the pages are
 * silent) go to the level of smaller magnitude. */
int oracle_nf4_code(float x) {
  int best = 0;
  double bestd = fabs((double)x - (double)NF4_LEVELS[0]);
  for (int i = 1; i < 16; i++) {
    double d = fabs((double)x - (double)NF4_LEVELS[i]);
    if (d < bestd || (d == bestd && fabsf(NF4_LEVELS[i]) < fabsf(NF4_LEVELS[best]))) {
      best = i;
      bestd = d;
    }
  }
  return best;
}

float oracle_nf4_level(int i) { return NF4_LEVELS[i & 15]; }

/* ------------------------------------------------------------------------ */
/* Quantize.                                                                */
/* ------------------------------------------------------------------------ */

static void put_nibble(uint8_t *buf, int64_t j, int v) {
  /* [NF4] dequantize_nf4 unpacks `p & 0xF` first, `(p >> 4) & 0xF` second:
   * element 2j is the low nibble of byte j, element 2j+1 the high nibble. */
  if (j & 1) buf[j >> 1] = (uint8_t)((buf[j >> 1] & 0x0F) | ((v & 15) << 4));
  else buf[j >> 1] = (uint8_t)((buf[j >> 1] & 0xF0) | (v & 15));
}
static int get_nibble(const uint8_t *buf, int64_t j) {
  return (j & 1) ? (buf[j >> 1] >> 4) & 15 : buf[j >> 1] & 15;
}

static int clampi(int v, int lo, int hi) { return v < lo ? lo : (v > hi ? hi : v); }

/* The pairwise fp64 sum used for the double-quantization mean: level by
 * level, adjacent pairs are added (x[2i] + x[2i+1]) and an odd last element
 * is carried up unchanged, until one value remains.  `v` is overwritten. */
double oracle_pairwise_sum(double *v, int64_t n) {
  if (n <= 0) return 0.0;
  while (n > 1) {
    int64_t half = n / 2;
    for (int64_t i = 0; i < half; i++) v[i] = v[2 * i] + v[2 * i + 1];
    if (n & 1) { v[half] = v[n - 1]; n = half + 1; }
    else n = half;
  }
  return v[0];
}

/*
 * oracle_quantize: W (n 16-bit floats, flattened row-major) -> packed codes
 * and per-block state.  Blocks are contiguous runs of `blocksize` elements
 * [BWQ]; the last block holds the remainder.  nb = ceil(n / blocksize).
 *
 *  NF4       ([BWQ], [NF4]): c = max|w|; x = w / c (binary32, correctly
 *            rounded); code = nearest level; absmax[b] = c.
 *  INT4_SYM  ([NF4] "INT4 symmetric", [INT4]): s = c / 7; q = clamp(rint(w /
 *            s), -8, 7) stored as the two's-complement nibble; absmax[b] = s.
 *  INT4_ASYM ([INT4] "How it works", "Components"): mn = min(min w, 0), mx =
 *            max(max w, 0); s = (mx - mn) / 15; z = clamp(rint(-mn / s), 0,
 *            15); q = clamp(rint(w / s) + z, 0, 15); absmax[b] = s and the
 *            zero-point nibble b of `zero` = z.
 *  scale_f16 (INT4 only, [INT4] "Components": the per-group scale is
 *            "usually stored in FP16"): s is rounded to binary16 (IEEE,
 *            ties to even) as soon as it is formed, and z and every q are
 *            computed against that rounded s; absmax[b] holds its value.
 *  double_quant (NF4 only, [BWQ] "quantises the per-block scales
 *            themselves (blocks of 256, to 8 bits)"): mu = fp32(S / nb) with
 *            S the pairwise fp64 sum of all c; per group g of 256 blocks:
 *            m2 = max|c - mu|, s2 = m2 / 127, q2 = clamp(rint((c - mu) / s2),
 *            -128, 127) (q2 = 0 when s2 = 0).  Outputs absmax_q[nb],
 *            absmax_scale[ceil(nb/256)], absmax_mean[1].  absmax keeps c.
 *
 * Outputs must be sized by the caller; packed must hold ceil(n/2) bytes and
 * is fully written (an odd n leaves the final high nibble 0).
 */
void oracle_quantize_s(const uint16_t *w, int is_bf16, int64_t n, int blocksize, int qtype,
                       int double_quant, int scale_f16, uint8_t *packed, float *absmax, uint8_t *zero,
                       int8_t *absmax_q, float *absmax_scale, float *absmax_mean) {
  int64_t nb = (n + blocksize - 1) / blocksize;
  memset(packed, 0, (size_t)((n + 1) / 2));
  if (qtype == QT_INT4_ASYM) memset(zero, 0, (size_t)((nb + 1) / 2));

#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
  for (int64_t b = 0; b < nb; b++) {
    int64_t lo = b * blocksize, hi = lo + blocksize < n ? lo + blocksize : n;
    if (qtype == QT_NF4) {
      float c = 0.0f;
      for (int64_t j = lo; j < hi; j++) {
        float a = fabsf(to_f32(w[j], is_bf16));
        if (a > c) c = a;
      }
      absmax[b] = c;
      for (int64_t j = lo; j < hi; j++) {
        float x = (c == 0.0f) ? 0.0f : to_f32(w[j], is_bf16) / c;
        put_nibble(packed, j, oracle_nf4_code(x));
      }
    } else if (qtype == QT_INT4_SYM) {
      float c = 0.0f;
      for (int64_t j = lo; j < hi; j++) {
        float a = fabsf(to_f32(w[j], is_bf16));
        if (a > c) c = a;
      }
      float s = c / 7.0f;
      if (scale_f16) s = oracle_half_to_float(oracle_float_to_half(s));
      absmax[b] = s;
      for (int64_t j = lo; j < hi; j++) {
        int q = 0;
        if (s != 0.0f) q = clampi((int)rintf(to_f32(w[j], is_bf16) / s), -8, 7);
        put_nibble(packed, j, q & 15);
      }
    } else { /* QT_INT4_ASYM */
      float mn = 0.0f, mx = 0.0f;
      for (int64_t j = lo; j < hi; j++) {
        float v = to_f32(w[j], is_bf16);
        if (v < mn) mn = v;
        if (v > mx) mx = v;
      }
      float s = (mx - mn) / 15.0f;
      if (scale_f16) s = oracle_half_to_float(oracle_float_to_half(s));
      int z = 0;
      if (s != 0.0f) z = clampi((int)rintf(-mn / s), 0, 15);
      absmax[b] = s;
      /* zero-points are packed like codes: group b -> nibble b */
#ifdef _OPENMP
#pragma omp critical
#endif
      put_nibble(zero, b, z);
      for (int64_t j = lo; j < hi; j++) {
        int q = 0;
        if (s != 0.0f) q = clampi((int)rintf(to_f32(w[j], is_bf16) / s) + z, 0, 15);
        put_nibble(packed, j, q);
      }
    }
  }
  /* put_nibble on packed is race-free only if blocks own whole bytes: with an
   * odd blocksize two blocks could share a byte.  Blocksizes are even. */

  if (double_quant && qtype == QT_NF4) {
    double *tmp = (double *)malloc(sizeof(double) * (size_t)(nb > 0 ? nb : 1));
    for (int64_t b = 0; b < nb; b++) tmp[b] = (double)absmax[b];
    double S = oracle_pairwise_sum(tmp, nb);
    free(tmp);
    float mu = (float)(S / (double)nb);
    absmax_mean[0] = mu;
    int64_t ng = (nb + DQ_GROUP - 1) / DQ_GROUP;
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
    for (int64_t g = 0; g < ng; g++) {
      int64_t lo = g * DQ_GROUP, hi = lo + DQ_GROUP < nb ? lo + DQ_GROUP : nb;
      float m2 = 0.0f;
      for (int64_t b = lo; b < hi; b++) {
        float d = fabsf(absmax[b] - mu);
        if (d > m2) m2 = d;
      }
      float s2 = m2 / 127.0f;
      absmax_scale[g] = s2;
      for (int64_t b = lo; b < hi; b++) {
        int q2 = 0;
        if (s2 != 0.0f) q2 = clampi((int)rintf((absmax[b] - mu) / s2), -128, 127);
        absmax_q[b] = (int8_t)q2;
      }
    }
  }
}

/* oracle_quantize_s with binary32 scales. */
void oracle_quantize(const uint16_t *w, int is_bf16, int64_t n, int blocksize, int qtype,
                     int double_quant, uint8_t *packed, float *absmax, uint8_t *zero,
                     int8_t *absmax_q, float *absmax_scale, float *absmax_mean) {
  oracle_quantize_s(w, is_bf16, n, blocksize, qtype, double_quant, 0, packed, absmax, zero, absmax_q,
                    absmax_scale, absmax_mean);
}

/* ------------------------------------------------------------------------ */
/* Dequantize ([NF4] dequantize_nf4: NF4_VALUES[idx] * scale per block;      */
/* [BWQ]: w^ = c * Q[i]).  One binary32 multiply, then one rounding to the    */
/* 16-bit output format.                                                     */
/* ------------------------------------------------------------------------ */

/* Per-block scale as dequantization sees it: c, or c~ = q2 * s2 + mu with two
 * separately rounded binary32 operations when double_quant is set. */
static float block_scale(const float *absmax, const int8_t *absmax_q, const float *absmax_scale,
                         const float *absmax_mean, int double_quant, int64_t b) {
  if (!double_quant) return absmax[b];
  float t = (float)absmax_q[b] * absmax_scale[b / DQ_GROUP];
  return t + absmax_mean[0];
}

/* The binary32 product for every element, before rounding to 16 bits. */
void oracle_dequantize_f32(const uint8_t *packed, const float *absmax, const uint8_t *zero,
                           const int8_t *absmax_q, const float *absmax_scale,
                           const float *absmax_mean, int64_t n, int blocksize, int qtype,
                           int double_quant, float *out) {
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
  for (int64_t j = 0; j < n; j++) {
    int64_t b = j / blocksize;
    float sc = block_scale(absmax, absmax_q, absmax_scale, absmax_mean, double_quant, b);
    int code = get_nibble(packed, j);
    float v;
    if (qtype == QT_NF4) v = sc * NF4_LEVELS[code];
    else if (qtype == QT_INT4_SYM) v = (float)(code >= 8 ? code - 16 : code) * sc;
    else v = (float)(code - get_nibble(zero, b)) * sc;
    out[j] = v;
  }
}

void oracle_dequantize(const uint8_t *packed, const float *absmax, const uint8_t *zero,
                       const int8_t *absmax_q, const float *absmax_scale,
                       const float *absmax_mean, int64_t n, int blocksize, int qtype,
                       int double_quant, int out_bf16, uint16_t *out) {
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
  for (int64_t j = 0; j < n; j++) {
    int64_t b = j / blocksize;
    float sc = block_scale(absmax, absmax_q, absmax_scale, absmax_mean, double_quant, b);
    int code = get_nibble(packed, j);
    float v;
    if (qtype == QT_NF4) v = sc * NF4_LEVELS[code];
    else if (qtype == QT_INT4_SYM) v = (float)(code >= 8 ? code - 16 : code) * sc;
    else v = (float)(code - get_nibble(zero, b)) * sc;
    out[j] = from_f32(v, out_bf16);
  }
}

/* ------------------------------------------------------------------------ */
/* The consumer ([BNB]: weights are dequantized to the compute dtype and a   */
/* 16-bit matmul follows; [BWQ] "Where the accuracy goes": Linear4bit        */
/* dequantises to compute_dtype and runs a standard 16-bit GEMM).            */
/* Y[m, r] = sum_k A[m, k] * W^[row_r, k] in binary64, where W^ is the       */
/* 16-bit dequantized weight [N, K] row-major and A is [M, K] row-major.     */
/* rows == NULL means all N rows (r = n).                                    */
/* ------------------------------------------------------------------------ */
void oracle_matmul(const uint16_t *A, int a_bf16, int64_t M, const uint16_t *W, int w_bf16,
                   int64_t N, int64_t K, const int64_t *rows, int64_t nrows, double *Y) {
  int64_t R = rows ? nrows : N;
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
  for (int64_t r = 0; r < R; r++) {
    int64_t nrow = rows ? rows[r] : r;
    const uint16_t *wr = W + nrow * K;
    for (int64_t m = 0; m < M; m++) {
      const uint16_t *ar = A + m * K;
      double acc = 0.0;
      for (int64_t k = 0; k < K; k++)
        acc += (double)to_f32(ar[k], a_bf16) * (double)to_f32(wr[k], w_bf16);
      Y[m * R + r] = acc;
    }
  }
}

/* Thread control for the timed CPU baseline. */
int oracle_set_threads(int t) {
#ifdef _OPENMP
  if (t > 0) omp_set_num_threads(t);
  return omp_get_max_threads();
#else
  (void)t;
  return 1;
#endif
}
