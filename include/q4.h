/*
 * q4.h -- C ABI of libq4.so: blockwise 4-bit weight quantization and its
 * fused consumers on NVIDIA B200 (sm_100a).
 *
 * What the operations compute is defined by these pages (cited by title and
 * section):
 *  [BWQ]  learn.pranaymahendrakar.com, "Loading a model in 4-bit", section
 *         "Block-wise quantisation, stated exactly": contiguous blocks of B,
 *         c = max|w| per block, each weight mapped to the nearest of 16
 *         codebook entries after dividing by c, w^ = c * Q[i]; double
 *         quantization of the block scales "blocks of 256, to 8 bits";
 *         section "Where the accuracy goes": dequantize to the compute dtype,
 *         then a standard 16-bit matmul.
 *  [NF4]  n4n.ai, "What is 4-bit quantization and why does it matter?", code
 *         block "Conceptual NF4 dequantization": the 16 NF4 levels and
 *         dequantize_nf4(packed_uint8, scale, block_size) with the low
 *         nibble unpacked first; "INT4 symmetric": levels -8..7, scale
 *         max|w|/7; "Why it matters for deployment": decode at batch < 32 is
 *         bound by reading the weights.
 *  [INT4] robotsatlas.com, "INT4", "How it works" and "Components": a group
 *         range fit into [0,15] with an integer zero-point (asymmetric) or
 *         [-8,7] without (symmetric).
 *  [BNB]  mbrenndoerfer.com, "INT4 Quantization > Practical Implementation
 *         with bitsandbytes": the knobs quant_type / compute_dtype /
 *         use_double_quant, and dequantize-then-16-bit-matmul.
 *
 * Conventions for every entry point:
 *  - Return Q4_OK (0) or a negative Q4_ERR_* code; q4_strerror() names it.
 *    Invalid arguments are rejected on the host before anything is launched.
 *  - Pointers named as device memory are caller-owned device memory of the
 *    current CUDA device; the library never allocates, frees or copies
 *    between host and device, and never synchronizes (except the two
 *    q4_*device_status calls, which read one device word synchronously).
 *  - All work is enqueued asynchronously on `stream` (a cudaStream_t passed
 *    as void*; NULL is the legacy default stream).
 *  - There is no CPU fallback: without an sm_100 device the compute calls
 *    return Q4_ERR_NO_DEVICE or Q4_ERR_ARCH.
 *  - Weights are W[rows = N, cols = K] row-major (nn.Linear, out x in); the
 *    blocks of [BWQ] run over the flattened row-major order.  Activations
 *    are A[M, K] row-major; outputs Y[M, N] row-major; Y = A . W^T.
 */
#ifndef Q4_H
#define Q4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exported symbols of libq4.so (everything else in the library is hidden). */
#if defined(__GNUC__)
#define Q4_API __attribute__((visibility("default")))
#else
#define Q4_API
#endif

/* ---- status codes ------------------------------------------------------ */
#define Q4_OK 0
#define Q4_ERR_ARG (-1)        /* bad enum, NULL pointer, unsupported combination */
#define Q4_ERR_SHAPE (-2)      /* sizes out of range / not block-aligned */
#define Q4_ERR_ALIGN (-3)      /* a pointer is not 16-byte aligned */
#define Q4_ERR_NO_DEVICE (-4)  /* no CUDA device visible */
#define Q4_ERR_ARCH (-5)       /* the device is not sm_100 */
#define Q4_ERR_CUDA (-6)       /* a CUDA runtime call or launch failed */
#define Q4_ERR_WORKSPACE (-7)  /* workspace NULL or smaller than required */

/* Sticky device status bits (q4_device_status). */
#define Q4_STATUS_NONFINITE 1  /* quantize met a block with a non-finite absmax */
#define Q4_STATUS_TIMEOUT 2    /* a bounded device-side wait gave up */
#define Q4_STATUS_LAYOUT 4     /* a kernel found too little shared memory and computed nothing */

/* ---- enums ------------------------------------------------------------- */
typedef enum {
  Q4_NF4 = 0,       /* [BWQ]/[NF4]: absmax per block, 16 NF4 levels */
  Q4_INT4_SYM = 1,  /* [NF4]/[INT4]: s = max|w|/7, q in [-8, 7] */
  Q4_INT4_ASYM = 2  /* [INT4]: s = (max - min)/15, integer zero-point z in [0, 15] */
} q4_qtype;

typedef enum { Q4_F16 = 0, Q4_BF16 = 1, Q4_F32 = 2 /* outputs only */ } q4_dtype;

/* OR'ed into an INT4 qtype (Q4_INT4_SYM | Q4_SCALE_F16, Q4_INT4_ASYM |
 * Q4_SCALE_F16) at q4_state_sizes / q4_quantize*: the group scale is stored
 * as binary16 ([INT4] "Components": the per-group scale is "usually stored
 * in FP16").  s is rounded to binary16 (round to nearest even) as soon as
 * it is formed, and the zero-point and every code are computed against the
 * rounded s; the state's qtype keeps the plain INT4 value and its
 * scale_f16 field is 1.  Not defined for NF4 (Q4_ERR_ARG). */
#define Q4_SCALE_F16 0x100

#define Q4_DQ_GROUP 256 /* [BWQ]: the block scales are quantized in blocks of 256 */

/*
 * A quantized tensor.  The caller allocates the device buffers with the
 * sizes q4_state_sizes() returns and sets the six pointers; q4_quantize
 * fills every other field and the buffers.  Layout in device memory:
 *   packed       uint8 [ceil(n/2)]: element 2j in the low nibble of byte j,
 *                element 2j+1 in the high nibble ([NF4] unpack order); NF4 and
 *                INT4_ASYM codes are 0..15, INT4_SYM codes are the
 *                two's-complement nibble of q in [-8, 7].
 *   absmax       float [nb], nb = ceil(n / blocksize): the NF4 absmax c, or
 *                the INT4 scale s.  With double_quant it still holds c.
 *                With scale_f16 it holds binary16 [nb] (the pointer type is
 *                unchanged; the buffer is nb * 2 bytes).
 *   zero         uint8 [ceil(nb/2)] (INT4_ASYM only, else NULL): zero-point
 *                of block b in nibble b, low nibble first.
 *   absmax_q     int8 [nb] (double_quant only, else NULL): 8-bit code of c.
 *   absmax_scale float [ceil(nb/256)] (double_quant only): second-level scale.
 *   absmax_mean  float [1] (double_quant only): the mean subtracted from c.
 */
typedef struct {
  int32_t qtype;        /* q4_qtype */
  int32_t src_dtype;    /* q4_dtype of the quantized input (F16 / BF16) */
  int64_t n;            /* number of weights = rows * cols */
  int64_t rows, cols;   /* N, K */
  int32_t blocksize;    /* B: 32, 64, 128 or 256 */
  int32_t double_quant; /* 0 / 1 (NF4 only) */
  int32_t dq_group;     /* Q4_DQ_GROUP */
  int32_t scale_f16;    /* 0 / 1: binary16 INT4 scales (see Q4_SCALE_F16) */
  uint8_t *packed;
  float *absmax;
  uint8_t *zero;
  int8_t *absmax_q;
  float *absmax_scale;
  float *absmax_mean;
} q4_state;

/* ---- sizes (host only, no device needed) ------------------------------ */

/* Byte sizes of the six state buffers, in struct order (0 for an unused
 * buffer).  Errors: Q4_ERR_ARG for a bad qtype / blocksize / double_quant
 * combination (double quantization is defined for the NF4 absmax only),
 * Q4_ERR_SHAPE for n < 1. */
Q4_API int q4_state_sizes(int32_t qtype, int64_t n, int32_t blocksize, int32_t double_quant,
                   size_t sizes_out[6]);

/* Device workspace q4_quantize needs (0 without double quantization).  The
 * workspace must be zero-filled before its first use; every call leaves it
 * zero-filled again, so one allocation serves all later calls on one stream
 * (calls that run concurrently need separate workspaces). */
Q4_API int q4_quantize_workspace_size(int32_t qtype, int64_t n, int32_t blocksize, int32_t double_quant,
                               size_t *bytes);

/* ---- quantize --------------------------------------------------------- */

/*
 * q4_quantize -- load-time blockwise quantization ([BWQ]; [BNB] "load-time
 * quantization", no calibration data).
 *   W          device, 16-byte aligned, rows*cols 16-bit floats of w_dtype
 *              (Q4_F16 / Q4_BF16), row-major.
 *   blocksize  32, 64, 128 or 256 (64 is the [BWQ] default for NF4).
 *   qtype      Q4_NF4 / Q4_INT4_SYM / Q4_INT4_ASYM, the INT4 ones
 *              optionally | Q4_SCALE_F16.
 *   double_quant  0 or 1; 1 only with Q4_NF4.
 *   out        host struct; its six pointers must already point to device
 *              buffers of q4_state_sizes() bytes (packed/absmax 16-byte
 *              aligned); the scalar fields are written by this call.
 *   workspace  device, q4_quantize_workspace_size() bytes, zero-filled
 *              (may be NULL when that size is 0).
 * Arithmetic: IEEE binary32, correctly rounded division, round-half-even
 * rint; codes, packed bytes, absmax, zero-points and the double-quant state
 * are bit-exact functions of W.  NF4 ties go to the level nearer zero.
 * Non-finite inputs give unspecified codes and set Q4_STATUS_NONFINITE.
 */
Q4_API int q4_quantize(const void *W, int32_t w_dtype, int64_t rows, int64_t cols, int32_t blocksize,
                int32_t qtype, int32_t double_quant, q4_state *out, void *workspace,
                size_t workspace_bytes, void *stream);

/*
 * q4_quantize_noalloc -- q4_quantize for callers that cannot allocate device
 * memory when they quantize (a plugin whose host application owns every
 * device allocation, a latency-critical path that must not pay for the
 * device-wide synchronization of cudaMalloc/cudaFree, a runtime that reserves
 * all memory at start-up).  It takes the same arguments as q4_quantize minus
 * the workspace: the caller still passes W and the output state buffers.
 * The pages have no counterpart to this call; it exists only for those
 * callers.
 *   Scratch: a fixed array of Q4_NOALLOC_SCRATCH_BYTES in the library's own
 *   static device memory, held by every GPU that loads the library until the
 *   process exits.  Its device address is looked up on the first call on
 *   each device (with that device current); make that first call before any
 *   stream capture.  Each call clears the part it uses with an asynchronous
 *   memset on `stream`, and no call allocates or frees device memory.
 *   All calls on a device share the array and it keeps the last call's
 *   contents: calls that overlap on the GPU (different streams, or the same
 *   call from several threads at once) race on it and must be serialized by
 *   the caller.
 *   Limit: returns Q4_ERR_WORKSPACE if the workspace q4_quantize would need
 *   (q4_quantize_workspace_size) exceeds Q4_NOALLOC_SCRATCH_BYTES; every
 *   other error is that of q4_quantize.
 */
#define Q4_NOALLOC_SCRATCH_BYTES 32768
Q4_API int q4_quantize_noalloc(const void *W, int32_t w_dtype, int64_t rows, int64_t cols,
                               int32_t blocksize, int32_t qtype, int32_t double_quant,
                               q4_state *out, void *stream);

/*
 * q4_quantize_grouped -- q4_quantize of `count` (1..16) matrices in one
 * launch (plus one launch of the second-level quantization with
 * double_quant), e.g. the seven projections of a decoder layer at load time.
 * One format for all: w_dtype, blocksize, qtype and double_quant are
 * shared; W[i] is [rows[i], cols[i]] and out[i] its state, with the rules
 * and results of q4_quantize for each (bit for bit the same state).
 * Runs one CTA per SM over the 256-block chunks of all matrices; W[i] must
 * be 16-byte aligned (its pieces are copied by the bulk-copy engine).
 * With double_quant, a matrix may hold at most 65536 groups of 256 blocks
 * (Q4_ERR_SHAPE otherwise: e.g. 2^30 weights at blocksize 64).
 *   workspace  device, q4_quantize_grouped_workspace_size() bytes,
 *              zero-filled; every call leaves it zero-filled (after a
 *              Q4_STATUS_TIMEOUT it must be zero-filled again).
 */
Q4_API int q4_quantize_grouped_workspace_size(int32_t count, const int64_t *rows, const int64_t *cols,
                                              int32_t blocksize, int32_t qtype, int32_t double_quant,
                                              size_t *bytes);
Q4_API int q4_quantize_grouped(int32_t count, const void *const *W, int32_t w_dtype, const int64_t *rows,
                               const int64_t *cols, int32_t blocksize, int32_t qtype, int32_t double_quant,
                               q4_state *const *out, void *workspace, size_t workspace_bytes, void *stream);

/* ---- dequantize ------------------------------------------------------- */

/*
 * q4_dequantize -- [NF4] dequantize_nf4 / [BWQ] w^ = c * Q[i]:
 *   out[j] = cvt_rn(c~_b * level(code_j)), one binary32 multiply rounded once
 *   to out_dtype (Q4_F16 / Q4_BF16), where c~ = q2 * s2 + mu (two separately
 *   rounded operations) with double quantization, else c.  INT4_SYM level =
 *   q, INT4_ASYM level = q - z.
 *   Wq   host struct describing device buffers (as filled by q4_quantize).
 *   out  device, n elements, 16-byte aligned.
 */
Q4_API int q4_dequantize(const q4_state *Wq, void *out, int32_t out_dtype, void *stream);

/* q4_dequantize of `count` (1..16) states of one format (qtype, blocksize,
 * double_quant) in one launch; out[i] receives state i (16-byte aligned,
 * n elements of out_dtype).  Bit for bit the result of q4_dequantize. */
Q4_API int q4_dequantize_grouped(int32_t count, const q4_state *const *Wq, void *const *out, int32_t out_dtype,
                                 void *stream);

/* ---- fused dequant-GEMV (decode, M <= 32) ------------------------------ */

/* Workspace for q4_gemv / q4_gemv_grouped (fp32 partial sums and arrival
 * counters).  Zero-filled before first use; every call leaves it zeroed. */
Q4_API int q4_gemv_workspace_size(int32_t count, const q4_state *const *Wq, int64_t M, size_t *bytes);

/*
 * q4_gemv -- Y[M, N] = A[M, K] . W^[N, K]^T for 1 <= M <= 32 ([NF4] "Why it
 * matters": memory-bound decode at small batch; [BWQ]/[BNB] dequantize to
 * the compute dtype then matmul), with the dequantization fused into the
 * streaming of the packed weights and fp32 accumulation; one pass over the
 * weights for every M.
 *   A      device, a_dtype (Q4_F16 / Q4_BF16), [M, K] row-major, 16-byte
 *          aligned, K = Wq->cols.
 *   Wq     NF4 state (with or without double quantization), INT4 symmetric
 *          state (the codebook is the integers -8..7 and the group scale
 *          takes the place of c~) or INT4 asymmetric state (codes 0..15,
 *          w^ = (q - z) s: the kernel subtracts z times each block's
 *          activation sum); K % blocksize == 0, blocksize in {32, 64, 128,
 *          256}.
 *   Y      device, y_dtype (Q4_F16 / Q4_BF16 / Q4_F32), [M, N] row-major.
 *   workspace  device, q4_gemv_workspace_size() bytes, zero-filled.
 * Result: within relative Frobenius error 1e-3 of the binary64 product of A
 * and the 16-bit dequantized weights (rounded once to y_dtype).  The
 * summation order is fixed: identical calls give identical bits.
 */
Q4_API int q4_gemv(const void *A, int32_t a_dtype, int64_t M, const q4_state *Wq, void *Y,
            int32_t y_dtype, void *workspace, size_t workspace_bytes, void *stream);

/* q4_gemv over `count` (1..16) independent matrices in ONE launch (e.g. the
 * seven projections of a decoder layer); one format per call.  A[i], Wq[i], Y[i] are host arrays
 * of device pointers / host structs; M, dtypes and the rules of q4_gemv
 * apply to every entry. */
Q4_API int q4_gemv_grouped(int32_t count, const void *const *A, const q4_state *const *Wq,
                    void *const *Y, int64_t M, int32_t a_dtype, int32_t y_dtype, void *workspace,
                    size_t workspace_bytes, void *stream);

/* ---- W4A16 GEMM (prefill, large M) ------------------------------------ */

/* Workspace for q4_gemm / q4_gemm_grouped: room for fp32 partial tiles and
 * arrival counters when the launch cuts tiles in halves of their k range
 * to even out the CTAs' work (a launch of few tiles, or of matrices with
 * very different K).  0 when no cut pays off.  The size depends on the
 * shapes, M and the current device's SM count.  Its first 64 KB hold the
 * arrival counters (at that fixed place whatever the call), the partial
 * tiles follow.  Zero-filled before first use; every call leaves the
 * counters zeroed (after Q4_STATUS_TIMEOUT, zero-fill it again). */
Q4_API int q4_gemm_workspace_size(int32_t count, const q4_state *const *Wq, int64_t M, size_t *bytes);

/* How a q4_gemm_grouped launch over these matrices would run on a device of
 * `sms` streaming multiprocessors with `workspace_bytes` of workspace
 * (SIZE_MAX: as much as q4_gemm_workspace_size asks for): the tokens per
 * output tile (*tile_m: 512, or 256 for launches of few tiles and for M <=
 * 256), the CTAs of the grid (*grid) and the tiles cut in halves of their k
 * range (*cut_tiles).  Host only: it reads the states' shapes and formats,
 * touches no device and allocates nothing; the same shape and format
 * checks as q4_gemm_workspace_size (Q4_ERR_ARG / Q4_ERR_SHAPE), and sms
 * outside 1 .. 1024 is Q4_ERR_ARG.  The planning it reports: the host deals
 * work items longest first onto the least-loaded CTA, for both tile
 * heights, and keeps the height whose busiest CTA finishes first. */
Q4_API int q4_gemm_plan_info(int32_t count, const q4_state *const *Wq, int64_t M, int32_t sms,
                             size_t workspace_bytes, int32_t *tile_m, int32_t *grid, int64_t *cut_tiles);

/*
 * q4_gemm -- the same product for any M >= 1, computed by dequantizing
 * weight tiles into shared memory (bit-exact w^ in a_dtype) and feeding
 * tcgen05 tensor-core MMAs with fp32 accumulators in tensor memory.
 *   A   device, a_dtype (Q4_BF16 / Q4_F16), [M, K] row-major, 16-byte aligned.
 *   Wq  any state (NF4 with or without double quantization, INT4
 *       symmetric, INT4 asymmetric; blocksize 32, 64, 128 or 256) with
 *       K % 64 == 0 (and K a multiple of the blocksize), N % 16 == 0.
 *       The weight tile is w^ = cvt(c~ * level) for NF4, cvt(s * q) for
 *       INT4 symmetric and cvt(s * (q - z)) for INT4 asymmetric: bit for
 *       bit what q4_dequantize gives.
 *   Y   device, y_dtype (a_dtype or Q4_F32), [M, N] row-major.
 *   workspace  device, 16-byte aligned, q4_gemm_workspace_size() bytes,
 *       zero-filled; or NULL / fewer bytes: then no tile is cut (the same
 *       result, only the balance of the CTAs differs).  A cut tile's two
 *       partial sums are added once, a + b, so the bits do not depend on
 *       which half finishes first.
 * Same tolerance as q4_gemv.  A grouped call takes one format (qtype,
 * blocksize, double_quant) for all its matrices (Q4_ERR_ARG otherwise).
 * Host cost: each launch is planned on the host (tile height, per-CTA
 * tile lists, cuts; q4_gemm_plan_info reports the outcome).  Planning a
 * decoder layer takes up to about a millisecond of host time; each host
 * thread keeps its last 8 plans (keyed by shapes, M, SM count and
 * workspace bytes), so repeated shapes plan once.
 */
Q4_API int q4_gemm(const void *A, int32_t a_dtype, int64_t M, const q4_state *Wq, void *Y,
            int32_t y_dtype, void *workspace, size_t workspace_bytes, void *stream);

/* q4_gemm over `count` (1..16) matrices in one persistent launch. */
Q4_API int q4_gemm_grouped(int32_t count, const void *const *A, const q4_state *const *Wq,
                    void *const *Y, int64_t M, int32_t a_dtype, int32_t y_dtype, void *workspace,
                    size_t workspace_bytes, void *stream);

/* ---- status and introspection ----------------------------------------- */

/* Bound, in nanoseconds, of every device-side wait (a pipeline barrier
 * between a kernel's copy and compute warps) of the kernels launched after
 * this call, process-wide; 0 restores the default of 2 s.  A wait that runs
 * out raises Q4_STATUS_TIMEOUT: the kernel stops, waits for its own copies
 * in flight and returns, leaving its outputs undefined.  After a timeout the
 * GEMV or grouped-quantize workspace must be zero-filled again before its
 * next use.  Host only; no device needed. */
Q4_API int q4_set_wait_limit_ns(uint64_t ns);

/* Test hook for the bounded waits, process-wide: while `on` is non-zero the
 * copy warp of the decode GEMV, the GEMM and the grouped quantize issues no
 * copies, so every compute warp's wait for a stage runs out after the wait
 * limit (set a short one first) and the call returns with
 * Q4_STATUS_TIMEOUT and undefined outputs.  Leave it off otherwise.  Host
 * only. */
Q4_API int q4_set_copy_stall(int32_t on);

/* Reads (synchronously) the sticky device status word of the current
 * device: an OR of Q4_STATUS_* bits set by kernels since the last clear. */
Q4_API int q4_device_status(int32_t *status);
Q4_API int q4_clear_device_status(void);

/* Q4_OK when the current device is an sm_100 part, else the error code. */
Q4_API int q4_check_device(void);

/* The library's NF4 codebook (the 16 printed levels as binary32) and the 15
 * decision thresholds derived from it on the host: code = #{i : x >= t_i}
 * reproduces nearest-level coding with ties toward the level nearer zero.
 * Host only. */
Q4_API int q4_nf4_levels(float out[16]);
Q4_API int q4_nf4_thresholds(float out[15]);

Q4_API const char *q4_strerror(int code);

#ifdef __cplusplus
}
#endif

#endif /* Q4_H */
