// q4_api.cu -- the C ABI of include/q4.h (libq4.so).
//
// Host side only: argument validation, launch planning, TMA descriptors and
// status codes.  Every step of the computation runs in the sm_100a kernels of
// the other translation units; the host never touches tensor data and never
// allocates device memory.
#include <cuda.h>
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <queue>
#include <vector>

#include "q4_internal.h"

namespace q4 {
__device__ int g_status = 0;
// Bound of every device-side wait of the kernels launched from now on.
std::atomic<uint64_t> g_wait_limit_ns{kWaitLimitNs};
// Test hook of the bounded waits: the GEMV copy warps issue no copies.
std::atomic<int32_t> g_copy_stall{0};
}

using namespace q4;

namespace {

// The 16 NF4 levels exactly as printed on n4n.ai, "What is 4-bit
// quantization and why does it matter?", code block "Conceptual NF4
// dequantization", read as binary32.
const float kNF4Levels[16] = {-1.0f,  -0.696f, -0.525f, -0.395f, -0.284f, -0.185f,
                              -0.091f, 0.0f,    0.079f,  0.161f,  0.246f,  0.338f,
                              0.441f,  0.562f,  0.720f,  1.0f};

// Decision thresholds of nearest-level coding: t_i is the smallest binary32 x
// whose nearest level is L_{i+1} or above.  At an exact midpoint the level of
// smaller magnitude wins (the pages give no tie rule).
void derive_thresholds(float t[15]) {
  for (int i = 0; i < 15; ++i) {
    const double lo = kNF4Levels[i], hi = kNF4Levels[i + 1];
    const double m = (lo + hi) * 0.5;  // exact in binary64
    const bool tie_goes_up = fabs(hi) < fabs(lo);
    float f = (float)m;
    if (tie_goes_up) {
      if ((double)f < m) f = nextafterf(f, INFINITY);
    } else {
      if ((double)f <= m) f = nextafterf(f, INFINITY);
    }
    t[i] = f;
  }
}

// Bin table of the quantize kernel: the bin of x is the low 5 bits of
// fmaf(x, 15, 12582927) (round(15x) + 15); each bin may hold one threshold.
bool build_bin_table(Nf4BinTable *tab) {
  float t[15];
  derive_thresholds(t);
  int bin_of[15];
  for (int i = 0; i < 15; ++i) {
    const float v = fmaf(t[i], 15.0f, 12582927.0f);
    uint32_t u;
    memcpy(&u, &v, 4);
    bin_of[i] = (int)(u & 31u);
  }
  for (int j = 0; j < 32; ++j) {
    tab->thr[j] = INFINITY;
    tab->base[j] = 0;
    int hits = 0;
    for (int i = 0; i < 15; ++i) {
      if (bin_of[i] < j) tab->base[j]++;
      if (bin_of[i] == j) {
        tab->thr[j] = t[i];
        hits++;
      }
    }
    if (hits > 1) return false;
  }
  return true;
}

struct DeviceInfo {
  int ok = Q4_ERR_NO_DEVICE;
  int sms = 0;
  int *status = nullptr;  // device address of q4::g_status
};

DeviceInfo device_info() {
  static DeviceInfo cache[64];
  static bool filled[64] = {};
  static std::mutex mu;
  int count = 0;
  if (cudaGetDeviceCount(&count) != cudaSuccess || count == 0) {
    cudaGetLastError();
    return DeviceInfo{};
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return DeviceInfo{Q4_ERR_CUDA, 0, nullptr};
  std::lock_guard<std::mutex> lk(mu);
  if (filled[dev]) return cache[dev];
  DeviceInfo d;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || d.sms < 1) {
    cudaGetLastError();
    return DeviceInfo{Q4_ERR_CUDA, 0, nullptr};  // not cached: a later call asks again
  }
  d.ok = (major == 10 && minor == 0) ? Q4_OK : Q4_ERR_ARCH;
  if (d.ok == Q4_OK) {
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, q4::g_status) != cudaSuccess) {
      cudaGetLastError();
      d.ok = Q4_ERR_CUDA;
    }
    d.status = reinterpret_cast<int *>(ptr);
  }
  cache[dev] = d;
  filled[dev] = true;
  return d;
}

inline bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }
inline bool valid_bs(int b) { return b == 32 || b == 64 || b == 128 || b == 256; }
inline bool valid_in_dtype(int d) { return d == Q4_F16 || d == Q4_BF16; }
inline bool valid_out_dtype(int d) { return d == Q4_F16 || d == Q4_BF16 || d == Q4_F32; }
inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

int check_state(const q4_state *s) {
  if (!s || !s->packed) return Q4_ERR_ARG;
  if (s->qtype < 0 || s->qtype > 2 || !valid_bs(s->blocksize)) return Q4_ERR_ARG;
  if (s->scale_f16 != 0 && (s->scale_f16 != 1 || s->qtype == Q4_NF4)) return Q4_ERR_ARG;
  if (s->double_quant) {
    if (s->qtype != Q4_NF4 || !s->absmax_q || !s->absmax_scale || !s->absmax_mean) return Q4_ERR_ARG;
  } else if (!s->absmax) {
    return Q4_ERR_ARG;
  }
  if (s->qtype == Q4_INT4_ASYM && !s->zero) return Q4_ERR_ARG;
  if (s->n < 1 || s->rows < 1 || s->cols < 1 || s->rows * s->cols != s->n) return Q4_ERR_SHAPE;
  if (!aligned16(s->packed)) return Q4_ERR_ALIGN;
  return Q4_OK;
}

// ---- GEMV planning ----------------------------------------------------------
// Every format runs the decode kernel of gemv_small.cuh in one pass for
// every M <= 32 (one, two or four column tiles of 8 activation rows).
// Tiles of 256 rows cut into 128-k stages, the stages of all matrices split
// evenly over at most kGsMaxCtas CTAs.  Workspace: a 256-byte head, the
// per-CTA partial-row slots, then per matrix one counter per 16 rows; the
// kernel leaves all of it zeroed.
constexpr size_t kGemvWsHead = 256;
size_t gemv_counters_for(const q4_state *s) { return align256((size_t)ceil_div(s->rows, 16) * 4); }
size_t gemv_ws_for(const q4_state *s, int64_t *n_tiles, int64_t *n_stages) {
  *n_tiles = ceil_div(s->rows, kGsRows);
  *n_stages = ceil_div(s->cols, kGsStageK);  // stages per tile
  return gemv_counters_for(s);
}
// Slots of the decode kernel: [grid][2][256 rows][8, 16 or 32] fp32.
size_t gemv_small_slots(int64_t total_stages, int64_t M) {
  const int64_t grid = std::min<int64_t>(total_stages, kGsMaxCtas);
  return align256((size_t)grid * 2 * kGsRows * (M <= 8 ? 8 : (M <= 16 ? 16 : 32)) * 4);
}

// ---- TMA descriptors ----------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    cudaGetLastError();
  });
  return fn;
}

// 2-D row-major tensor [rows, cols] of `esize`-byte elements, box {bx, by}.
bool make_map(CUtensorMap *m, CUtensorMapDataType dt, const void *base, int64_t rows, int64_t cols,
              int esize, int bx, int by, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(cols * esize)};
  const cuuint32_t box[2] = {(cuuint32_t)bx, (cuuint32_t)by};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The decode-batch path (M <= 16): the mma.sync kernel of gemv_small.cuh.
int gemv_small_grouped(int32_t count, const void *const *A, const q4_state *const *Wq, void *const *Y,
                       int64_t M, int32_t a_dtype, int32_t y_dtype, void *workspace, size_t workspace_bytes,
                       void *stream) {
  static thread_local GsParams p;  // host staging of the kernel parameters (~6 KB)
  memset(&p, 0, sizeof(p));
  p.count = count;
  p.M = (int)M;
  p.y_dtype = y_dtype;
  const int bs = Wq[0]->blocksize;
  const int dq = Wq[0]->double_quant;
  const int qt = Wq[0]->qtype;
  const DeviceInfo di = device_info();
  if (!workspace || workspace_bytes < kGemvWsHead) return Q4_ERR_WORKSPACE;
  int64_t total = 0;
  for (int i = 0; i < count; ++i) {
    int64_t t, q;
    gemv_ws_for(Wq[i], &t, &q);
    total += t * q;
  }
  const size_t slot_bytes = gemv_small_slots(total, M);
  int64_t stages = 0;
  size_t ws_off = kGemvWsHead + slot_bytes;
  if (ws_off > workspace_bytes) return Q4_ERR_WORKSPACE;
  p.slots = reinterpret_cast<float *>((char *)workspace + kGemvWsHead);
  for (int i = 0; i < count; ++i) {
    const q4_state *s = Wq[i];
    int rc = check_state(s);
    if (rc != Q4_OK) return rc;
    // one format per grouped call
    if (s->qtype != qt || s->blocksize != bs || s->double_quant != dq) return Q4_ERR_ARG;
    if (s->cols % bs || s->rows > INT32_MAX || s->cols > INT32_MAX) return Q4_ERR_SHAPE;
    if (!A[i] || !Y[i]) return Q4_ERR_ARG;
    if (!aligned16(A[i])) return Q4_ERR_ALIGN;
    if (di.ok != Q4_OK) return di.ok;
    int64_t n_tiles, n_stages;
    const size_t need = gemv_ws_for(s, &n_tiles, &n_stages);
    if (n_tiles * n_stages > INT32_MAX) return Q4_ERR_SHAPE;
    GsMat &m = p.mat[i];
    const CUtensorMapDataType adt =
        a_dtype == Q4_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    if (!make_map(&m.tmW, CU_TENSOR_MAP_DATA_TYPE_UINT8, s->packed, s->rows, s->cols / 2, 1, kGsStageK / 2, kGsRows,
                  CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map(&m.tmA, adt, A[i], M, s->cols, 2, 64, (int)M, CU_TENSOR_MAP_SWIZZLE_128B))
      return Q4_ERR_CUDA;
    m.absmax = s->absmax;
    m.absmax_q = s->absmax_q;
    m.absmax_scale = s->absmax_scale;
    m.absmax_mean = s->absmax_mean;
    m.zero = s->zero;
    m.Y = Y[i];
    m.N = (int32_t)s->rows;
    m.K = (int32_t)s->cols;
    m.n_tiles = (int32_t)n_tiles;
    m.n_stages = (int32_t)n_stages;
    m.stage_begin = (uint32_t)stages;
    stages += n_tiles * n_stages;
    if (stages * kGsMaxCtas >= ((int64_t)1 << 32)) return Q4_ERR_SHAPE;  // 32-bit stage indices
    if (ws_off + need > workspace_bytes) return Q4_ERR_WORKSPACE;
    m.cnt = reinterpret_cast<unsigned *>((char *)workspace + ws_off);
    ws_off += need;
  }
  p.dq = dq;
  p.total_stages = (uint32_t)stages;
  p.status = di.status;
  p.wait_ns = g_wait_limit_ns.load(std::memory_order_relaxed);
  p.stall_copies = g_copy_stall.load(std::memory_order_relaxed);
  p.scale_f16 = Wq[0]->scale_f16;
  if (qt == Q4_NF4) {
    memcpy(p.levels, kNF4Levels, sizeof(kNF4Levels));
  } else if (qt == Q4_INT4_SYM) {
    // INT4 symmetric: code j is the two's-complement nibble of q, w^ = q * s
    for (int j = 0; j < 16; ++j) p.levels[j] = (float)((j ^ 8) - 8);
  } else {
    // INT4 asymmetric: code j is q itself, w^ = (q - z) * s
    for (int j = 0; j < 16; ++j) p.levels[j] = (float)j;
  }
  return run_gemv_small(a_dtype, bs, (int)M, qt == Q4_INT4_ASYM, p, di.sms, (cudaStream_t)stream);
}


}  // namespace

// =============================================================================
extern "C" {

const char *q4_strerror(int code) {
  switch (code) {
    case Q4_OK: return "ok";
    case Q4_ERR_ARG: return "invalid argument";
    case Q4_ERR_SHAPE: return "invalid shape";
    case Q4_ERR_ALIGN: return "pointer not 16-byte aligned";
    case Q4_ERR_NO_DEVICE: return "no CUDA device (there is no CPU fallback)";
    case Q4_ERR_ARCH: return "device is not sm_100 (B200)";
    case Q4_ERR_CUDA: return "CUDA runtime error";
    case Q4_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown error";
}

int q4_nf4_levels(float out[16]) {
  if (!out) return Q4_ERR_ARG;
  memcpy(out, kNF4Levels, sizeof(kNF4Levels));
  return Q4_OK;
}

int q4_nf4_thresholds(float out[15]) {
  if (!out) return Q4_ERR_ARG;
  derive_thresholds(out);
  return Q4_OK;
}

int q4_check_device(void) { return device_info().ok; }

// qtype with an optional Q4_SCALE_F16: the plain qtype and the flag, or -1.
static int split_qtype(int32_t qtype, bool *f16) {
  *f16 = (qtype & Q4_SCALE_F16) != 0;
  const int32_t q = qtype & ~Q4_SCALE_F16;
  if (q < 0 || q > 2 || (*f16 && q == Q4_NF4)) return -1;
  return q;
}

int q4_state_sizes(int32_t qtype_in, int64_t n, int32_t blocksize, int32_t double_quant,
                   size_t sizes_out[6]) {
  bool f16 = false;
  const int qtype = split_qtype(qtype_in, &f16);
  if (!sizes_out || qtype < 0 || !valid_bs(blocksize) ||
      (double_quant != 0 && double_quant != 1) || (double_quant && qtype != Q4_NF4))
    return Q4_ERR_ARG;
  if (n < 1) return Q4_ERR_SHAPE;
  const int64_t nb = ceil_div(n, blocksize);
  sizes_out[0] = (size_t)((n + 1) / 2);
  sizes_out[1] = (size_t)nb * (f16 ? 2 : 4);
  sizes_out[2] = qtype == Q4_INT4_ASYM ? (size_t)((nb + 1) / 2) : 0;
  sizes_out[3] = double_quant ? (size_t)nb : 0;
  sizes_out[4] = double_quant ? (size_t)ceil_div(nb, Q4_DQ_GROUP) * 4 : 0;
  sizes_out[5] = double_quant ? 4 : 0;
  return Q4_OK;
}

int q4_quantize_workspace_size(int32_t qtype, int64_t n, int32_t blocksize, int32_t double_quant,
                               size_t *bytes) {
  size_t sz[6];
  const int rc = q4_state_sizes(qtype, n, blocksize, double_quant, sz);
  if (rc != Q4_OK) return rc;
  if (!bytes) return Q4_ERR_ARG;
  *bytes = double_quant ? (size_t)(kMaxRunPartials * 8 + 256) : 0;
  return Q4_OK;
}

int q4_quantize(const void *W, int32_t w_dtype, int64_t rows, int64_t cols, int32_t blocksize,
                int32_t qtype_in, int32_t double_quant, q4_state *out, void *workspace,
                size_t workspace_bytes, void *stream) {
  if (!W || !out || !valid_in_dtype(w_dtype)) return Q4_ERR_ARG;
  if (rows < 1 || cols < 1) return Q4_ERR_SHAPE;
  const int64_t n = rows * cols;
  size_t sz[6];
  int rc = q4_state_sizes(qtype_in, n, blocksize, double_quant, sz);
  if (rc != Q4_OK) return rc;
  bool f16 = false;
  const int qtype = split_qtype(qtype_in, &f16);
  if (!out->packed || !out->absmax || (qtype == Q4_INT4_ASYM && !out->zero)) return Q4_ERR_ARG;
  if (double_quant && (!out->absmax_q || !out->absmax_scale || !out->absmax_mean)) return Q4_ERR_ARG;
  if (!aligned16(W) || !aligned16(out->packed) || ((uintptr_t)out->absmax & (f16 ? 1u : 3u))) return Q4_ERR_ALIGN;
  size_t need = 0;
  q4_quantize_workspace_size(qtype, n, blocksize, double_quant, &need);
  if (need && (!workspace || workspace_bytes < need)) return Q4_ERR_WORKSPACE;
  const DeviceInfo di = device_info();
  if (di.ok != Q4_OK) return di.ok;

  static Nf4BinTable tab;
  static bool tab_ok = false;
  static std::once_flag once;
  std::call_once(once, [] { tab_ok = build_bin_table(&tab); });
  if (!tab_ok) return Q4_ERR_ARG;

  out->qtype = qtype;
  out->src_dtype = w_dtype;
  out->n = n;
  out->rows = rows;
  out->cols = cols;
  out->blocksize = blocksize;
  out->double_quant = double_quant;
  out->dq_group = Q4_DQ_GROUP;
  out->scale_f16 = f16 ? 1 : 0;
  if (!double_quant) out->absmax_q = nullptr, out->absmax_scale = nullptr, out->absmax_mean = nullptr;
  if (qtype != Q4_INT4_ASYM) out->zero = nullptr;

  const int64_t nb = ceil_div(n, blocksize);
  const int64_t n_chunks = ceil_div(nb, kChunkBlocks);
  int64_t run = 1;
  while (ceil_div(n_chunks, run) > kMaxRunPartials) run <<= 1;
  const int grid = (int)ceil_div(n_chunks, run);

  QuantParams p;
  memset(&p, 0, sizeof(p));
  p.W = reinterpret_cast<const uint16_t *>(W);
  p.n = n;
  p.nb = nb;
  p.n_chunks = n_chunks;
  p.run = run;
  p.packed = out->packed;
  p.absmax = out->absmax;
  p.zero = out->zero;
  if (double_quant) {
    p.partials = reinterpret_cast<double *>(workspace);
    p.counter = reinterpret_cast<unsigned *>((char *)workspace + kMaxRunPartials * 8);
    p.absmax_mean = out->absmax_mean;
  }
  p.status = di.status;
  p.scale_f16 = f16 ? 1 : 0;
  p.tab = tab;
  cudaStream_t st = (cudaStream_t)stream;
  rc = run_quantize(w_dtype, qtype, blocksize, double_quant != 0, p, grid, st);
  if (rc != Q4_OK) return rc;
  if (double_quant) rc = run_double_quant(out->absmax, nb, out->absmax_mean, out->absmax_q, out->absmax_scale, st);
  return rc;
}

int q4_quantize_grouped_workspace_size(int32_t count, const int64_t *rows, const int64_t *cols,
                                       int32_t blocksize, int32_t qtype, int32_t double_quant, size_t *bytes) {
  if (!bytes || !rows || !cols || count < 1 || count > kQMaxGroup) return Q4_ERR_ARG;
  size_t total = 256;  // one arrival counter per matrix
  for (int i = 0; i < count; ++i) {
    if (rows[i] < 1 || cols[i] < 1) return Q4_ERR_SHAPE;
    size_t sz[6];
    const int rc = q4_state_sizes(qtype, rows[i] * cols[i], blocksize, double_quant, sz);
    if (rc != Q4_OK) return rc;
    const int64_t nb = ceil_div(rows[i] * cols[i], blocksize);
    // the grouped kernel sums at most 65536 chunk sums per matrix
    if (double_quant && ceil_div(nb, kChunkBlocks) > kQgMaxChunks) return Q4_ERR_SHAPE;
    if (double_quant) total += align256((size_t)ceil_div(nb, kChunkBlocks) * 8);
  }
  *bytes = double_quant ? total : 0;
  return Q4_OK;
}

int q4_quantize_grouped(int32_t count, const void *const *W, int32_t w_dtype, const int64_t *rows,
                        const int64_t *cols, int32_t blocksize, int32_t qtype_in, int32_t double_quant,
                        q4_state *const *out, void *workspace, size_t workspace_bytes, void *stream) {
  if (count < 1 || count > kQMaxGroup || !W || !rows || !cols || !out || !valid_in_dtype(w_dtype)) return Q4_ERR_ARG;
  for (int i = 0; i < count; ++i)
    if (!W[i] || !out[i]) return Q4_ERR_ARG;
  size_t need = 0;
  int rc = q4_quantize_grouped_workspace_size(count, rows, cols, blocksize, qtype_in, double_quant, &need);
  if (rc != Q4_OK) return rc;
  bool f16 = false;
  const int qtype = split_qtype(qtype_in, &f16);
  for (int i = 0; i < count; ++i) {
    q4_state *o = out[i];
    if (!o->packed || !o->absmax || (qtype == Q4_INT4_ASYM && !o->zero)) return Q4_ERR_ARG;
    if (double_quant && (!o->absmax_q || !o->absmax_scale || !o->absmax_mean)) return Q4_ERR_ARG;
    if (!aligned16(W[i]) || !aligned16(o->packed) || ((uintptr_t)o->absmax & (f16 ? 1u : 3u))) return Q4_ERR_ALIGN;
  }
  if (need && (!workspace || workspace_bytes < need)) return Q4_ERR_WORKSPACE;
  const DeviceInfo di = device_info();
  if (di.ok != Q4_OK) return di.ok;
  static Nf4BinTable tab;
  static bool tab_ok = false;
  static std::once_flag once;
  std::call_once(once, [] { tab_ok = build_bin_table(&tab); });
  if (!tab_ok) return Q4_ERR_ARG;

  static thread_local QuantGroupParams p;
  static thread_local DqGroupParams dp;
  memset(&p, 0, sizeof(p));
  memset(&dp, 0, sizeof(dp));
  int64_t chunks = 0, groups = 0;
  size_t ws_off = 256;
  for (int i = 0; i < count; ++i) {
    q4_state *o = out[i];
    const int64_t n = rows[i] * cols[i];
    const int64_t nb = ceil_div(n, blocksize);
    o->qtype = qtype;
    o->src_dtype = w_dtype;
    o->n = n;
    o->rows = rows[i];
    o->cols = cols[i];
    o->blocksize = blocksize;
    o->double_quant = double_quant;
    o->dq_group = Q4_DQ_GROUP;
    o->scale_f16 = f16 ? 1 : 0;
    if (!double_quant) o->absmax_q = nullptr, o->absmax_scale = nullptr, o->absmax_mean = nullptr;
    if (qtype != Q4_INT4_ASYM) o->zero = nullptr;
    QMat &m = p.mat[i];
    m.W = reinterpret_cast<const uint16_t *>(W[i]);
    m.n = n;
    m.nb = nb;
    m.n_chunks = ceil_div(nb, kChunkBlocks);
    m.chunk_begin = chunks;
    m.packed = o->packed;
    m.absmax = o->absmax;
    m.zero = o->zero;
    if (double_quant) {
      m.absmax_mean = o->absmax_mean;
      m.counter = reinterpret_cast<unsigned *>((char *)workspace + 4 * i);
      m.partials = reinterpret_cast<double *>((char *)workspace + ws_off);
      ws_off += align256((size_t)m.n_chunks * 8);
      DqMat &d = dp.mat[i];
      d.absmax = o->absmax;
      d.nb = nb;
      d.mean = o->absmax_mean;
      d.absmax_q = o->absmax_q;
      d.absmax_scale = o->absmax_scale;
      d.group_begin = groups;
      groups += ceil_div(nb, Q4_DQ_GROUP);
    }
    chunks += m.n_chunks;
  }
  p.count = count;
  p.total_chunks = chunks;
  p.status = di.status;
  p.wait_ns = g_wait_limit_ns.load();
  p.stall_copies = g_copy_stall.load();
  p.scale_f16 = f16 ? 1 : 0;
  p.tab = tab;
  dp.count = count;
  dp.total_groups = groups;
  const cudaStream_t st = (cudaStream_t)stream;
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(chunks, (int64_t)di.sms));
  rc = run_quantize_grouped(w_dtype, qtype, blocksize, double_quant != 0, p, grid, st);
  if (rc == Q4_OK && double_quant) rc = run_double_quant_grouped(dp, st);
  return rc;
}

int q4_dequantize(const q4_state *Wq, void *out, int32_t out_dtype, void *stream) {
  return q4_dequantize_grouped(1, &Wq, &out, out_dtype, stream);  // the same kernel, a group of one
}

int q4_dequantize_grouped(int32_t count, const q4_state *const *Wq, void *const *out, int32_t out_dtype,
                          void *stream) {
  if (count < 1 || count > kDqMaxGroup || !Wq || !out || !valid_in_dtype(out_dtype)) return Q4_ERR_ARG;
  for (int i = 0; i < count; ++i) {
    if (!Wq[i] || !out[i]) return Q4_ERR_ARG;
    const int rc = check_state(Wq[i]);
    if (rc != Q4_OK) return rc;
    if (Wq[i]->qtype != Wq[0]->qtype || Wq[i]->blocksize != Wq[0]->blocksize ||
        Wq[i]->double_quant != Wq[0]->double_quant || Wq[i]->scale_f16 != Wq[0]->scale_f16)
      return Q4_ERR_ARG;  // one format per grouped call
    if (!aligned16(out[i])) return Q4_ERR_ALIGN;
  }
  const DeviceInfo di = device_info();
  if (di.ok != Q4_OK) return di.ok;
  static thread_local DequantGroupParams p;
  memset(&p, 0, sizeof(p));
  int64_t spans = 0;
  for (int i = 0; i < count; ++i) {
    const q4_state *s = Wq[i];
    DqGMat &m = p.mat[i];
    m.packed = s->packed;
    m.absmax = s->absmax;
    m.zero = s->zero;
    m.absmax_q = s->absmax_q;
    m.absmax_scale = s->absmax_scale;
    m.absmax_mean = s->absmax_mean;
    m.n = s->n;
    m.out = out[i];
    m.span_begin = spans;
    spans += ceil_div(s->n, kDqSpan);
  }
  p.count = count;
  p.total_spans = spans;
  p.scale_f16 = Wq[0]->scale_f16;
  memcpy(p.levels, kNF4Levels, sizeof(kNF4Levels));
  return run_dequantize(Wq[0]->qtype, out_dtype, Wq[0]->blocksize, Wq[0]->double_quant != 0, p, di.sms,
                        (cudaStream_t)stream);
}

int q4_gemv_workspace_size(int32_t count, const q4_state *const *Wq, int64_t M, size_t *bytes) {
  if (!bytes || !Wq || count < 1 || count > kGsMaxGroup) return Q4_ERR_ARG;
  if (M < 1 || M > 32) return Q4_ERR_SHAPE;
  for (int i = 0; i < count; ++i) {
    if (!Wq[i]) return Q4_ERR_ARG;
    if (!valid_bs(Wq[i]->blocksize) || Wq[i]->cols % Wq[i]->blocksize || Wq[i]->rows < 1) return Q4_ERR_SHAPE;
  }
  size_t total = kGemvWsHead;
  int64_t units = 0;
  for (int i = 0; i < count; ++i) {
    total += gemv_counters_for(Wq[i]);
    int64_t t, q;
    gemv_ws_for(Wq[i], &t, &q);
    units += t * q;
  }
  total += gemv_small_slots(units, M);
  *bytes = total;
  return Q4_OK;
}

int q4_gemv_grouped(int32_t count, const void *const *A, const q4_state *const *Wq,
                    void *const *Y, int64_t M, int32_t a_dtype, int32_t y_dtype, void *workspace,
                    size_t workspace_bytes, void *stream) {
  if (count < 1 || count > kGsMaxGroup || !A || !Wq || !Y) return Q4_ERR_ARG;
  if (!valid_in_dtype(a_dtype) || !valid_out_dtype(y_dtype)) return Q4_ERR_ARG;
  if (M < 1 || M > 32) return Q4_ERR_SHAPE;
  // every entry is checked before any of them is dereferenced
  for (int i = 0; i < count; ++i)
    if (!Wq[i] || !A[i] || !Y[i]) return Q4_ERR_ARG;
  for (int i = 0; i < count; ++i)  // one format per grouped call
    if (Wq[i]->qtype != Wq[0]->qtype || Wq[i]->scale_f16 != Wq[0]->scale_f16) return Q4_ERR_ARG;
  return gemv_small_grouped(count, A, Wq, Y, M, a_dtype, y_dtype, workspace, workspace_bytes, stream);
}

int q4_gemv(const void *A, int32_t a_dtype, int64_t M, const q4_state *Wq, void *Y,
            int32_t y_dtype, void *workspace, size_t workspace_bytes, void *stream) {
  const void *a[1] = {A};
  const q4_state *w[1] = {Wq};
  void *y[1] = {Y};
  return q4_gemv_grouped(1, a, w, y, M, a_dtype, y_dtype, workspace, workspace_bytes, stream);
}

// ---- GEMM planning -----------------------------------------------------------
// A launch of at most kGemmListTiles work items deals them to the CTAs
// longest first (k-blocks), each onto the CTA with the least work so far;
// every CTA then runs its items in ascending order.  With a workspace the
// planner may also cut tiles into two halves of their k range (split-K):
// it deals three candidates -- whole tiles, the longest tiles cut, every
// tile of at least two k-blocks cut -- and keeps the one whose busiest CTA
// has the least work (ties: fewer cuts), a cut only when it takes at least
// a tenth off the whole tiles' busiest CTA (the cut instance also carries
// the split-K code, which costs its registers).  A half counts its k-blocks plus
// kGemmSplitCost for its fix-up (an fp32 partial written, counted and, by
// the second half, read back; measured at M = 512 on one B200 as about 16
// k-blocks' time).  Larger launches deal whole tiles round robin, which is
// then within a few percent of even.
//
// Tiles are kGemmBM tokens high (one accumulator; each dequantized weight
// stage feeds two MMAs) or kGemmHalfM (two accumulators that alternate, so
// an epilogue overlaps the next tile's MMAs; twice the dequant work per
// flop).  The planner weighs a k-block of a token half at kGemmCostHalf in
// the first and kGemmCostWhole in the second (measured on the 7B layer at
// M = 512 and 2048: 820 -> 955 and 878 -> 1102 TFLOP/s) and takes the
// height whose busiest CTA finishes first: the tall tiles unless they
// leave most SMs idle (few tiles) or M fits one half anyway.
constexpr int kGemmSplitCost = 16;
constexpr int kGemmCostHalf = 17, kGemmCostWhole = 20;
struct GemmPlan {
  int64_t grid = 0;    // CTAs
  int64_t slots = 0;   // split tiles
  int64_t max_load = 0;
  int listed = 0;
  int cut = 0;         // 0 none, 1 the longest tiles, 2 every tile
};
size_t gemm_split_bytes(int64_t slots) {
  return slots ? kGemmSplitCntBytes + (size_t)slots * kGemmSplitSlotBytes : 0;
}
// The items of cut mode `cut` as (work, encoded item); slots counts the cut
// tiles.  Work is k-blocks (plus the fix-up of a cut) times the tile's
// token halves times the cost of a half at this tile height.
static void gemm_items(const GemmParams &p, int count, int cut, std::vector<std::pair<int, uint32_t>> &items,
                       int64_t &slots) {
  int max_nk = 0;
  for (int i = 0; i < count; ++i) max_nk = std::max(max_nk, p.mat[i].K / kGemmBK);
  items.clear();
  slots = 0;
  for (int i = 0; i < count; ++i) {
    const GemmMat &m = p.mat[i];
    const int nk = m.K / kGemmBK;
    const bool split = nk >= 2 && (cut == 2 || (cut == 1 && nk == max_nk));
    const int64_t n = (int64_t)m.tiles_m * m.tiles_n;
    for (int64_t t = 0; t < n; ++t) {
      const uint32_t tile = (uint32_t)(m.tile_begin + t);
      const int64_t tm = t % m.tiles_m;  // m-tiles fastest, as the kernel decodes them
      const int unit = p.tile_m == kGemmBM ? kGemmCostHalf * (tm * kGemmBM + kGemmHalfM < m.M ? 2 : 1)
                                           : kGemmCostWhole;
      if (split) {
        items.emplace_back((nk / 2 + kGemmSplitCost) * unit, tile | (1u << 16) | ((uint32_t)slots << 18));
        items.emplace_back((nk - nk / 2 + kGemmSplitCost) * unit, tile | (2u << 16) | ((uint32_t)slots << 18));
        ++slots;
      } else {
        items.emplace_back(nk * unit, tile);
      }
    }
  }
}
// Longest first onto the least loaded of `grid` CTAs; the busiest CTA's
// k-blocks.  With `out`, its lists are written there.
static int64_t gemm_lpt(std::vector<std::pair<int, uint32_t>> items, int64_t grid, GemmParams *out) {
  std::stable_sort(items.begin(), items.end(),
                   [](const std::pair<int, uint32_t> &a, const std::pair<int, uint32_t> &b) { return a.first > b.first; });
  std::vector<std::vector<uint32_t>> per((size_t)grid);
  std::vector<int64_t> load((size_t)grid, 0);
  // the least loaded CTA (the lowest index among equals) from a min-heap
  std::priority_queue<std::pair<int64_t, int64_t>, std::vector<std::pair<int64_t, int64_t>>,
                      std::greater<std::pair<int64_t, int64_t>>> heap;
  for (int64_t c = 0; c < grid; ++c) heap.emplace(0, c);
  for (const auto &o : items) {
    const int64_t best = heap.top().second;
    heap.pop();
    load[(size_t)best] += o.first;
    per[(size_t)best].push_back(o.second);
    heap.emplace(load[(size_t)best], best);
  }
  if (out) {
    int off = 0;
    for (int64_t c = 0; c < grid; ++c) {
      out->cta_off[c] = (uint16_t)off;
      std::sort(per[(size_t)c].begin(), per[(size_t)c].end(),
                [](uint32_t a, uint32_t b) { return (a & 0xFFFFu) != (b & 0xFFFFu) ? (a & 0xFFFFu) < (b & 0xFFFFu) : a < b; });
      for (uint32_t v : per[(size_t)c]) out->tile_list[off++] = v;
    }
    out->cta_off[grid] = (uint16_t)off;
  }
  return *std::max_element(load.begin(), load.end());
}
// The plan of a launch over p's matrices (tiles set); `max_split_bytes`
// bounds the workspace a cut may use (0: no cuts).  With `out`, the chosen
// lists are written there.  max_load is 0 for round robin (not estimated).
static GemmPlan gemm_plan(const GemmParams &p, int count, int sms, size_t max_split_bytes, GemmParams *out) {
  GemmPlan best;
  const int64_t tiles = p.total_tiles;
  best.grid = std::min<int64_t>(tiles, sms);
  if (tiles > kGemmListTiles) return best;  // round robin over whole tiles
  std::vector<std::pair<int, uint32_t>> items;
  bool have = false;
  int64_t whole_load = 0;  // the busiest CTA of whole tiles (cut 0 comes first)
  for (int cut = 0; cut <= 2; ++cut) {
    int64_t slots = 0;
    gemm_items(p, count, cut, items, slots);
    if (cut > 0 && (slots == 0 || gemm_split_bytes(slots) > max_split_bytes)) continue;
    if ((int64_t)items.size() > kGemmListTiles || slots > kGemmListTiles / 2) continue;
    const int64_t grid = std::min<int64_t>({(int64_t)items.size(), (int64_t)sms, (int64_t)kGemmListCtas});
    const int64_t mx = gemm_lpt(items, grid, nullptr);
    if (cut > 0 && 10 * mx > 9 * whole_load) continue;
    if (!have || mx < best.max_load || (mx == best.max_load && slots < best.slots)) {
      best.grid = grid;
      best.slots = slots;
      best.max_load = mx;
      best.cut = cut;
      // a list is needed for cut tiles, or to balance more tiles than CTAs
      best.listed = (slots > 0 || (int64_t)items.size() > grid) ? 1 : 0;
      have = true;
    }
    if (cut == 0) whole_load = mx;
  }
  if (out && best.listed) {
    int64_t slots = 0;
    gemm_items(p, count, best.cut, items, slots);
    gemm_lpt(items, best.grid, out);
  }
  return best;
}

// Token tiles of height tile_m for every matrix of p (M, N set).
static void gemm_tiles(GemmParams &p, int tile_m) {
  int64_t tiles = 0;
  p.tile_m = tile_m;
  for (int i = 0; i < p.count; ++i) {
    GemmMat &m = p.mat[i];
    m.tiles_m = (int32_t)ceil_div(m.M, tile_m);
    m.tile_begin = tiles;
    tiles += (int64_t)m.tiles_m * m.tiles_n;
  }
  p.total_tiles = tiles;
}

// Shapes and formats of a GEMM call (host only); fills the per-matrix tile
// counts of `p` (tall tiles).
static int gemm_check(int32_t count, const q4_state *const *Wq, int64_t M, GemmParams &p) {
  for (int i = 0; i < count; ++i) {
    const q4_state *s = Wq[i];
    if (!s) return Q4_ERR_ARG;
    const int rc = check_state(s);
    if (rc != Q4_OK) return rc;
    // one format per grouped call
    if (s->qtype != Wq[0]->qtype || s->blocksize != Wq[0]->blocksize ||
        s->double_quant != Wq[0]->double_quant || s->scale_f16 != Wq[0]->scale_f16)
      return Q4_ERR_ARG;
    // whole 64-k blocks of whole quantization blocks
    if (s->cols % 64 || s->cols % s->blocksize || s->rows % 16 || s->rows > INT32_MAX || s->cols > INT32_MAX)
      return Q4_ERR_SHAPE;
    GemmMat &m = p.mat[i];
    m.M = (int32_t)M;
    m.N = (int32_t)s->rows;
    m.K = (int32_t)s->cols;
    m.tiles_n = (int32_t)ceil_div(s->rows, kGemmBN);
  }
  p.count = count;
  gemm_tiles(p, kGemmBM);
  return Q4_OK;
}

// The tile height of a launch (kGemmBM or kGemmHalfM) and its plan; p's
// tiles are set for that height and, with `lists`, its item lists written.
static GemmPlan gemm_choose_uncached(GemmParams &p, int count, int sms, size_t max_split_bytes, bool lists) {
  int tile_m = kGemmBM;
  if (p.mat[0].M <= kGemmHalfM) {
    tile_m = kGemmHalfM;  // one half per tile either way: two accumulators overlap the epilogue
  } else {
    gemm_tiles(p, kGemmBM);
    const GemmPlan tall = gemm_plan(p, count, sms, max_split_bytes, nullptr);
    if (tall.max_load > 0) {  // listed: compare with the half-height tiles
      gemm_tiles(p, kGemmHalfM);
      const GemmPlan low = gemm_plan(p, count, sms, max_split_bytes, nullptr);
      if (low.max_load > 0 && low.max_load < tall.max_load) tile_m = kGemmHalfM;
    }
  }
  gemm_tiles(p, tile_m);
  return gemm_plan(p, count, sms, max_split_bytes, lists ? &p : nullptr);
}

// Planning a listed launch takes up to nine list-scheduling passes (two
// tile heights, three cut modes, the final lists): hundreds of
// microseconds of host time for a decoder layer.  A plan depends only on
// the shapes, M, the SM count and the workspace bound, so the last few
// plans of each host thread are kept and reused.
struct GemmPlanKey {
  int32_t count, sms;
  int64_t M;
  size_t max_split_bytes;
  int32_t N[16], K[16];
  bool operator==(const GemmPlanKey &o) const {
    if (count != o.count || sms != o.sms || M != o.M || max_split_bytes != o.max_split_bytes) return false;
    for (int i = 0; i < count; ++i)
      if (N[i] != o.N[i] || K[i] != o.K[i]) return false;
    return true;
  }
};
struct GemmPlanEntry {
  bool used = false;
  GemmPlanKey key;
  GemmPlan plan;
  int32_t tile_m = 0;
  uint16_t cta_off[kGemmListCtas + 1];
  uint32_t tile_list[kGemmListTiles];
};
constexpr int kGemmPlanCache = 8;
static GemmPlan gemm_choose(GemmParams &p, int count, int sms, size_t max_split_bytes, bool lists) {
  static thread_local GemmPlanEntry cache[kGemmPlanCache];
  static thread_local int next = 0;
  GemmPlanKey key;
  memset(&key, 0, sizeof(key));
  key.count = count;
  key.sms = sms;
  key.M = p.mat[0].M;
  key.max_split_bytes = max_split_bytes;
  for (int i = 0; i < count; ++i) key.N[i] = p.mat[i].N, key.K[i] = p.mat[i].K;
  for (GemmPlanEntry &e : cache) {
    if (!e.used || !(e.key == key)) continue;
    gemm_tiles(p, e.tile_m);
    if (lists && e.plan.listed) {
      memcpy(p.cta_off, e.cta_off, sizeof(uint16_t) * (size_t)(e.plan.grid + 1));
      memcpy(p.tile_list, e.tile_list, sizeof(uint32_t) * e.cta_off[e.plan.grid]);
    }
    return e.plan;
  }
  const GemmPlan plan = gemm_choose_uncached(p, count, sms, max_split_bytes, true);
  GemmPlanEntry &e = cache[next];
  next = (next + 1) % kGemmPlanCache;
  e.used = true;
  e.key = key;
  e.plan = plan;
  e.tile_m = p.tile_m;
  if (plan.listed) {
    memcpy(e.cta_off, p.cta_off, sizeof(uint16_t) * (size_t)(plan.grid + 1));
    memcpy(e.tile_list, p.tile_list, sizeof(uint32_t) * p.cta_off[plan.grid]);
  }
  return plan;
}

int q4_gemm_workspace_size(int32_t count, const q4_state *const *Wq, int64_t M, size_t *bytes) {
  if (!bytes || !Wq || count < 1 || count > kGsMaxGroup) return Q4_ERR_ARG;
  if (M < 1 || M > INT32_MAX) return Q4_ERR_SHAPE;
  static thread_local GemmParams p;
  memset(&p, 0, sizeof(p));
  const int rc = gemm_check(count, Wq, M, p);
  if (rc != Q4_OK) return rc;
  const DeviceInfo di = device_info();
  if (di.ok != Q4_OK) return di.ok;
  const GemmPlan plan = gemm_choose(p, count, di.sms, (size_t)-1, false);
  *bytes = gemm_split_bytes(plan.slots);
  return Q4_OK;
}

int q4_gemm_plan_info(int32_t count, const q4_state *const *Wq, int64_t M, int32_t sms, size_t workspace_bytes,
                      int32_t *tile_m, int32_t *grid, int64_t *cut_tiles) {
  if (!tile_m || !grid || !cut_tiles || !Wq || count < 1 || count > kGsMaxGroup) return Q4_ERR_ARG;
  if (sms < 1 || sms > 1024) return Q4_ERR_ARG;
  if (M < 1 || M > INT32_MAX) return Q4_ERR_SHAPE;
  static thread_local GemmParams p;
  memset(&p, 0, sizeof(p));
  const int rc = gemm_check(count, Wq, M, p);
  if (rc != Q4_OK) return rc;
  const GemmPlan plan = gemm_choose(p, count, sms, workspace_bytes, false);
  *tile_m = p.tile_m;
  *grid = (int32_t)plan.grid;
  *cut_tiles = plan.slots;
  return Q4_OK;
}

int q4_gemm_grouped(int32_t count, const void *const *A, const q4_state *const *Wq,
                    void *const *Y, int64_t M, int32_t a_dtype, int32_t y_dtype, void *workspace,
                    size_t workspace_bytes, void *stream) {
  if (count < 1 || count > kGsMaxGroup || !A || !Wq || !Y) return Q4_ERR_ARG;
  if (!valid_in_dtype(a_dtype) || !valid_out_dtype(y_dtype)) return Q4_ERR_ARG;
  if (y_dtype != Q4_F32 && y_dtype != a_dtype) return Q4_ERR_ARG;
  if (M < 1 || M > INT32_MAX) return Q4_ERR_SHAPE;
  for (int i = 0; i < count; ++i)
    if (!Wq[i] || !A[i] || !Y[i]) return Q4_ERR_ARG;
  static thread_local GemmParams p;  // host staging of the kernel parameters (~14 KB)
  memset(&p, 0, sizeof(p));
  // every matrix's format and shape first (host only), then the device
  int rc = gemm_check(count, Wq, M, p);
  if (rc != Q4_OK) return rc;
  for (int i = 0; i < count; ++i)
    if (!aligned16(A[i]) || !aligned16(Y[i])) return Q4_ERR_ALIGN;
  if (workspace && !aligned16(workspace)) return Q4_ERR_ALIGN;
  const DeviceInfo di = device_info();
  if (di.ok != Q4_OK) return di.ok;
  const int dq = Wq[0]->double_quant;
  for (int i = 0; i < count && rc == Q4_OK; ++i) {
    const q4_state *s = Wq[i];
    GemmMat &m = p.mat[i];
    const CUtensorMapDataType adt = a_dtype == Q4_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    if (!make_map(&m.tmA, adt, A[i], M, s->cols, 2, kGemmBK, kGemmHalfM, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&m.tmW, CU_TENSOR_MAP_DATA_TYPE_UINT8, s->packed, s->rows, s->cols / 2, 1, kGemmBK / 2,
                  kGemmBN, CU_TENSOR_MAP_SWIZZLE_NONE)) {
      rc = Q4_ERR_CUDA;
      break;
    }
    m.absmax_q = s->absmax_q;
    m.absmax_scale = s->absmax_scale;
    m.absmax_mean = s->absmax_mean;
    m.absmax = s->absmax;
    m.zero = s->zero;
    m.Y = Y[i];
  }
  if (rc == Q4_OK) {
    p.y_dtype = y_dtype;
    p.dq = dq;
    p.status = di.status;
    const int qt = Wq[0]->qtype;
    int mode = dq ? kGemmDq : kGemmPlain;
    if (qt == Q4_NF4) {
      memcpy(p.levels, kNF4Levels, sizeof(kNF4Levels));
    } else if (qt == Q4_INT4_SYM) {
      for (int j = 0; j < 16; ++j) p.levels[j] = (float)((j ^ 8) - 8);  // two's-complement nibble q: w^ = q s
    } else {
      for (int j = 0; j < 16; ++j) p.levels[j] = (float)j;  // w^ = (q - z) s
      mode = kGemmAsym;
    }
    p.log2_bs = __builtin_ctz((unsigned)Wq[0]->blocksize);
    p.scale_f16 = Wq[0]->scale_f16;
    const GemmPlan plan = gemm_choose(p, count, di.sms, workspace ? workspace_bytes : 0, true);
    p.listed = plan.listed;
    p.grid = (int32_t)plan.grid;
    if (plan.slots) {
      p.split_cnt = reinterpret_cast<unsigned *>(workspace);
      p.partials = reinterpret_cast<float *>((char *)workspace + kGemmSplitCntBytes);
    }
    p.wait_ns = g_wait_limit_ns.load(std::memory_order_relaxed);
    p.stall_copies = g_copy_stall.load(std::memory_order_relaxed);
    rc = run_gemm(a_dtype, mode, plan.slots > 0, p, (cudaStream_t)stream);
  }
  return rc;
}

int q4_gemm(const void *A, int32_t a_dtype, int64_t M, const q4_state *Wq, void *Y,
            int32_t y_dtype, void *workspace, size_t workspace_bytes, void *stream) {
  const void *a[1] = {A};
  const q4_state *w[1] = {Wq};
  void *y[1] = {Y};
  return q4_gemm_grouped(1, a, w, y, M, a_dtype, y_dtype, workspace, workspace_bytes, stream);
}

int q4_set_wait_limit_ns(uint64_t ns) {
  g_wait_limit_ns.store(ns ? ns : kWaitLimitNs, std::memory_order_relaxed);
  return Q4_OK;
}

int q4_set_copy_stall(int32_t on) {
  g_copy_stall.store(on ? 1 : 0, std::memory_order_relaxed);
  return Q4_OK;
}

int q4_device_status(int32_t *status) {
  if (!status) return Q4_ERR_ARG;
  const DeviceInfo di = device_info();
  if (di.ok != Q4_OK) return di.ok;
  int v = 0;
  if (cudaMemcpy(&v, di.status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return Q4_ERR_CUDA;
  *status = v;
  return Q4_OK;
}

int q4_clear_device_status(void) {
  const DeviceInfo di = device_info();
  if (di.ok != Q4_OK) return di.ok;
  if (cudaMemset(di.status, 0, sizeof(int)) != cudaSuccess) return Q4_ERR_CUDA;
  return Q4_OK;
}

}  // extern "C"
