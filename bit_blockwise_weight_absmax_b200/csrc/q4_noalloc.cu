// q4_noalloc.cu -- q4_quantize_noalloc: quantization for callers that cannot
// hand the library a device workspace.
//
// Some callers are not allowed to allocate device memory at the point where
// they quantize: a plugin inside a host application whose allocator owns all
// device memory, code that must not trigger the implicit device-wide
// synchronization of cudaMalloc/cudaFree in a latency-critical path, or an
// embedded runtime that reserves all memory up front.  q4_quantize needs a
// small zero-filled workspace when double quantization is on (the per-CTA
// partial sums of the absmax mean and an arrival counter).  This entry point
// supplies that workspace itself from a fixed array in the library's own
// device memory, so the caller passes only the input weights and the output
// state buffers.
//
// The array is file-scope static device memory: every GPU that loads the
// library holds Q4_NOALLOC_SCRATCH_BYTES of it until the process exits, and
// all calls on a device share it.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/q4.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[Q4_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

// Device address of g_noalloc_scratch for the current device.  In host code
// the symbol name is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and cached.
int scratch_address(void **out) {
  static void *addr[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return Q4_ERR_NO_DEVICE;
  }
  if (dev < 0 || dev >= kMaxDevices) return Q4_ERR_ARG;
  std::lock_guard<std::mutex> lk(mu);
  if (!addr[dev]) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress((void **)&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      cudaGetLastError();
      return Q4_ERR_CUDA;
    }
    addr[dev] = p;
  }
  *out = addr[dev];
  return Q4_OK;
}

}  // namespace

extern "C" int q4_quantize_noalloc(const void *W, int32_t w_dtype, int64_t rows, int64_t cols,
                                   int32_t blocksize, int32_t qtype, int32_t double_quant,
                                   q4_state *out, void *stream) {
  if (rows < 1 || cols < 1) return Q4_ERR_SHAPE;
  size_t need = 0;
  int rc = q4_quantize_workspace_size(qtype, rows * cols, blocksize, double_quant, &need);
  if (rc != Q4_OK) return rc;
  if (need > (size_t)Q4_NOALLOC_SCRATCH_BYTES) return Q4_ERR_WORKSPACE;
  void *ws = nullptr;
  if (need) {
    rc = q4_check_device();
    if (rc != Q4_OK) return rc;
    rc = scratch_address(&ws);
    if (rc != Q4_OK) return rc;
    // The array keeps whatever the previous call left; the workspace contract
    // of q4_quantize wants it zero-filled, so clear it on the caller's stream
    // (a memset, not an allocation).
    if (cudaMemsetAsync(ws, 0, need, (cudaStream_t)stream) != cudaSuccess) {
      cudaGetLastError();
      return Q4_ERR_CUDA;
    }
  }
  return q4_quantize(W, w_dtype, rows, cols, blocksize, qtype, double_quant, out, ws, need, stream);
}
