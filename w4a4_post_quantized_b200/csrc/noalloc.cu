// noalloc.cu -- w4a4_linear_fused_noalloc: the fused quantized linear for
// callers that cannot allocate device memory themselves.
//
// w4a4_linear_fused needs a caller-provided workspace (the packed activation
// codes and per-token steps passed from the quantize kernel to the GEMM).  Some
// callers cannot get one: code running where cudaMalloc/cudaFree are off limits
// (cudaFree synchronizes the whole device, and a serving loop with a fixed
// memory budget or a plugin host's enqueue callback may forbid any allocation
// after start-up), or a plain C caller that was only handed its input and
// output buffers by another runtime.  This entry point uses a scratch array
// built into the library instead.
//
// The scratch is a file-scope device array of W4A4_NOALLOC_SCRATCH_BYTES; every
// GPU that loads the library keeps it until the process exits.  In host code
// the array's name is only a host-side stand-in for the symbol, so its device
// address is looked up with cudaGetSymbolAddress, once per device (with that
// device current), the first time the entry point runs on it.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "w4a4.h"

namespace {

static_assert(W4A4_NOALLOC_SCRATCH_BYTES % 256 == 0, "scratch size");

// Shared by every call on a device; holds the last call's codes and steps.
static __device__ __align__(256) unsigned char g_noalloc_scratch[W4A4_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void *g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mutex;

// Device address of the scratch array on the current device (looked up once
// per device).  Returns nullptr and sets *err when the lookup fails.
void *scratch_on_current_device(cudaError_t *err) {
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= kMaxDevices) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_addr[dev]) {
    void *p = nullptr;
    *err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (*err != cudaSuccess) return nullptr;
    g_scratch_addr[dev] = p;
  }
  return g_scratch_addr[dev];
}

}  // namespace

extern "C" w4a4_status w4a4_linear_fused_noalloc(const uint16_t *X, int64_t M,
                                                 const w4a4_weights_t *w, uint16_t *Y,
                                                 uint32_t flags, void *stream) {
  if (!w) return W4A4_ERR_ARG;
  if (M < 0) return W4A4_ERR_SHAPE;
  // the workspace this call needs must fit the built-in scratch; unsupported K
  // is reported by w4a4_linear_fused below
  const size_t need = w4a4_workspace_bytes_min(M, w->K, flags);
  if (need > W4A4_NOALLOC_SCRATCH_BYTES) return W4A4_ERR_SHAPE;
  cudaError_t err = cudaSuccess;
  void *scratch = scratch_on_current_device(&err);
  if (!scratch) return W4A4_ERR_CUDA;
  // Nothing in the scratch has to start at zero: the quantize kernel writes
  // every code byte and step the GEMM then reads.
  return w4a4_linear_fused(X, M, w, Y, scratch, W4A4_NOALLOC_SCRATCH_BYTES, flags, stream);
}
