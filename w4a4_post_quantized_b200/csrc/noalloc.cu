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
// address is looked up with cudaGetSymbolAddress, once per device and context
// (with that device current), the first time the entry point runs there.
#include <cuda_runtime.h>

#include <cstdint>

#include "ctxcache.h"
#include "w4a4.h"

namespace {

static_assert(W4A4_NOALLOC_SCRATCH_BYTES % 256 == 0, "scratch size");

// Shared by every call on a device; holds the last call's codes and steps.
static __device__ __align__(256) unsigned char g_noalloc_scratch[W4A4_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch array in the current context, looked up once
// per context (a context that replaces an earlier one, e.g. after
// cudaDeviceReset, looks it up again).  Returns nullptr and sets *err when the
// lookup fails.
void *scratch_on_current_device(cudaError_t *err) {
  static w4a4::ContextCache<void *> cache;
  void *p = nullptr;
  *err = cache.get(&p, [](void **v) { return cudaGetSymbolAddress(v, g_noalloc_scratch); });
  if (*err == cudaSuccess && p == nullptr) *err = cudaErrorInvalidSymbol;
  return *err == cudaSuccess ? p : nullptr;
}

// The flags w4a4_linear_fused accepts (it picks the code layout itself, so
// W4A4_FLAG_UNPACKED is not among them).
constexpr uint32_t kFusedFlags =
    W4A4_FLAG_GELU | W4A4_FLAG_PLAIN | W4A4_FLAG_INT8 | W4A4_FLAG_GELU_OUT;

}  // namespace

extern "C" w4a4_status w4a4_linear_fused_noalloc(const uint16_t *X, int64_t M,
                                                 const w4a4_weights_t *w, uint16_t *Y,
                                                 uint32_t flags, void *stream) {
  if (!w) return W4A4_ERR_ARG;
  // flags first, so that a call w4a4_linear_fused would refuse for its flags
  // gets the same status here whatever M is
  if (flags & ~kFusedFlags) return W4A4_ERR_UNSUPPORTED;
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
