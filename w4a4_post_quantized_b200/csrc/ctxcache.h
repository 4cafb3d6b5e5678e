// ctxcache.h -- values that belong to one CUDA context, computed once per
// context: a kernel's shared-memory attribute and occupancy, the device
// address of a module variable (the status word, the allocation-free scratch
// array).  A context that replaces an earlier one on the same device (after
// cudaDeviceReset, or a caller's own non-primary context) gets a new
// identifier and therefore its own entry, so no value of a destroyed context is
// ever reused.  Lookups and insertions are serialised by a mutex, so host
// threads may make their first calls concurrently.
#pragma once

#include <cuda_runtime.h>

#include <mutex>

namespace w4a4 {

// Unique identifier of the calling thread's current CUDA context (the
// driver's context ID, never reused within a process); 0 when no context is
// current yet or the driver cannot say.
unsigned long long current_context_id();

template <typename T, int kSlots = 64>
class ContextCache {
 public:
  // *out = the value for the current context.  On the first call in a context
  // make(&value) computes it (returning cudaSuccess, or an error that is passed
  // on and leaves nothing cached).
  template <typename Make>
  cudaError_t get(T *out, Make make) {
    std::lock_guard<std::mutex> lock(mu_);
    unsigned long long id = current_context_id();
    if (id != 0)
      for (int i = 0; i < used_; ++i)
        if (ids_[i] == id) {
          *out = vals_[i];
          return cudaSuccess;
        }
    T v{};
    const cudaError_t e = make(&v);
    if (e != cudaSuccess) return e;
    id = current_context_id();  // make() may have created the primary context
    if (id != 0) {
      const int slot = used_ < kSlots ? used_++ : static_cast<int>(next_++ % kSlots);
      ids_[slot] = id;
      vals_[slot] = v;
    }
    *out = v;
    return cudaSuccess;
  }

 private:
  std::mutex mu_;
  unsigned long long ids_[kSlots] = {};
  T vals_[kSlots] = {};
  int used_ = 0;
  unsigned next_ = 0;
};

}  // namespace w4a4
