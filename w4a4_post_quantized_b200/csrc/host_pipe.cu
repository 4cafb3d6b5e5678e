// host_pipe.cu -- w4a4_linear_fused_host: the fused linear on host buffers,
// pipelined over row chunks so that the two copy directions and the kernels
// overlap.
//
// Chunk c uses workspace slot c % W4A4_PIPE_DEPTH:
//   copy-in stream:   [wait: slot's previous compute done]  X chunk host->device  -> ev_in
//   compute stream:   [wait: ev_in, slot's previous copy-out done]  quantize + GEMM -> ev_done
//   copy-out stream:  [wait: ev_done]  Y chunk device->host  -> ev_out
// cudaStreamWaitEvent waits for the event's most recent record, so reusing
// the events chunk after chunk orders each slot's uses.
#include <cuda_runtime.h>

#include <cstdint>

#include "w4a4.h"

struct w4a4_host_pipe {
  int device;
  cudaStream_t copy_in, copy_out;
  cudaEvent_t ev_in[W4A4_PIPE_DEPTH], ev_done[W4A4_PIPE_DEPTH], ev_out[W4A4_PIPE_DEPTH];
};

namespace {

size_t round256(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }

struct Slot {
  uint16_t *x;
  uint16_t *y;
  void *ws;
  size_t ws_bytes;
};

Slot slot_of(void *workspace, int64_t chunk_rows, int32_t K, int32_t N, int i) {
  const size_t xb = round256(static_cast<size_t>(chunk_rows) * K * 2);
  const size_t yb = round256(static_cast<size_t>(chunk_rows) * N * 2);
  const size_t wb = round256(w4a4_workspace_bytes(chunk_rows, K));
  uint8_t *base = static_cast<uint8_t *>(workspace) + static_cast<size_t>(i) * (xb + yb + wb);
  return Slot{reinterpret_cast<uint16_t *>(base), reinterpret_cast<uint16_t *>(base + xb),
              base + xb + yb, wb};
}

}  // namespace

extern "C" w4a4_status w4a4_host_pipe_create(w4a4_host_pipe_t **out) {
  if (!out) return W4A4_ERR_ARG;
  *out = nullptr;
  w4a4_host_pipe_t *p = new w4a4_host_pipe_t{};
  bool ok = cudaGetDevice(&p->device) == cudaSuccess &&
            cudaStreamCreateWithFlags(&p->copy_in, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&p->copy_out, cudaStreamNonBlocking) == cudaSuccess;
  for (int i = 0; ok && i < W4A4_PIPE_DEPTH; ++i)
    ok = cudaEventCreateWithFlags(&p->ev_in[i], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&p->ev_done[i], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&p->ev_out[i], cudaEventDisableTiming) == cudaSuccess;
  if (!ok) {
    w4a4_host_pipe_destroy(p);
    return W4A4_ERR_CUDA;
  }
  *out = p;
  return W4A4_OK;
}

extern "C" w4a4_status w4a4_host_pipe_destroy(w4a4_host_pipe_t *p) {
  if (!p) return W4A4_OK;
  bool ok = true;
  if (p->copy_in) ok &= cudaStreamSynchronize(p->copy_in) == cudaSuccess;
  if (p->copy_out) ok &= cudaStreamSynchronize(p->copy_out) == cudaSuccess;
  for (int i = 0; i < W4A4_PIPE_DEPTH; ++i) {
    if (p->ev_in[i]) cudaEventDestroy(p->ev_in[i]);
    if (p->ev_done[i]) cudaEventDestroy(p->ev_done[i]);
    if (p->ev_out[i]) cudaEventDestroy(p->ev_out[i]);
  }
  if (p->copy_in) cudaStreamDestroy(p->copy_in);
  if (p->copy_out) cudaStreamDestroy(p->copy_out);
  delete p;
  return ok ? W4A4_OK : W4A4_ERR_CUDA;
}

extern "C" size_t w4a4_host_workspace_bytes(int64_t chunk_rows, int32_t K, int32_t N) {
  if (chunk_rows <= 0 || K <= 0 || N <= 0) return 0;
  const size_t xb = round256(static_cast<size_t>(chunk_rows) * K * 2);
  const size_t yb = round256(static_cast<size_t>(chunk_rows) * N * 2);
  const size_t wb = round256(w4a4_workspace_bytes(chunk_rows, K));
  return W4A4_PIPE_DEPTH * (xb + yb + wb);
}

extern "C" w4a4_status w4a4_linear_fused_host(const uint16_t *X_host, int64_t M,
                                              const w4a4_weights_t *w, uint16_t *Y_host,
                                              int64_t chunk_rows, void *workspace,
                                              size_t workspace_bytes, w4a4_host_pipe_t *pipe,
                                              uint32_t flags, void *stream) {
  if (!w || !pipe) return W4A4_ERR_ARG;
  if (M < 0 || chunk_rows <= 0) return W4A4_ERR_SHAPE;
  if (M == 0) return W4A4_OK;
  if (!X_host || !Y_host || !workspace) return W4A4_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 15) != 0) return W4A4_ERR_ALIGN;
  if (workspace_bytes < w4a4_host_workspace_bytes(chunk_rows, w->K, w->N)) return W4A4_ERR_SHAPE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != pipe->device) return W4A4_ERR_ARG;
  // X or Y may stay in device memory (the first or last layer of a stack run
  // on the device): that side's copies are skipped and the kernels read X /
  // write Y in place
  const bool x_dev = (flags & W4A4_FLAG_X_DEVICE) != 0, y_dev = (flags & W4A4_FLAG_Y_DEVICE) != 0;
  flags &= ~(W4A4_FLAG_X_DEVICE | W4A4_FLAG_Y_DEVICE);
  if ((x_dev && (reinterpret_cast<uintptr_t>(X_host) & 15) != 0) ||
      (y_dev && (reinterpret_cast<uintptr_t>(Y_host) & 15) != 0))
    return W4A4_ERR_ALIGN;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const int64_t nchunks = (M + chunk_rows - 1) / chunk_rows;
  // the copy-in stream starts after everything already enqueued on `stream`
  // (the caller may have just written the weights or the host buffers'
  // producers may be ordered on it): record once, wait once
  if (cudaEventRecord(pipe->ev_done[0], cs) != cudaSuccess ||
      cudaStreamWaitEvent(pipe->copy_in, pipe->ev_done[0], 0) != cudaSuccess ||
      cudaStreamWaitEvent(pipe->copy_out, pipe->ev_done[0], 0) != cudaSuccess)
    return W4A4_ERR_CUDA;
  for (int64_t c = 0; c < nchunks; ++c) {
    const int i = static_cast<int>(c % W4A4_PIPE_DEPTH);
    const int64_t r0 = c * chunk_rows;
    const int64_t rows = (M - r0 < chunk_rows) ? M - r0 : chunk_rows;
    const Slot sl = slot_of(workspace, chunk_rows, w->K, w->N, i);
    const uint16_t *x = x_dev ? X_host + r0 * w->K : sl.x;
    uint16_t *y = y_dev ? Y_host + r0 * w->N : sl.y;
    if (!x_dev) {
      // X chunk in: its slot's X buffer was last read by compute of chunk c - DEPTH
      if (c >= W4A4_PIPE_DEPTH && cudaStreamWaitEvent(pipe->copy_in, pipe->ev_done[i], 0) != cudaSuccess)
        return W4A4_ERR_CUDA;
      if (cudaMemcpyAsync(sl.x, X_host + r0 * w->K, static_cast<size_t>(rows) * w->K * 2,
                          cudaMemcpyHostToDevice, pipe->copy_in) != cudaSuccess ||
          cudaEventRecord(pipe->ev_in[i], pipe->copy_in) != cudaSuccess)
        return W4A4_ERR_CUDA;
      // compute needs the X chunk
      if (cudaStreamWaitEvent(cs, pipe->ev_in[i], 0) != cudaSuccess) return W4A4_ERR_CUDA;
    }
    // ... and the slot's Y buffer drained by copy-out of chunk c - DEPTH
    if (!y_dev && c >= W4A4_PIPE_DEPTH && cudaStreamWaitEvent(cs, pipe->ev_out[i], 0) != cudaSuccess)
      return W4A4_ERR_CUDA;
    const w4a4_status s = w4a4_linear_fused(x, rows, w, y, sl.ws, sl.ws_bytes, flags, cs);
    if (s != W4A4_OK) return s;
    if (cudaEventRecord(pipe->ev_done[i], cs) != cudaSuccess) return W4A4_ERR_CUDA;
    // Y chunk out
    if (!y_dev &&
        (cudaStreamWaitEvent(pipe->copy_out, pipe->ev_done[i], 0) != cudaSuccess ||
         cudaMemcpyAsync(Y_host + r0 * w->N, sl.y, static_cast<size_t>(rows) * w->N * 2,
                         cudaMemcpyDeviceToHost, pipe->copy_out) != cudaSuccess ||
         cudaEventRecord(pipe->ev_out[i], pipe->copy_out) != cudaSuccess))
      return W4A4_ERR_CUDA;
  }
  // `stream` sees the call complete once the last copy-out has finished (the
  // copy-out stream is in order, so its latest event covers every chunk); with
  // Y in device memory the kernels on `stream` are the last work
  const int last = static_cast<int>((nchunks - 1) % W4A4_PIPE_DEPTH);
  if (!y_dev && cudaStreamWaitEvent(cs, pipe->ev_out[last], 0) != cudaSuccess) return W4A4_ERR_CUDA;
  return W4A4_OK;
}
