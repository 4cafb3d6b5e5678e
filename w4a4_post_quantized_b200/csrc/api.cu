// api.cu -- the C ABI of libw4a4 (include/w4a4.h): argument checks on the
// host, then kernel launches on the caller's stream.  No allocation, no
// synchronization (except w4a4_get_device_status), no exceptions.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "kernels.h"
#include "w4a4.h"

namespace {

constexpr uint32_t kKnownFlags = W4A4_FLAG_GELU | W4A4_FLAG_PLAIN | W4A4_FLAG_INT8 |
                                 W4A4_FLAG_UNPACKED | W4A4_FLAG_GELU_OUT | W4A4_FLAG_FWHT;
// flags of the activation quantizer (w4a4_quantize_act and the workspace sizes)
constexpr uint32_t kActFlags =
    W4A4_FLAG_GELU | W4A4_FLAG_PLAIN | W4A4_FLAG_INT8 | W4A4_FLAG_UNPACKED | W4A4_FLAG_FWHT;
constexpr uint32_t kWeightFlags = W4A4_FLAG_PLAIN | W4A4_FLAG_INT8;  // fixed at preparation

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool k_ok(int32_t K) { return K == 1024 || K == 4096; }
bool n_ok(int32_t N) { return N > 0 && N % 256 == 0; }
bool m_ok(int64_t M) { return M >= 0 && M < (int64_t(1) << 31); }
cudaStream_t as_stream(void *s) { return static_cast<cudaStream_t>(s); }
size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

w4a4_status cuda_status(cudaError_t e) { return e == cudaSuccess ? W4A4_OK : W4A4_ERR_CUDA; }

bool int8_weights(const w4a4_weights_t *w) { return (w->flags & W4A4_FLAG_INT8) != 0; }

w4a4_status check_weights(const w4a4_weights_t *w) {
  if (!w) return W4A4_ERR_ARG;
  if (!k_ok(w->K)) return W4A4_ERR_UNSUPPORTED;
  if (!n_ok(w->N)) return W4A4_ERR_SHAPE;
  if (w->flags & ~kWeightFlags) return W4A4_ERR_UNSUPPORTED;
  if (!w->scale_ch || !w->bias || !w->smooth || !w->inv_smooth) return W4A4_ERR_ARG;
  if (int8_weights(w)) {
    if (!w->qw8) return W4A4_ERR_ARG;  // the 8-bit codes; qw and colsum are not used
  } else {
    if (!w->qw) return W4A4_ERR_ARG;
    if ((w->qw8 == nullptr) != (w->colsum == nullptr)) return W4A4_ERR_ARG;
  }
  if (!aligned16(w->qw) || !aligned16(w->scale_ch) || !aligned16(w->bias) || !aligned16(w->smooth) ||
      !aligned16(w->inv_smooth) || !aligned16(w->qw8) || !aligned16(w->colsum))
    return W4A4_ERR_ALIGN;
  return W4A4_OK;
}

// one code per byte (int8 codes, or int4 codes in operand order) or two
bool one_per_byte(uint32_t flags) { return (flags & (W4A4_FLAG_INT8 | W4A4_FLAG_UNPACKED)) != 0; }

// code bytes of M rows of width K
size_t code_bytes(int64_t M, int32_t K, uint32_t flags) {
  return static_cast<size_t>(M) * (one_per_byte(flags) ? K : K / 2);
}
// The activation quantizer for these flags: the rotation on the tensor cores
// (quant_tc.cu) for DSFQ without GELU, unless W4A4_FLAG_FWHT asks for the
// CUDA-core transform; the CUDA-core kernel (quant.cu) otherwise.
cudaError_t quantize_rows(const uint16_t *X, int64_t M, int32_t K, const float *inv_smooth,
                          uint8_t *qx, float *scale_tok, uint32_t flags, w4a4::CodeFormat fmt,
                          cudaStream_t st) {
  const bool rot = !(flags & W4A4_FLAG_PLAIN), gelu = (flags & W4A4_FLAG_GELU) != 0;
  if (rot && !gelu && !(flags & W4A4_FLAG_FWHT))
    return w4a4::launch_quantize_rows_tc(X, M, K, inv_smooth, qx, scale_tok, fmt, st);
  return w4a4::launch_quantize_rows(X, M, K, inv_smooth, qx, scale_tok, rot, gelu, fmt, st);
}

w4a4::CodeFormat code_format(uint32_t flags) {
  if (flags & W4A4_FLAG_INT8) return w4a4::kCodeBytes8;
  return (flags & W4A4_FLAG_UNPACKED) ? w4a4::kCodeBytes4 : w4a4::kCodePacked4;
}

w4a4_status check_act(const void *X, int64_t M, int32_t K, const float *inv_smooth, const void *qx,
                      const float *scale_tok, uint32_t flags) {
  if (flags & ~kActFlags) return W4A4_ERR_UNSUPPORTED;
  if (!k_ok(K)) return W4A4_ERR_UNSUPPORTED;
  if (!m_ok(M)) return W4A4_ERR_SHAPE;
  if (M == 0) return W4A4_OK;
  if (!X || !qx || !scale_tok) return W4A4_ERR_ARG;
  if (!(flags & W4A4_FLAG_PLAIN) && !inv_smooth) return W4A4_ERR_ARG;
  if (!aligned16(X) || !aligned16(qx) || !aligned16(scale_tok) ||
      (inv_smooth && !aligned16(inv_smooth)))
    return W4A4_ERR_ALIGN;
  return W4A4_OK;
}

}  // namespace

extern "C" {

size_t w4a4_workspace_bytes_min(int64_t M, int32_t K, uint32_t flags) {
  if (!k_ok(K) || !m_ok(M) || (flags & ~kKnownFlags)) return 0;
  return round256(code_bytes(M, K, flags)) + sizeof(float) * static_cast<size_t>(M);
}

namespace {
// The arrays of a prepared layer in one allocation: byte offsets (each a
// multiple of 256) and sizes; SIZE_MAX marks an array the layout leaves out.
struct WeightsLayout {
  size_t qw, qw8, scale_ch, bias, smooth, inv_smooth, colsum, total;
};
constexpr size_t kAbsent = ~size_t(0);
constexpr uint32_t kLayoutFlags = W4A4_FLAG_PLAIN | W4A4_FLAG_INT8 | W4A4_FLAG_UNPACKED;

bool weights_layout(int32_t N, int32_t K, uint32_t flags, WeightsLayout *L) {
  if (!k_ok(K) || !n_ok(N) || (flags & ~kLayoutFlags)) return false;
  const bool int8 = (flags & W4A4_FLAG_INT8) != 0;
  const bool expanded = int8 || (flags & W4A4_FLAG_UNPACKED) != 0;
  const size_t n = static_cast<size_t>(N), k = static_cast<size_t>(K);
  size_t off = 0;
  auto place = [&](bool present, size_t bytes) {
    if (!present) return kAbsent;
    const size_t at = off;
    off += round256(bytes);
    return at;
  };
  L->qw = place(!int8, n * k / 2);
  L->qw8 = place(expanded, n * k);
  L->scale_ch = place(true, 4 * n);
  L->bias = place(true, 4 * n);
  L->smooth = place(true, 4 * k);
  L->inv_smooth = place(true, 4 * k);
  L->colsum = place(expanded && !int8, 4 * n);
  L->total = off;
  return true;
}
}  // namespace

size_t w4a4_weights_bytes(int32_t N, int32_t K, uint32_t flags) {
  WeightsLayout L;
  return weights_layout(N, K, flags, &L) ? L.total : 0;
}

w4a4_status w4a4_weights_bind(void *base, size_t bytes, int32_t N, int32_t K, uint32_t flags,
                              w4a4_weights_t *out) {
  if (!base || !out) return W4A4_ERR_ARG;
  if (flags & ~kLayoutFlags) return W4A4_ERR_UNSUPPORTED;
  if (!aligned16(base)) return W4A4_ERR_ALIGN;
  WeightsLayout L;
  if (!weights_layout(N, K, flags, &L)) return k_ok(K) ? W4A4_ERR_SHAPE : W4A4_ERR_UNSUPPORTED;
  if (bytes < L.total) return W4A4_ERR_SHAPE;
  uint8_t *b = static_cast<uint8_t *>(base);
  auto at = [&](size_t off) { return off == kAbsent ? nullptr : b + off; };
  out->N = N;
  out->K = K;
  out->qw = at(L.qw);
  out->qw8 = reinterpret_cast<int8_t *>(at(L.qw8));
  out->scale_ch = reinterpret_cast<float *>(at(L.scale_ch));
  out->bias = reinterpret_cast<float *>(at(L.bias));
  out->smooth = reinterpret_cast<float *>(at(L.smooth));
  out->inv_smooth = reinterpret_cast<float *>(at(L.inv_smooth));
  out->colsum = reinterpret_cast<int32_t *>(at(L.colsum));
  out->flags = 0;
  return W4A4_OK;
}

size_t w4a4_workspace_bytes(int64_t M, int32_t K) {
  return w4a4_workspace_bytes_min(M, K, W4A4_FLAG_UNPACKED);
}

w4a4_status w4a4_prepare_weights(const uint16_t *W, const uint16_t *bias, int32_t N, int32_t K,
                                 const uint16_t *X_calib, int64_t M_calib, float alpha,
                                 uint32_t flags, w4a4_weights_t *out, void *stream) {
  if (flags & ~kWeightFlags) return W4A4_ERR_UNSUPPORTED;
  if (!k_ok(K)) return W4A4_ERR_UNSUPPORTED;
  if (!n_ok(N)) return W4A4_ERR_SHAPE;
  if (!out || !W) return W4A4_ERR_ARG;
  const bool int8 = (flags & W4A4_FLAG_INT8) != 0;
  if (out->N != N || out->K != K) return W4A4_ERR_SHAPE;
  const bool plain = (flags & W4A4_FLAG_PLAIN) != 0;
  if (!plain) {
    if (!X_calib || M_calib < 1) return W4A4_ERR_ARG;
    if (!m_ok(M_calib)) return W4A4_ERR_SHAPE;
    if (!(alpha >= 0.0f && alpha <= 1.0f)) return W4A4_ERR_ARG;
    if (!aligned16(X_calib)) return W4A4_ERR_ALIGN;
  }
  if (!out->scale_ch || !out->bias || !out->smooth || !out->inv_smooth) return W4A4_ERR_ARG;
  if (int8 ? !out->qw8 : (!out->qw || (out->qw8 == nullptr) != (out->colsum == nullptr)))
    return W4A4_ERR_ARG;
  if (!aligned16(out->qw8) || !aligned16(out->colsum)) return W4A4_ERR_ALIGN;
  if (!aligned16(W) || (bias && !aligned16(bias)) || !aligned16(out->qw) ||
      !aligned16(out->scale_ch) || !aligned16(out->bias) || !aligned16(out->smooth) ||
      !aligned16(out->inv_smooth))
    return W4A4_ERR_ALIGN;
  cudaStream_t st = as_stream(stream);
  cudaError_t e;
  // 4-bit codes packed into qw, or 8-bit codes into qw8 (natural order)
  uint8_t *codes = int8 ? reinterpret_cast<uint8_t *>(out->qw8) : out->qw;
  const w4a4::CodeFormat fmt = int8 ? w4a4::kCodeBytes8 : w4a4::kCodePacked4;
  if (plain) {
    if ((e = w4a4::launch_fill(out->smooth, K, 1.0f, st)) != cudaSuccess) return cuda_status(e);
    if ((e = w4a4::launch_fill(out->inv_smooth, K, 1.0f, st)) != cudaSuccess) return cuda_status(e);
    e = w4a4::launch_quantize_rows(W, N, K, nullptr, codes, out->scale_ch, false, false, fmt, st);
  } else {
    // column maxima of the rotated calibration activations -> out->smooth,
    // of the rotated weights -> out->inv_smooth; then s and 1/s in place
    if ((e = w4a4::launch_colmax(X_calib, M_calib, K, out->smooth, st)) != cudaSuccess)
      return cuda_status(e);
    if ((e = w4a4::launch_colmax(W, N, K, out->inv_smooth, st)) != cudaSuccess) return cuda_status(e);
    if ((e = w4a4::launch_smooth_factors(out->smooth, out->inv_smooth, K, alpha, st)) != cudaSuccess)
      return cuda_status(e);
    e = w4a4::launch_quantize_rows(W, N, K, out->smooth, codes, out->scale_ch, true, false, fmt, st);
  }
  if (e != cudaSuccess) return cuda_status(e);
  if ((e = w4a4::launch_bias_to_f32(bias, out->bias, N, st)) != cudaSuccess) return cuda_status(e);
  out->flags = flags & kWeightFlags;
  if (!int8 && out->qw8) return w4a4_expand_weights(out, stream);
  return W4A4_OK;
}

w4a4_status w4a4_expand_weights(w4a4_weights_t *w, void *stream) {
  if (!w) return W4A4_ERR_ARG;
  if (!k_ok(w->K)) return W4A4_ERR_UNSUPPORTED;
  if (!n_ok(w->N)) return W4A4_ERR_SHAPE;
  if (!w->qw || !w->qw8 || !w->colsum) return W4A4_ERR_ARG;
  if (w->flags & W4A4_FLAG_INT8) return W4A4_ERR_ARG;  // 8-bit codes need no widening
  if (!aligned16(w->qw) || !aligned16(w->qw8) || !aligned16(w->colsum)) return W4A4_ERR_ALIGN;
  return cuda_status(w4a4::launch_expand_weights(w->qw, w->N, w->K, w->qw8, w->colsum,
                                                 as_stream(stream)));
}

w4a4_status w4a4_quantize_act(const uint16_t *X, int64_t M, int32_t K, const float *inv_smooth,
                              uint8_t *qx, float *scale_tok, uint32_t flags, void *stream) {
  if ((flags & W4A4_FLAG_INT8) && (flags & W4A4_FLAG_UNPACKED)) return W4A4_ERR_UNSUPPORTED;
  w4a4_status s = check_act(X, M, K, inv_smooth, qx, scale_tok, flags);
  if (s != W4A4_OK) return s;
  return cuda_status(quantize_rows(X, M, K, inv_smooth, qx, scale_tok, flags, code_format(flags),
                                   as_stream(stream)));
}

w4a4_status w4a4_linear_ex(const uint8_t *qx, const float *scale_tok, int64_t M,
                           const w4a4_weights_t *w, uint16_t *Y, uint32_t flags, void *stream) {
  w4a4_status s = check_weights(w);
  if (s != W4A4_OK) return s;
  if (flags & ~(W4A4_FLAG_UNPACKED | W4A4_FLAG_GELU_OUT)) return W4A4_ERR_UNSUPPORTED;
  // one-per-byte 4-bit codes pair with the expanded weight codes
  if ((flags & W4A4_FLAG_UNPACKED) && (int8_weights(w) || !w->qw8)) return W4A4_ERR_ARG;
  if (!m_ok(M)) return W4A4_ERR_SHAPE;
  if (M == 0) return W4A4_OK;
  if (!qx || !scale_tok || !Y) return W4A4_ERR_ARG;
  if (!aligned16(qx) || !aligned16(scale_tok) || !aligned16(Y)) return W4A4_ERR_ALIGN;
  w4a4::GemmArgs a{qx, w->qw, w->qw8, w->colsum, scale_tok, w->scale_ch, w->bias, Y, nullptr,
                   M, w->N, w->K, int8_weights(w) || (flags & W4A4_FLAG_UNPACKED) != 0,
                   (flags & W4A4_FLAG_GELU_OUT) != 0};
  a.acc22 = !int8_weights(w);
  return cuda_status(w4a4::launch_gemm(a, as_stream(stream)));
}

w4a4_status w4a4_linear(const uint8_t *qx, const float *scale_tok, int64_t M,
                        const w4a4_weights_t *w, uint16_t *Y, void *stream) {
  return w4a4_linear_ex(qx, scale_tok, M, w, Y, 0, stream);
}

w4a4_status w4a4_linear_fused(const uint16_t *X, int64_t M, const w4a4_weights_t *w, uint16_t *Y,
                              void *workspace, size_t workspace_bytes, uint32_t flags,
                              void *stream) {
  w4a4_status s = check_weights(w);
  if (s != W4A4_OK) return s;
  if (flags & ~kKnownFlags) return W4A4_ERR_UNSUPPORTED;
  if (flags & W4A4_FLAG_UNPACKED) return W4A4_ERR_UNSUPPORTED;  // the call picks the route
  if ((flags ^ w->flags) & kWeightFlags) return W4A4_ERR_ARG;
  if (!m_ok(M)) return W4A4_ERR_SHAPE;
  if (M == 0) return W4A4_OK;  // empty input: nothing to read or write
  if (!X || !Y || !workspace) return W4A4_ERR_ARG;
  if (workspace_bytes < w4a4_workspace_bytes_min(M, w->K, flags)) return W4A4_ERR_SHAPE;
  if (!aligned16(X) || !aligned16(Y) || !aligned16(workspace)) return W4A4_ERR_ALIGN;
  // 4-bit codes go one per byte (in the operand order of the expanded weights)
  // when the weights carry that expansion and the workspace has the room: the
  // GEMM then reads them without widening each tile again; else packed.
  uint32_t cf = flags;
  if (!int8_weights(w) && w->qw8 &&
      workspace_bytes >= w4a4_workspace_bytes_min(M, w->K, flags | W4A4_FLAG_UNPACKED))
    cf |= W4A4_FLAG_UNPACKED;
  uint8_t *qx = static_cast<uint8_t *>(workspace);
  float *st = reinterpret_cast<float *>(qx + round256(code_bytes(M, w->K, cf)));
  cudaStream_t cs = as_stream(stream);
  cudaError_t e = quantize_rows(X, M, w->K, w->inv_smooth, qx, st, flags, code_format(cf), cs);
  if (e != cudaSuccess) return cuda_status(e);
  w4a4::GemmArgs a{qx, w->qw, w->qw8, w->colsum, st, w->scale_ch, w->bias, Y, nullptr,
                   M, w->N, w->K, one_per_byte(cf), (flags & W4A4_FLAG_GELU_OUT) != 0};
  a.acc22 = !int8_weights(w);
  return cuda_status(w4a4::launch_gemm(a, cs));
}

w4a4_status w4a4_gemm_s32_ex(const uint8_t *qx, int64_t M, const w4a4_weights_t *w, int32_t *acc,
                             uint32_t flags, void *stream) {
  if (!w) return W4A4_ERR_ARG;
  if (flags & ~(W4A4_FLAG_UNPACKED | W4A4_DEBUG_STALL)) return W4A4_ERR_UNSUPPORTED;
  if (!k_ok(w->K)) return W4A4_ERR_UNSUPPORTED;
  if (!n_ok(w->N) || !m_ok(M)) return W4A4_ERR_SHAPE;
  if (w->flags & ~kWeightFlags) return W4A4_ERR_UNSUPPORTED;
  const bool int8 = int8_weights(w);
  if (int8 ? !w->qw8 : ((w->qw8 == nullptr) != (w->colsum == nullptr))) return W4A4_ERR_ARG;
  const bool unpacked = (flags & W4A4_FLAG_UNPACKED) != 0;
  if (unpacked && (int8 || !w->qw8)) return W4A4_ERR_ARG;
  if (M == 0) return W4A4_OK;
  if (!qx || !acc || (!w->qw && !w->qw8)) return W4A4_ERR_ARG;
  if (!aligned16(qx) || !aligned16(acc) || !aligned16(w->qw) || !aligned16(w->qw8) ||
      !aligned16(w->colsum))
    return W4A4_ERR_ALIGN;
  w4a4::GemmArgs a{qx, w->qw, w->qw8, w->colsum, nullptr, nullptr, nullptr, nullptr, acc,
                   M, w->N, w->K, int8 || unpacked};
  a.stall = (flags & W4A4_DEBUG_STALL) != 0;
  return cuda_status(w4a4::launch_gemm(a, as_stream(stream)));
}

w4a4_status w4a4_gemm_s32(const uint8_t *qx, int64_t M, const w4a4_weights_t *w, int32_t *acc,
                          void *stream) {
  return w4a4_gemm_s32_ex(qx, M, w, acc, 0, stream);
}

w4a4_status w4a4_get_device_status(void *stream, uint32_t *status) {
  if (!status) return W4A4_ERR_ARG;
  unsigned int v = 0;
  cudaError_t e = w4a4::read_status(&v, as_stream(stream));
  if (e != cudaSuccess) return W4A4_ERR_CUDA;
  *status = v;
  return v ? W4A4_ERR_TIMEOUT : W4A4_OK;
}

w4a4_status w4a4_clear_device_status(void *stream) {
  return cuda_status(w4a4::clear_status(as_stream(stream)));
}

const char *w4a4_status_string(w4a4_status s) {
  switch (s) {
    case W4A4_OK: return "ok";
    case W4A4_ERR_ARG: return "invalid argument";
    case W4A4_ERR_SHAPE: return "unsupported shape or workspace size";
    case W4A4_ERR_ALIGN: return "misaligned pointer";
    case W4A4_ERR_UNSUPPORTED: return "unsupported K or flag";
    case W4A4_ERR_CUDA: return "CUDA error";
    case W4A4_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

const char *w4a4_version(void) { return "libw4a4 0.1 (sm_100a)"; }

}  // extern "C"
