// kernels.h -- internal launchers shared by the C-ABI layer (api.cu) and the
// kernel translation units.  Not part of the public interface.
#pragma once

#include <cuda.h>  // CUtensorMap types (the encode function is fetched at run time)
#include <cuda_runtime.h>

#include <cstdint>

namespace w4a4 {

int device_sm_count();

// quant.cu
// Code formats of the quantize kernel:
//   kCodePacked4  int4 codes, two per byte (q [M, K/2])
//   kCodeBytes4   int4 codes, one per byte in the tensor-core operand order
//                 (within every 8 elements: 0, 2, 4, 6, 1, 3, 5, 7) (q [M, K])
//   kCodeBytes8   int8 codes (step absmax / 127), natural order (q [M, K])
enum CodeFormat : int { kCodePacked4 = 0, kCodeBytes4 = 1, kCodeBytes8 = 2 };
cudaError_t launch_quantize_rows(const uint16_t *X, int64_t M, int K, const float *mult,
                                 uint8_t *q, float *scale, bool rot, bool gelu, CodeFormat code,
                                 cudaStream_t st);
cudaError_t launch_colmax(const uint16_t *X, int64_t M, int K, float *colmax, cudaStream_t st);
cudaError_t launch_smooth_factors(float *s_io, float *inv_io, int K, double alpha, cudaStream_t st);
cudaError_t launch_bias_to_f32(const uint16_t *b, float *out, int n, cudaStream_t st);
cudaError_t launch_fill(float *out, int n, float v, cudaStream_t st);

// gemm.cu
struct GemmArgs {
  const uint8_t *qx;        // [M, K/2] packed int4, or [M, K] one code per byte when a8
  const uint8_t *qw;        // [N, K/2] packed int4 (used when qw8 == nullptr)
  const int8_t *qw8;        // [N, K] one weight code per byte (same order as qx when a8), or nullptr
  const int32_t *colsum;    // [N] per-row code sums (with qw8)
  const float *scale_tok;   // [M]
  const float *scale_ch;    // [N]
  const float *bias;        // [N]
  uint16_t *y;              // [M, N] bf16 (when acc == nullptr)
  int32_t *acc;             // [M, N] int32 accumulators instead of y (test path)
  int64_t M;
  int N, K;
  bool a8;                  // qx and qw8 hold one code per byte in the same order (int8 codes,
                            // or int4 codes in operand order): no widening
  bool gelu_out = false;    // y = bf16(GELU(bf16 result)) (an MLP's first linear)
  bool stall = false;       // failure-path test: the TMA producer issues nothing and every
                            // bounded wait gives up after 1 ms (sets the status word)
  bool acc22 = false;       // every accumulator is below 2^22 in magnitude (4-bit weight codes
                            // in [-7, 7], activation bytes in [-128, 127], K <= 4096): with
                            // byte operands the epilogue converts them with the exact
                            // integer-add bias instead of the int -> float conversion
};
cudaError_t launch_gemm(const GemmArgs &a, cudaStream_t st);
cudaError_t launch_expand_weights(const uint8_t *qw, int N, int K, int8_t *qw8, int32_t *colsum,
                                  cudaStream_t st);

// A 2-D TMA tensor map (cuTensorMapEncodeTiled through the runtime's driver
// entry point): `outer` rows of `inner` elements, rows `row_bytes` apart, box
// box_inner x box_outer, no interleave, 256-byte L2 promotion, zero fill.
bool encode_tensor_map_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t inner,
                          uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                          CUtensorMapSwizzle swz);

// quant_tc.cu: the activation quantizer with the rotation on the tensor cores
// (DSFQ: rotation and smoothing on; no GELU).  Same arguments and outputs as
// launch_quantize_rows with rot = true, gelu = false.
cudaError_t launch_quantize_rows_tc(const uint16_t *X, int64_t M, int K, const float *mult,
                                    uint8_t *q, float *scale, CodeFormat code, cudaStream_t st);

// status word: *out = its device address in the current context (for kernel
// arguments); an error when the lookup fails (nothing may then be launched)
cudaError_t status_word(unsigned int **out);
cudaError_t read_status(unsigned int *out, cudaStream_t st);
cudaError_t clear_status(cudaStream_t st);

}  // namespace w4a4
