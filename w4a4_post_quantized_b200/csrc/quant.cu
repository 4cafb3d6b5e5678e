// quant.cu -- the HBM-bound half of the DSFQ W4A4 linear on sm_100a:
//   * quantize_rows: bf16 row -> (optional GELU) -> Hadamard rotation (fast
//     Walsh-Hadamard transform, fp32) -> per-channel multiplier -> per-row
//     absmax -> symmetric int4 codes packed two per byte + fp32 step.
//     Activations use multiplier 1/s (pre-global rotation, then post-local
//     smoothing), weights use s; both follow page "十亿参数的三维重建模型，能塞进手机吗？",
//     sections 预全局旋转 / 后局部平滑 / 训练后量化（PTQ） / 细粒度量化粒度.
//   * colmax: per-channel max |rotated value| over rows (the statistics the
//     smoothing factors are computed from).
//   * smooth_factors, bias conversion, fill: small offline helpers.
//
// Row layout (one warp per row of K = 32*V values):
//   phase 1: lane l holds x[l + 32 j], j < V: 16-bit loads, every warp-wide
//            load instruction covers 64 contiguous bytes.  The butterflies over
//            the bits of j (index bits 5 .. log2 K - 1) run in registers.
//   transpose through a 32 x 32 fp32 shared-memory tile per warp (XOR-swizzled
//            columns, conflict-free both ways), P = V/32 passes.
//   phase 2: lane l holds x[V l + r], r < V: the butterflies over index bits
//            0..4 run in registers; each lane then owns V consecutive outputs,
//            i.e. V/2 consecutive bytes of packed codes, stored with 16-byte
//            stores.
// The transform is the Sylvester (natural-order) Hadamard product x H, scaled
// by 1/sqrt(K) (an exact power of two for K = 1024 and 4096).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.h"

namespace w4a4 {

namespace {

constexpr int kQuantWarps = 8;  // warps per block of the row kernels

__device__ __forceinline__ float bf16_bits_to_float(unsigned short h) {
  return __uint_as_float(static_cast<uint32_t>(h) << 16);
}

// Exact-erf GELU evaluated in fp32, rounded to bf16 (the activation an MLP's
// second linear receives).
__device__ __forceinline__ float gelu_bf16(float x) {
  const float g = 0.5f * x * (1.0f + erff(x * 0.70710678118654752f));
  return __bfloat162float(__float2bfloat16_rn(g));
}

// Butterflies for index bits [B0, B0 + NB) of a register array (natural order:
// the lower index of each pair receives the sum).
template <int V, int B0, int NB>
__device__ __forceinline__ void butterflies(float (&v)[V]) {
#pragma unroll
  for (int s = 0; s < NB; ++s) {
    const int h = 1 << (B0 + s);
#pragma unroll
    for (int j = 0; j < V; ++j) {
      if ((j & h) == 0) {
        const float a = v[j], b = v[j + h];
        v[j] = a + b;
        v[j + h] = a - b;
      }
    }
  }
}

template <int K>
struct RowShape {
  static constexpr int V = K / 32;  // values per lane
  static constexpr int P = V / 32;  // transpose passes
  static constexpr int LOGV = (V == 32) ? 5 : 7;
  static constexpr float kInvSqrtK = (K == 1024) ? 0.03125f : 0.015625f;
  static_assert(K == 1024 || K == 4096, "K must be 1024 or 4096");
};

// Loads one row in phase-1 layout, applies optional GELU, runs the full
// transform (when ROT) and leaves the row in phase-2 layout in v.
template <int K, bool ROT, bool GELU>
__device__ __forceinline__ void load_transform_row(const uint16_t *__restrict__ xrow, int lane,
                                                   float *__restrict__ tile,
                                                   float (&v)[RowShape<K>::V]) {
  constexpr int V = RowShape<K>::V;
  constexpr int P = RowShape<K>::P;
  const unsigned short *x = reinterpret_cast<const unsigned short *>(xrow);
  float u[V];
#pragma unroll
  for (int j = 0; j < V; ++j) {
    float f = bf16_bits_to_float(__ldcs(x + lane + 32 * j));
    if (GELU) f = gelu_bf16(f);
    u[j] = f;
  }
  if (ROT) butterflies<V, 0, RowShape<K>::LOGV>(u);  // index bits 5 .. log2(K)-1
  // transpose: value u[P*l2 + p] of lane l moves to lane l2, register 32p + l
#pragma unroll
  for (int p = 0; p < P; ++p) {
#pragma unroll
    for (int l2 = 0; l2 < 32; ++l2) tile[l2 * 32 + (lane ^ l2)] = u[P * l2 + p];
    __syncwarp();
#pragma unroll
    for (int l = 0; l < 32; ++l) v[32 * p + l] = tile[lane * 32 + (l ^ lane)];
    __syncwarp();
  }
  if (ROT) butterflies<V, 0, 5>(v);  // index bits 0..4
}

// quantize_rows: one warp per row, grid-stride over rows.
template <int K, bool ROT, bool GELU>
__global__ void __launch_bounds__(kQuantWarps * 32)
    quantize_rows_kernel(const uint16_t *__restrict__ X, int64_t M, const float *__restrict__ mult,
                         uint8_t *__restrict__ q, float *__restrict__ scale) {
  constexpr int V = RowShape<K>::V;
  __shared__ float tiles[kQuantWarps][32 * 32];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  float *tile = tiles[warp];
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kQuantWarps;
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * kQuantWarps + warp; row < M; row += stride) {
    float v[V];
    load_transform_row<K, ROT, GELU>(X + row * K, lane, tile, v);
    if (ROT) {
      const float4 *m4 = reinterpret_cast<const float4 *>(mult + static_cast<int64_t>(V) * lane);
#pragma unroll
      for (int c = 0; c < V / 4; ++c) {
        const float4 m = __ldg(m4 + c);
        v[4 * c + 0] *= m.x * RowShape<K>::kInvSqrtK;
        v[4 * c + 1] *= m.y * RowShape<K>::kInvSqrtK;
        v[4 * c + 2] *= m.z * RowShape<K>::kInvSqrtK;
        v[4 * c + 3] *= m.w * RowShape<K>::kInvSqrtK;
      }
    }
    float amax = 0.0f;
#pragma unroll
    for (int r = 0; r < V; ++r) amax = fmaxf(amax, fabsf(v[r]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if (lane == 0) scale[row] = amax / 7.0f;
    // rows whose maximum is tiny are rescaled by an exact power of two so that
    // 7/amax stays finite; the scaled product equals the unscaled one
    const float pre = (amax < 0x1p-100f) ? 0x1p+100f : 1.0f;
    const float inv = (amax > 0.0f) ? 7.0f / (amax * pre) : 0.0f;
    // code = round-half-even(v * inv); |v * inv| <= 7 (1 + 2^-24), so no clamp
    // can ever act.  Adding 1.5 * 2^23 in the same fused operation rounds the
    // exact product to an integer whose low 4 bits are the two's-complement code.
    uint32_t words[V / 8];
#pragma unroll
    for (int w = 0; w < V / 8; ++w) {
      uint32_t acc = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float f = fmaf(v[8 * w + k] * pre, inv, 12582912.0f);
        acc |= (__float_as_uint(f) & 0xFu) << (4 * k);
      }
      words[w] = acc;
    }
    uint4 *dst = reinterpret_cast<uint4 *>(q + row * (K / 2) + static_cast<int64_t>(lane) * (V / 2));
#pragma unroll
    for (int c = 0; c < V / 32; ++c)
      dst[c] = make_uint4(words[4 * c + 0], words[4 * c + 1], words[4 * c + 2], words[4 * c + 3]);
  }
}

// colmax: colmax[j] = max over rows of |(x H / sqrt(K))[j]| (as float bits,
// atomically max-reduced; colmax must be zero on entry).
template <int K>
__global__ void __launch_bounds__(kQuantWarps * 32)
    colmax_kernel(const uint16_t *__restrict__ X, int64_t M, unsigned int *__restrict__ colmax) {
  constexpr int V = RowShape<K>::V;
  __shared__ float tiles[kQuantWarps][32 * 32];
  __shared__ unsigned int cm[K];
  for (int i = threadIdx.x; i < K; i += blockDim.x) cm[i] = 0u;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kQuantWarps;
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * kQuantWarps + warp; row < M; row += stride) {
    float v[V];
    load_transform_row<K, true, false>(X + row * K, lane, tiles[warp], v);
#pragma unroll
    for (int r = 0; r < V; ++r)
      atomicMax(&cm[V * lane + r], __float_as_uint(fabsf(v[r] * RowShape<K>::kInvSqrtK)));
  }
  __syncthreads();
  for (int i = threadIdx.x; i < K; i += blockDim.x)
    if (cm[i]) atomicMax(&colmax[i], cm[i]);
}

// s_j = cx^alpha / cw^(1-alpha) (1 when either maximum is zero), evaluated in
// fp64 and rounded to fp32; inv_s = 1/s.  In place: reads the maxima from
// s_io (activations) and inv_io (weights).
__global__ void smooth_factors_kernel(float *__restrict__ s_io, float *__restrict__ inv_io, int K,
                                      double alpha) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= K) return;
  const double cx = s_io[j], cw = inv_io[j];
  double s = 1.0;
  if (cx > 0.0 && cw > 0.0) s = pow(cx, alpha) / pow(cw, 1.0 - alpha);
  s_io[j] = static_cast<float>(s);
  inv_io[j] = static_cast<float>(1.0 / s);
}

__global__ void bias_to_f32_kernel(const uint16_t *__restrict__ b, float *__restrict__ out, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = b ? bf16_bits_to_float(b[i]) : 0.0f;
}

__global__ void fill_kernel(float *__restrict__ out, int n, float v) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = v;
}

int g_num_sms = 0;

int num_sms() {
  if (g_num_sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (g_num_sms <= 0) g_num_sms = 148;
  }
  return g_num_sms;
}

template <typename Kern>
int row_grid(Kern kern, int64_t rows) {
  int per_sm = 0;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kQuantWarps * 32, 0);
  if (per_sm < 1) per_sm = 1;
  const int64_t need = (rows + kQuantWarps - 1) / kQuantWarps;
  const int64_t g = static_cast<int64_t>(num_sms()) * per_sm;
  return static_cast<int>(need < g ? need : g);
}

template <int K, bool ROT, bool GELU>
cudaError_t launch_quant_k(const uint16_t *X, int64_t M, const float *mult, uint8_t *q,
                           float *scale, cudaStream_t st) {
  auto kern = quantize_rows_kernel<K, ROT, GELU>;
  const int grid = row_grid(kern, M);
  kern<<<grid, kQuantWarps * 32, 0, st>>>(X, M, mult, q, scale);
  return cudaGetLastError();
}

}  // namespace

int device_sm_count() { return num_sms(); }

cudaError_t launch_quantize_rows(const uint16_t *X, int64_t M, int K, const float *mult,
                                 uint8_t *q, float *scale, bool rot, bool gelu, cudaStream_t st) {
  if (M <= 0) return cudaSuccess;
  if (K == 1024) {
    if (rot) return gelu ? launch_quant_k<1024, true, true>(X, M, mult, q, scale, st)
                         : launch_quant_k<1024, true, false>(X, M, mult, q, scale, st);
    return gelu ? launch_quant_k<1024, false, true>(X, M, mult, q, scale, st)
                : launch_quant_k<1024, false, false>(X, M, mult, q, scale, st);
  }
  if (rot) return gelu ? launch_quant_k<4096, true, true>(X, M, mult, q, scale, st)
                       : launch_quant_k<4096, true, false>(X, M, mult, q, scale, st);
  return gelu ? launch_quant_k<4096, false, true>(X, M, mult, q, scale, st)
              : launch_quant_k<4096, false, false>(X, M, mult, q, scale, st);
}

cudaError_t launch_colmax(const uint16_t *X, int64_t M, int K, float *colmax, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(colmax, 0, sizeof(float) * K, st);
  if (e != cudaSuccess || M <= 0) return e;
  if (K == 1024) {
    const int grid = row_grid(colmax_kernel<1024>, M);
    colmax_kernel<1024><<<grid, kQuantWarps * 32, 0, st>>>(X, M, reinterpret_cast<unsigned int *>(colmax));
  } else {
    const int grid = row_grid(colmax_kernel<4096>, M);
    colmax_kernel<4096><<<grid, kQuantWarps * 32, 0, st>>>(X, M, reinterpret_cast<unsigned int *>(colmax));
  }
  return cudaGetLastError();
}

cudaError_t launch_smooth_factors(float *s_io, float *inv_io, int K, double alpha, cudaStream_t st) {
  smooth_factors_kernel<<<(K + 255) / 256, 256, 0, st>>>(s_io, inv_io, K, alpha);
  return cudaGetLastError();
}

cudaError_t launch_bias_to_f32(const uint16_t *b, float *out, int n, cudaStream_t st) {
  bias_to_f32_kernel<<<(n + 255) / 256, 256, 0, st>>>(b, out, n);
  return cudaGetLastError();
}

cudaError_t launch_fill(float *out, int n, float v, cudaStream_t st) {
  fill_kernel<<<(n + 255) / 256, 256, 0, st>>>(out, n, v);
  return cudaGetLastError();
}

}  // namespace w4a4
