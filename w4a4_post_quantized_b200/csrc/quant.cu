// quant.cu -- the HBM-bound half of the DSFQ W4A4 linear on sm_100a:
//   * quantize_rows: bf16 row -> (optional GELU) -> Hadamard rotation (fast
//     Walsh-Hadamard transform, fp32) -> per-channel multiplier -> per-row
//     absmax -> symmetric int4 codes + fp32 step.  Three code formats:
//     int4 packed two per byte (the storage format); int4 one per byte in the
//     tensor-core operand order (within every 8 elements: 0, 2, 4, 6, 1, 3,
//     5, 7 -- the order of the expanded weights), which the GEMM then reads
//     without widening; int8 one per byte in natural order with step
//     absmax / 127 (the W8A8 setting).
//     Activations use multiplier 1/s (pre-global rotation, then post-local
//     smoothing), weights use s; both follow page "十亿参数的三维重建模型，能塞进手机吗？",
//     sections 预全局旋转 / 后局部平滑 / 训练后量化（PTQ） / 细粒度量化粒度.
//   * colmax: per-channel max |rotated value| over rows (the statistics the
//     smoothing factors are computed from).
//   * smooth_factors, bias conversion, fill: small offline helpers.
//
// Row layout (one warp per row of K = 32*V values; the transform routine,
// transform_row, is in fwht.cuh):
//   phase 1: lane l holds x[l + 32 j], j < V: 16-bit loads, every warp-wide
//            load instruction covers 64 contiguous bytes.  The butterflies over
//            the bits of j (index bits 5 .. log2 K - 1) run in registers.
//   transpose through a 32 x 32 fp32 shared-memory tile per warp, P = V/32
//            passes: each lane writes its 32 values of a pass as one tile row
//            with 16-byte stores (16-byte chunk c of row l at chunk position
//            c ^ (l % 8): conflict-free both ways) and reads a column back.
//            Phase-1 values sit in register slot phase1_slot(j) so that each
//            16-byte store takes four consecutive slots.
//   phase 2: lane l holds x[V l + r], r < V: the butterflies over index bits
//            0..4 run in registers; each lane then owns V consecutive outputs,
//            i.e. V/2 (packed) or V (one per byte) consecutive code bytes,
//            stored with 16-byte stores.
// Packed fp32x2 instructions do two butterflies, products or fused
// multiply-adds at once; adjacent register slots (2m, 2m + 1) form the pairs.
// The transform is the Sylvester (natural-order) Hadamard product x H, scaled
// by 1/sqrt(K) (an exact power of two for K = 1024 and 4096).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "codes.cuh"
#include "ctxcache.h"
#include "fwht.cuh"
#include "gelu.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace w4a4 {

namespace {

constexpr int kQuantWarps = 8;  // warps per block of the row kernels

__device__ __forceinline__ float bf16_bits_to_float(unsigned short h) {
  return __uint_as_float(static_cast<uint32_t>(h) << 16);
}

// Phase-1 load of one row: u[j] = x[lane + 32 j] (optional GELU).  `x` points
// at the row in global or shared memory.
template <int K, bool GELU, bool FROM_SMEM>
__device__ __forceinline__ void load_phase1(const unsigned short *__restrict__ x, int lane,
                                            float (&u)[RowShape<K>::V]) {
  constexpr int V = RowShape<K>::V;
#pragma unroll
  for (int j = 0; j < V; j += 2) {
    float f0 = bf16_bits_to_float(FROM_SMEM ? x[lane + 32 * j] : __ldcs(x + lane + 32 * j));
    float f1 = bf16_bits_to_float(FROM_SMEM ? x[lane + 32 * (j + 1)] : __ldcs(x + lane + 32 * (j + 1)));
    if (GELU) gelu2_bf16(f0, f1);
    u[phase1_slot<K>(j)] = f0;
    u[phase1_slot<K>(j + 1)] = f1;
  }
}

// Per-channel multiplier (from the block's shared table) and this lane's
// absmax of a phase-2 row (V values).
template <int V, bool ROT>
__device__ __forceinline__ float mult_lane_absmax(float (&v)[V], int lane,
                                                  const float4 *__restrict__ mtab) {
  if (ROT) {
#pragma unroll
    for (int c = 0; c < V / 4; ++c) {
      const float4 m = mtab[c * 32 + lane];
      mul_x2(v[4 * c + 0], v[4 * c + 1], m.x, m.y);
      mul_x2(v[4 * c + 2], v[4 * c + 3], m.z, m.w);
    }
  }
  float am[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
  for (int r = 0; r < V; r += 8)
#pragma unroll
    for (int a = 0; a < 4; ++a) am[a] = fmax3(am[a], fabsf(v[r + 2 * a]), fabsf(v[r + 2 * a + 1]));
  return fmax3(am[0], am[1], fmaxf(am[2], am[3]));
}

// Per-channel multiplier, per-row absmax, codes, store for a phase-2 row.
// The transform's 1/sqrt(K) is an exact power of two, so it changes neither
// the absmax position nor any code: it is applied to the stored step only.
// CODE (CodeFormat): kCodePacked4 codes in [-7, 7] two per byte; kCodeBytes4
// the same codes one per byte in operand order; kCodeBytes8 codes in
// [-127, 127] one per byte.
template <int K, bool ROT, int CODE>
__device__ __forceinline__ void quantize_store_row(float (&v)[RowShape<K>::V], int lane, int64_t row,
                                                   const float4 *__restrict__ mtab,
                                                   uint8_t *__restrict__ q, float *__restrict__ scale) {
  constexpr int V = RowShape<K>::V;
  float amax = mult_lane_absmax<V, ROT>(v, lane, mtab);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  constexpr float kQmax = CODE == kCodeBytes8 ? 127.0f : 7.0f;
  if (lane == 0) scale[row] = (ROT ? amax * RowShape<K>::kInvSqrtK : amax) / kQmax;
  store_codes<V, CODE>(v, amax, q + row * code_bytes_of<CODE>(K) + lane * code_bytes_of<CODE>(V));
}

template <int K>
struct QuantStaging {
  static constexpr int ROWB = 2 * K;                 // bf16 row bytes
  // rows in flight per warp: K = 1024 uses one slot, refilled as soon as the
  // row has been read into registers (measured faster than two slots)
  static constexpr int NS = K == 1024 ? 1 : 2;
  static constexpr int WARP_BYTES = NS * ROWB + 32 * 32 * 4;
  static constexpr int OFF_TAB = kQuantWarps * WARP_BYTES;        // multiplier table, K floats
  static constexpr int OFF_BAR = OFF_TAB + 4 * K;
  static constexpr int SMEM = OFF_BAR + kQuantWarps * NS * 8;
};

// quantize_rows: one warp per row, grid-stride over rows.  Each warp keeps
// NS rows in flight: 1-D bulk copies (TMA engine) stream its next rows into a
// private shared-memory ring while it transforms the current one, so the HBM
// latency is hidden without occupancy.
template <int K, bool ROT, bool GELU, int CODE>
__global__ void __launch_bounds__(kQuantWarps * 32)
    quantize_rows_kernel(const uint16_t *__restrict__ X, int64_t M, const float *__restrict__ mult,
                         uint8_t *__restrict__ q, float *__restrict__ scale,
                         unsigned int *__restrict__ status) {
  using S = QuantStaging<K>;
  constexpr int V = RowShape<K>::V;
  extern __shared__ __align__(1024) uint8_t qsmem[];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  uint8_t *ring = qsmem + warp * S::WARP_BYTES;
  float *tile = reinterpret_cast<float *>(ring + S::NS * S::ROWB);
  uint64_t *bars = reinterpret_cast<uint64_t *>(qsmem + S::OFF_BAR) + warp * S::NS;
  float4 *mtab = reinterpret_cast<float4 *>(qsmem + S::OFF_TAB);
  // rows r0, r0 + G, ...: consecutive r0 go to different blocks, so the rows
  // of the last, partial round are spread over all SMs
  const int64_t G = static_cast<int64_t>(gridDim.x) * kQuantWarps;
  const int64_t r0 = static_cast<int64_t>(warp) * gridDim.x + blockIdx.x;
  int64_t issued = 0;  // rows whose copy lane 0 has issued (sequence numbers 0..issued-1)
  if (lane == 0) {
    for (int s = 0; s < S::NS; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  // The barrier setup above may overlap the tail of the previous kernel of the
  // stream; X, mult, q and scale are touched only after it has completed.
  griddep_launch_dependents();
  griddep_wait();
  if (lane == 0) {
    fence_proxy_async_smem();
    // the first row now; the ring's second slot is filled once it has landed
    // (below), so at start-up every warp's first row arrives sooner
    if (r0 < M) {
      mbar_arrive_expect_tx(&bars[0], S::ROWB);
      bulk_load(ring, X + r0 * K, S::ROWB, &bars[0]);
      ++issued;
    }
  }
  if (ROT) {
    // (after the first copy is on its way) table[(r/4)*32 + l] holds
    // mult[V l + r .. +3]: lane l's 16-byte reads of one chunk are consecutive
    // across the warp (conflict-free)
    float *t = reinterpret_cast<float *>(mtab);
    for (int j = threadIdx.x; j < K; j += blockDim.x) {
      const int l = j / V, r = j % V;
      t[((r >> 2) * 32 + l) * 4 + (r & 3)] = __ldg(mult + j);
    }
    __syncthreads();
  }
  __syncwarp();
  int64_t i = 0;
  for (int64_t row = r0; row < M; row += G, ++i) {
    const int s = static_cast<int>(i % S::NS);
    if (!mbar_wait_drain(&bars[s], static_cast<uint32_t>((i / S::NS) & 1), status)) break;
    if (S::NS == 2 && i == 0 && lane == 0) {  // the ring's second slot
      const int64_t r = r0 + G;
      if (r < M) {
        mbar_arrive_expect_tx(&bars[1], S::ROWB);
        bulk_load(ring + S::ROWB, X + r * K, S::ROWB, &bars[1]);
        ++issued;
      }
    }
    float u[V];
    load_phase1<K, GELU, true>(reinterpret_cast<const unsigned short *>(ring + s * S::ROWB), lane, u);
    // slot s is refilled with the row NS rounds ahead as soon as every lane has
    // read it (one slot; GELU rows, whose long compute covers the copy), or
    // after the transform (K = 4096 without GELU, measured 2 % faster so)
    constexpr bool kEarly = S::NS == 1 || GELU;
    auto refill = [&]() {
      if (lane == 0) {
        const int64_t rn = row + S::NS * G;
        if (rn < M) {
          fence_proxy_async_smem();
          mbar_arrive_expect_tx(&bars[s], S::ROWB);
          bulk_load(ring + s * S::ROWB, X + rn * K, S::ROWB, &bars[s]);
          ++issued;
        }
      }
    };
    if (kEarly) {
      __syncwarp();
      refill();
    }
    float v[V];
    transform_row<K, ROT>(u, lane, tile, v);  // ends with __syncwarp: slot s is no longer read
    if (!kEarly) refill();
    quantize_store_row<K, ROT, CODE>(v, lane, row, mtab, q, scale);
  }
  // after a timed-out wait, let the copies still in flight land before exiting
  if (lane == 0)
    for (int64_t k = i; k < issued; ++k)
      mbar_wait_drain(&bars[k % S::NS], static_cast<uint32_t>((k / S::NS) & 1), status);
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
    float u[V], v[V];
    load_phase1<K, false, false>(reinterpret_cast<const unsigned short *>(X + row * K), lane, u);
    transform_row<K, true>(u, lane, tiles[warp], v);
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

int num_sms() {
  static ContextCache<int> sms;
  int n = 0;
  if (sms.get(&n, [](int *v) {
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(v, cudaDevAttrMultiProcessorCount, dev);
        return e;
      }) != cudaSuccess || n <= 0)
    return 148;
  return n;
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

template <int K, bool ROT, bool GELU, int CODE>
cudaError_t launch_quant_k(const uint16_t *X, int64_t M, const float *mult, uint8_t *q,
                           float *scale, cudaStream_t st) {
  auto kern = quantize_rows_kernel<K, ROT, GELU, CODE>;
  constexpr int smem = QuantStaging<K>::SMEM;
  constexpr int kRowsPerBlock = kQuantWarps;  // one warp per row
  static ContextCache<int> occupancy;  // per context: attribute set, resident blocks per SM
  int per_sm = 0;
  cudaError_t e = occupancy.get(&per_sm, [&](int *v) {
    cudaError_t r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (r != cudaSuccess) return r;
    int n = 0;
    r = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kQuantWarps * 32, smem);
    *v = n < 1 ? 1 : n;
    return r;
  });
  if (e != cudaSuccess) return e;
  unsigned int *status = nullptr;
  if ((e = status_word(&status)) != cudaSuccess) return e;
  const int64_t need = (M + kRowsPerBlock - 1) / kRowsPerBlock;
  const int64_t g = static_cast<int64_t>(num_sms()) * per_sm;
  const int grid = static_cast<int>(need < g ? need : g);
  // programmatic stream serialization: the block setup may overlap the
  // previous kernel's tail (the kernel waits for it before touching memory)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kQuantWarps * 32, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, X, M, mult, q, scale, status);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

int device_sm_count() { return num_sms(); }

namespace {
template <int K, int CODE>
cudaError_t launch_quant_kc(const uint16_t *X, int64_t M, const float *mult, uint8_t *q,
                            float *scale, bool rot, bool gelu, cudaStream_t st) {
  if (rot) return gelu ? launch_quant_k<K, true, true, CODE>(X, M, mult, q, scale, st)
                       : launch_quant_k<K, true, false, CODE>(X, M, mult, q, scale, st);
  return gelu ? launch_quant_k<K, false, true, CODE>(X, M, mult, q, scale, st)
              : launch_quant_k<K, false, false, CODE>(X, M, mult, q, scale, st);
}
template <int CODE>
cudaError_t launch_quant_c(const uint16_t *X, int64_t M, int K, const float *mult, uint8_t *q,
                           float *scale, bool rot, bool gelu, cudaStream_t st) {
  return K == 1024 ? launch_quant_kc<1024, CODE>(X, M, mult, q, scale, rot, gelu, st)
                   : launch_quant_kc<4096, CODE>(X, M, mult, q, scale, rot, gelu, st);
}
}  // namespace

cudaError_t launch_quantize_rows(const uint16_t *X, int64_t M, int K, const float *mult,
                                 uint8_t *q, float *scale, bool rot, bool gelu, CodeFormat code,
                                 cudaStream_t st) {
  if (M <= 0) return cudaSuccess;
  switch (code) {
    case kCodeBytes4: return launch_quant_c<kCodeBytes4>(X, M, K, mult, q, scale, rot, gelu, st);
    case kCodeBytes8: return launch_quant_c<kCodeBytes8>(X, M, K, mult, q, scale, rot, gelu, st);
    default: return launch_quant_c<kCodePacked4>(X, M, K, mult, q, scale, rot, gelu, st);
  }
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
