// tq.cu -- the 3DTurboQuant vector codec on sm_100a (page "3DTurboQuant:
// Training-Free Near-Optimal Quantization for 3D Reconstruction Models",
// technical summary: section 2.2 the pipeline, section 2.1 the Beta-distributed
// coordinates and their Lloyd-Max codebook, section 4.2 the DUSt3R KV cache at
// d = 1024, b = 4):
//   encode: gamma = ||theta||; y = Pi theta / gamma with Pi = H diag(s) / sqrt(d)
//           (H the natural-order Hadamard matrix, s a caller-given sign
//           vector); code_j = #{k : boundary_k < y_j}; codes two per byte
//           (element 2i in the low nibble); gamma stored as fp32.
//   decode: theta~ = gamma Pi^T c[code] = gamma diag(s) H c[code] / sqrt(d).
// One warp per vector with the register / shared-memory FWHT of fwht.cuh.
// The code decision compares the unnormalised transform (H diag(s) theta)_j
// with boundary_k * gamma * sqrt(d), all in binary32.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "ctxcache.h"
#include "fwht.cuh"
#include "kernels.h"
#include "ptx.cuh"
#include "tq.h"

namespace w4a4 {
namespace {

constexpr int kTqD = 1024;        // vector length
constexpr int kTqLevels = 16;     // 2^b, b = 4
constexpr int kTqWarps = 8;       // warps (vectors in flight) per block
constexpr float kTqSqrtD = 32.0f;

// The code decision by table: a uniform grid over |y| with cells narrower
// than the smallest gap between consecutive boundaries holds at most one
// boundary per cell, so m(|y|) = #{positive boundaries < |y|} = base[cell] +
// (|y| > boundary in the cell).  kTqCells bounds the grid: 1 / width cells
// cover |y| <= 1 (|y| <= 1 for a unit vector).
constexpr int kTqCells = 1024;

struct TqEncodeStaging {
  static constexpr int ROWB = 4 * kTqD;                 // fp32 vector bytes
  static constexpr int NS = 2;                          // vectors in flight per warp
  static constexpr int WARP_BYTES = NS * ROWB + 32 * 32 * 4;
  static constexpr int OFF_SIGN = kTqWarps * WARP_BYTES;  // 32 sign masks
  static constexpr int OFF_BND = OFF_SIGN + 32 * 4;       // 15 boundaries + the cell width
  static constexpr int OFF_CELL = OFF_BND + 64;           // [kTqCells] (base, boundary in cell units)
  static constexpr int OFF_BAR = OFF_CELL + kTqCells * 8;
  static constexpr int SMEM = OFF_BAR + kTqWarps * NS * 8;
};

// Lane-l sign mask: bit j set when s[l + 32 j] < 0 (the phase-1 layout).
__device__ __forceinline__ void load_sign_masks(const float *__restrict__ signs, uint32_t *masks) {
  if (threadIdx.x < 32) {
    uint32_t m = 0;
    for (int j = 0; j < 32; ++j) m |= (__ldg(signs + threadIdx.x + 32 * j) < 0.0f ? 1u : 0u) << j;
    masks[threadIdx.x] = m;
  }
}

// Fills the block's cell table from the 7 positive boundaries p (increasing):
// width w = 0.9 x the smallest gap; entry j describes cell c = max(j - 1, 0)
// (index j = floor(t) + 1 of t = |y| / w, with the index -1 of tiny t folded
// into cell 0): base = #{p_k < c w}, and the boundary inside [c w, (c + 1) w)
// in cell units (t units), or +inf.  Returns 1 / w.
__device__ __forceinline__ float fill_cells(const float *bnd, float2 *cells) {
  const float *p = bnd + 8;
  float gap = p[0];
  for (int k = 1; k < 7; ++k) gap = fminf(gap, p[k] - p[k - 1]);
  const float w = 0.9f * gap;
  for (int j = threadIdx.x; j < kTqCells; j += blockDim.x) {
    const int c = j > 0 ? j - 1 : 0;
    const float lo = c * w, hi = (c + 1) * w;
    int base = 0;
    float inside = __int_as_float(0x7F800000);  // +inf
    for (int k = 0; k < 7; ++k) {
      if (p[k] < lo) ++base;
      else if (p[k] < hi) inside = p[k] / w;
    }
    cells[j] = make_float2(__int_as_float(base), inside);
  }
  return 1.0f / w;
}

__global__ void __launch_bounds__(kTqWarps * 32)
    tq_encode_kernel(const float *__restrict__ X, int64_t n, const float *__restrict__ signs,
                     const float *__restrict__ boundaries, uint8_t *__restrict__ codes,
                     float *__restrict__ norms, unsigned int *__restrict__ status) {
  using S = TqEncodeStaging;
  constexpr int V = 32;
  extern __shared__ __align__(1024) uint8_t tsmem[];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  uint8_t *ring = tsmem + warp * S::WARP_BYTES;
  float *tile = reinterpret_cast<float *>(ring + S::NS * S::ROWB);
  uint32_t *masks = reinterpret_cast<uint32_t *>(tsmem + S::OFF_SIGN);
  float *bnd = reinterpret_cast<float *>(tsmem + S::OFF_BND);
  float2 *cells = reinterpret_cast<float2 *>(tsmem + S::OFF_CELL);
  uint64_t *bars = reinterpret_cast<uint64_t *>(tsmem + S::OFF_BAR) + warp * S::NS;
  const int64_t G = static_cast<int64_t>(gridDim.x) * kTqWarps;
  const int64_t r0 = static_cast<int64_t>(warp) * gridDim.x + blockIdx.x;
  int64_t issued = 0;
  if (lane == 0) {
    for (int s = 0; s < S::NS; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  griddep_launch_dependents();
  griddep_wait();
  if (lane == 0) {
    fence_proxy_async_smem();
    for (int s = 0; s < S::NS; ++s) {
      const int64_t r = r0 + s * G;
      if (r < n) {
        mbar_arrive_expect_tx(&bars[s], S::ROWB);
        bulk_load(ring + s * S::ROWB, X + r * kTqD, S::ROWB, &bars[s]);
        ++issued;
      }
    }
  }
  load_sign_masks(signs, masks);
  if (threadIdx.x < kTqLevels - 1) bnd[threadIdx.x] = __ldg(boundaries + threadIdx.x);
  __syncthreads();
  // (the codebook is odd-symmetric: boundary 7 is 0, boundaries 8..14 positive)
  const float inv_w = fill_cells(bnd, cells);
  __syncthreads();
  const uint32_t smask = masks[lane];
  int64_t i = 0;
  for (int64_t row = r0; row < n; row += G, ++i) {
    const int s = static_cast<int>(i % S::NS);
    if (!mbar_wait_drain(&bars[s], static_cast<uint32_t>((i / S::NS) & 1), status)) break;
    const float *x = reinterpret_cast<const float *>(ring + s * S::ROWB);
    float u[V], v[V];
    float ss[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int j = 0; j < V; ++j) {
      const float xv = x[lane + 32 * j];
      u[j] = __uint_as_float(__float_as_uint(xv) ^ (((smask >> j) & 1u) << 31));  // diag(s) theta
      ss[j & 3] = fmaf(xv, xv, ss[j & 3]);
    }
    __syncwarp();  // every lane has read slot s: the vector after next may land there
    if (lane == 0) {
      const int64_t rn = row + S::NS * G;
      if (rn < n) {
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&bars[s], S::ROWB);
        bulk_load(ring + s * S::ROWB, X + rn * kTqD, S::ROWB, &bars[s]);
        ++issued;
      }
    }
    transform_row<kTqD, true>(u, lane, tile, v);  // H diag(s) theta
    float sum = (ss[0] + ss[1]) + (ss[2] + ss[3]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float gamma = sqrtf(sum);
    if (lane == 0) norms[row] = gamma;
    // |y_j| = |(H diag(s) theta)_j| / (gamma sqrt(d)), in cell units t = |y_j| / w
    const float g = gamma * kTqSqrtD;
    const float tscale = g > 0.0f ? inv_w / g : 0.0f;
    // codes of elements 32 lane + r: 8 per 32-bit word, element 2i in the low nibble
    uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int r = 0; r < V; ++r) {
      const float t = fabsf(v[r]) * tscale;
      // 2^23 - 0.5 + t rounds to 2^23 + floor(t) (or one less at an exact
      // integer, where the cell below gives the same count); entry = that + 1,
      // clamped (unsigned) into the table for any input
      const uint32_t j = min(static_cast<uint32_t>(__float_as_int(t + 8388607.5f) - 0x4AFFFFFF),
                             static_cast<uint32_t>(kTqCells - 1));
      const float2 cell = cells[j];
      const int m = __float_as_int(cell.x) + (t > cell.y ? 1 : 0);
      const int code = v[r] > 0.0f ? 8 + m : 7 - m;  // odd symmetry around boundary 7 = 0
      w[r >> 3] |= static_cast<uint32_t>(code) << (4 * (r & 7));
    }
    *reinterpret_cast<uint4 *>(codes + row * (kTqD / 2) + lane * 16) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  if (lane == 0)
    for (int64_t k = i; k < issued; ++k)
      mbar_wait_drain(&bars[k % S::NS], static_cast<uint32_t>((k / S::NS) & 1), status);
}

// decode: one warp per vector; codes are read straight from global memory
// (16 bytes per lane = the lane's 32 consecutive elements: the phase-2 layout)
__global__ void __launch_bounds__(kTqWarps * 32)
    tq_decode_kernel(const uint8_t *__restrict__ codes, const float *__restrict__ norms, int64_t n,
                     const float *__restrict__ signs, const float *__restrict__ centroids,
                     float *__restrict__ Y) {
  __shared__ float tiles[kTqWarps][32 * 32];
  __shared__ float2 pair_tab[256];  // byte -> (c[low nibble], c[high nibble])
  __shared__ uint32_t masks[32];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  griddep_launch_dependents();
  griddep_wait();
  {
    const int t = threadIdx.x;  // 256 threads: one table entry each
    pair_tab[t] = make_float2(__ldg(centroids + (t & 15)), __ldg(centroids + (t >> 4)));
  }
  load_sign_masks(signs, masks);
  __syncthreads();
  const uint32_t smask = masks[lane];
  const int64_t G = static_cast<int64_t>(gridDim.x) * kTqWarps;
  const int64_t r0 = static_cast<int64_t>(warp) * gridDim.x + blockIdx.x;
  // the next vector's codes and norm are loaded while this one is transformed
  uint4 cw_next = make_uint4(0u, 0u, 0u, 0u);
  float gamma_next = 0.0f;
  if (r0 < n) {
    cw_next = __ldcs(reinterpret_cast<const uint4 *>(codes + r0 * (kTqD / 2)) + lane);
    gamma_next = __ldg(norms + r0);
  }
  for (int64_t row = r0; row < n; row += G) {
    const uint4 cw = cw_next;
    const float gamma = gamma_next;
    if (row + G < n) {
      cw_next = __ldcs(reinterpret_cast<const uint4 *>(codes + (row + G) * (kTqD / 2)) + lane);
      gamma_next = __ldg(norms + row + G);
    }
    const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
    float v[32], u[32];
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int by = 0; by < 4; ++by) {
        const float2 c2 = pair_tab[(words[q] >> (8 * by)) & 0xFFu];
        v[8 * q + 2 * by] = c2.x;
        v[8 * q + 2 * by + 1] = c2.y;
      }
    transform_row<kTqD, true>(v, lane, tiles[warp], u);  // H c[code], back in phase-1 layout
    const float scl = gamma * (1.0f / kTqSqrtD);
    float *y = Y + row * kTqD;
#pragma unroll
    for (int j = 0; j < 32; ++j)
      __stcs(y + lane + 32 * j,
             __uint_as_float(__float_as_uint(u[j] * scl) ^ (((smask >> j) & 1u) << 31)));
  }
}

template <typename Kern>
int blocks_per_sm(Kern kern, int smem) {
  int n = 0;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kTqWarps * 32, smem);
  return n < 1 ? 1 : n;
}

cudaError_t launch_pdl(void (*kern)(const float *, int64_t, const float *, const float *, uint8_t *,
                                    float *, unsigned int *),
                       int grid, int smem, cudaStream_t st, const float *X, int64_t n,
                       const float *signs, const float *bnd, uint8_t *codes, float *norms) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kTqWarps * 32, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  unsigned int *status = nullptr;
  const cudaError_t e = status_word(&status);
  if (e != cudaSuccess) return e;
  return cudaLaunchKernelEx(&cfg, kern, X, n, signs, bnd, codes, norms, status);
}

// ---------------------------------------------------------------- codebook
// Lloyd-Max quantizer of the coordinate density of a uniformly random unit
// vector in R^d, f(x) = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)) (1 - x^2)^((d-3)/2):
// the density is even, so the positive half is solved (boundary 0 in the
// middle) by the fixed-point iteration boundaries = midpoints, centroids =
// conditional means; integrals by composite Simpson's rule.
double coord_pdf(double x, int d, double lognorm) {
  const double a = 1.0 - x * x;
  return a > 0.0 ? std::exp(lognorm + 0.5 * (d - 3) * std::log(a)) : 0.0;
}

void cell_moments(double lo, double hi, int d, double lognorm, double *m0, double *m1) {
  constexpr int kIntervals = 512;  // even
  const double h = (hi - lo) / kIntervals;
  double s0 = 0.0, s1 = 0.0;
  for (int i = 0; i <= kIntervals; ++i) {
    const double x = lo + h * i;
    const double w = (i == 0 || i == kIntervals) ? 1.0 : ((i & 1) ? 4.0 : 2.0);
    const double f = coord_pdf(x, d, lognorm);
    s0 += w * f;
    s1 += w * x * f;
  }
  *m0 = s0 * h / 3.0;
  *m1 = s1 * h / 3.0;
}

void lloyd_max_half(int d, int half, double *c) {
  const double lognorm = std::lgamma(0.5 * d) - 0.5 * std::log(M_PI) - std::lgamma(0.5 * (d - 1));
  const double R = std::fmin(1.0, 12.0 / std::sqrt(static_cast<double>(d)));
  for (int k = 0; k < half; ++k) c[k] = R * (k + 0.5) / (2.0 * half);  // a spread-out start
  double edges[kTqLevels / 2 + 1];
  for (int it = 0; it < 20000; ++it) {
    edges[0] = 0.0;
    for (int k = 1; k < half; ++k) edges[k] = 0.5 * (c[k - 1] + c[k]);
    edges[half] = R;
    double change = 0.0;
    for (int k = 0; k < half; ++k) {
      double m0, m1;
      cell_moments(edges[k], edges[k + 1], d, lognorm, &m0, &m1);
      const double nc = m1 / m0;
      change = std::fmax(change, std::fabs(nc - c[k]));
      c[k] = nc;
    }
    if (change < 1e-17) break;
  }
}

}  // namespace
}  // namespace w4a4

extern "C" {

w4a4_status tq_codebook(int32_t d, int32_t b, float *centroids, float *boundaries) {
  if (d != w4a4::kTqD || b != 4) return W4A4_ERR_UNSUPPORTED;
  if (!centroids || !boundaries) return W4A4_ERR_ARG;
  constexpr int half = w4a4::kTqLevels / 2;
  double c[half];
  w4a4::lloyd_max_half(d, half, c);
  for (int k = 0; k < half; ++k) {
    centroids[half + k] = static_cast<float>(c[k]);
    centroids[half - 1 - k] = static_cast<float>(-c[k]);
  }
  boundaries[half - 1] = 0.0f;
  for (int k = 1; k < half; ++k) {
    const double t = 0.5 * (c[k - 1] + c[k]);
    boundaries[half - 1 + k] = static_cast<float>(t);
    boundaries[half - 1 - k] = static_cast<float>(-t);
  }
  return W4A4_OK;
}

static bool tq_aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

w4a4_status tq_encode(const float *X, int64_t n, int32_t d, const float *signs,
                      const float *boundaries, uint8_t *codes, float *norms, void *stream) {
  if (d != w4a4::kTqD) return W4A4_ERR_UNSUPPORTED;
  if (n < 0 || n >= (int64_t(1) << 31)) return W4A4_ERR_SHAPE;
  if (n == 0) return W4A4_OK;
  if (!X || !signs || !boundaries || !codes || !norms) return W4A4_ERR_ARG;
  if (!tq_aligned16(X) || !tq_aligned16(codes) || !tq_aligned16(signs) || !tq_aligned16(norms) ||
      !tq_aligned16(boundaries))
    return W4A4_ERR_ALIGN;
  using S = w4a4::TqEncodeStaging;
  static w4a4::ContextCache<int> occupancy;  // per context: attribute set, blocks per SM
  int per_sm = 0;
  if (occupancy.get(&per_sm, [](int *v) {
        const cudaError_t r = cudaFuncSetAttribute(
            w4a4::tq_encode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM);
        if (r == cudaSuccess) *v = w4a4::blocks_per_sm(w4a4::tq_encode_kernel, S::SMEM);
        return r;
      }) != cudaSuccess)
    return W4A4_ERR_CUDA;
  const int64_t need = (n + w4a4::kTqWarps - 1) / w4a4::kTqWarps;
  const int64_t g = static_cast<int64_t>(w4a4::device_sm_count()) * per_sm;
  const int grid = static_cast<int>(need < g ? need : g);
  cudaError_t e = w4a4::launch_pdl(w4a4::tq_encode_kernel, grid, S::SMEM,
                                   static_cast<cudaStream_t>(stream), X, n, signs, boundaries, codes,
                                   norms);
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? W4A4_OK : W4A4_ERR_CUDA;
}

w4a4_status tq_decode(const uint8_t *codes, const float *norms, int64_t n, int32_t d,
                      const float *signs, const float *centroids, float *Y, void *stream) {
  if (d != w4a4::kTqD) return W4A4_ERR_UNSUPPORTED;
  if (n < 0 || n >= (int64_t(1) << 31)) return W4A4_ERR_SHAPE;
  if (n == 0) return W4A4_OK;
  if (!codes || !norms || !signs || !centroids || !Y) return W4A4_ERR_ARG;
  if (!tq_aligned16(codes) || !tq_aligned16(Y) || !tq_aligned16(signs) || !tq_aligned16(norms) ||
      !tq_aligned16(centroids))
    return W4A4_ERR_ALIGN;
  static w4a4::ContextCache<int> occupancy;  // per context: blocks per SM
  int per_sm = 0;
  if (occupancy.get(&per_sm, [](int *v) {
        *v = w4a4::blocks_per_sm(w4a4::tq_decode_kernel, 0);
        return cudaSuccess;
      }) != cudaSuccess)
    return W4A4_ERR_CUDA;
  const int64_t need = (n + w4a4::kTqWarps - 1) / w4a4::kTqWarps;
  const int64_t g = static_cast<int64_t>(w4a4::device_sm_count()) * per_sm;
  const int grid = static_cast<int>(need < g ? need : g);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(w4a4::kTqWarps * 32, 1, 1);
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, w4a4::tq_decode_kernel, codes, norms, n, signs, centroids, Y);
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? W4A4_OK : W4A4_ERR_CUDA;
}

}  // extern "C"
