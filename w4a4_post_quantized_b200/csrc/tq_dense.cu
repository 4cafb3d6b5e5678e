// tq_dense.cu -- the 3DTurboQuant vector codec with the page's dense random
// rotation (page "3DTurboQuant: Training-Free Near-Optimal Quantization for 3D
// Reconstruction Models", technical summary: section 2.2 the pipeline -- norm,
// rotation by a random orthogonal matrix Pi obtained by QR of a Gaussian
// matrix, per-coordinate Lloyd-Max codes, reconstruction gamma Pi^T c --,
// section 2.1 the codebook, section 4.2 the DUSt3R KV cache at d = 1024,
// b = 4).
//
//   encode: gamma = ||x||, code_j = #{k : t_k < (Pi x)_j / gamma}
//   decode: x~ = gamma Pi^T c[code]
//
// Pi is dense, so both are matrix products on the tensor cores, in tf32 with
// the usual three-term split for fp32-level accuracy: every operand value v
// is hi + lo with hi = v with its low 13 mantissa bits cleared and lo =
// tf32-round(v - hi) (relative error 2^-22), and
//     A B ~ A_hi B_hi + A_hi B_lo + A_lo B_hi
// (the dropped A_lo B_lo term is below 2^-20 relative).  The matrix's hi and
// lo parts are prepared once on the host (tq_rotation_qr); the vectors' parts
// are formed in the kernel.
//
//   encode: D[m][j] = sum_k X[m][k] Pi[j][k]: A = X (TMA-loaded fp32 tile,
//           split in shared memory by four warps, which also sum x^2 for the
//           norm), B = Pi (rows j, K-major); the epilogue compares
//           D[m][j] with t_k gamma_m (the same decision as y_j against t_k,
//           gamma > 0), so no division, and packs the codes.
//   decode: D[m][j] = sum_k C[m][k] Pi[k][j] with C = centroids[codes]: A is
//           expanded from the 4-bit codes straight into the hi / lo operand
//           tiles (a 16-entry table), B = Pi^T (rows j, K-major); the
//           epilogue scales by gamma_m.
//
// Tiles 128 x 256 (256 tensor-memory columns, double-buffered), k-blocks of
// 32 values (128-byte swizzled rows), two stages; one persistent CTA of 384
// threads per SM:
//   warp 0      TMA producer          warp 1      MMA issuer (one thread)
//   warp 2      tensor-memory alloc   warps 4..7  split (encode) / expand (decode)
//   warps 8..11 epilogue (one row per thread)
// Every wait is bounded (ptx.cuh).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#include "ctxcache.h"
#include "kernels.h"
#include "ptx.cuh"
#include "tq.h"

namespace w4a4 {
namespace {

constexpr int kD = 1024;           // vector length
constexpr int BM = 128, BN = 256, BK = 32;
constexpr int NKB = kD / BK;       // k-blocks per tile
constexpr int NNT = kD / BN;       // column tiles
constexpr int kThreads = 384;
constexpr int W_TMA = 0, W_MMA = 1, W_ALLOC = 2, W_PREP0 = 4, W_EPI0 = 8;

template <bool ENC>
struct DensePlan {
  static constexpr int A_TILE = BM * BK * 4;       // 16 KB
  static constexpr int B_TILE = BN * BK * 4;       // 32 KB
  static constexpr int OFF_RAW = 0;                // encode: the TMA-loaded fp32 X tile
  static constexpr int OFF_AHI = ENC ? A_TILE : 0;
  static constexpr int OFF_ALO = OFF_AHI + A_TILE;
  static constexpr int OFF_BHI = OFF_ALO + A_TILE;
  static constexpr int OFF_BLO = OFF_BHI + B_TILE;
  static constexpr int STAGE = OFF_BLO + B_TILE;   // 112 KB (encode) / 96 KB (decode)
  static constexpr int STAGES = 2;
  static constexpr int OFF_GAM = STAGES * STAGE;   // [2][BM] row norms (encode)
  static constexpr int OFF_TAB = OFF_GAM + 2 * BM * 4;   // 16 float2 (hi, lo) centroids (decode)
  static constexpr int OFF_BAR = OFF_TAB + 16 * 8;
  static constexpr int NUM_BARS = 3 * STAGES + 2 * 2 + 2 * 2 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;
  static_assert(SMEM <= 232448, "shared-memory budget");
  static_assert(STAGE % 1024 == 0, "swizzled tiles need 1024-byte alignment");
  static constexpr uint32_t TX_BYTES = (ENC ? A_TILE : 0) + 2 * B_TILE;
};

// kind::tf32, fp32 D, both K-major, M = 128, N = 256
constexpr uint32_t kIdesc = (1u << 4) | (2u << 7) | (2u << 10) | ((BN >> 3) << 17) | ((BM >> 4) << 24);

__device__ __forceinline__ uint32_t tf32_rna_bits(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}

template <bool ENC>
__global__ void __launch_bounds__(kThreads, 1)
    tq_dense_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmBhi,
                    const __grid_constant__ CUtensorMap tmBlo, const uint8_t *__restrict__ codes_in,
                    const float *__restrict__ norms_in, const float *__restrict__ table,
                    uint8_t *__restrict__ codes_out, float *__restrict__ norms_out,
                    float *__restrict__ Y, int n, unsigned int *__restrict__ status) {
  using P = DensePlan<ENC>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + P::OFF_BAR);
  uint64_t *b_full = bars;                     // the stage's TMA bytes landed
  uint64_t *a_full = b_full + P::STAGES;       // its A hi / lo tiles written (4 warps)
  uint64_t *s_free = a_full + P::STAGES;       // its MMAs completed
  uint64_t *acc_full = s_free + P::STAGES;
  uint64_t *acc_empty = acc_full + 2;          // 4 epilogue warps
  uint64_t *gam_full = acc_empty + 2;          // encode: a tile's row norms written (4 warps)
  uint64_t *gam_free = gam_full + 2;           // encode: read by the epilogue (4 warps)
  uint64_t *mma_done = gam_free + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + P::OFF_MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + P::OFF_MISC + 4);
  float *gam = reinterpret_cast<float *>(smem + P::OFF_GAM);
  float2 *ctab = reinterpret_cast<float2 *>(smem + P::OFF_TAB);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_m = (n + BM - 1) / BM;
  const int num_tiles = num_m * NNT;

  if (threadIdx.x == 0) {
    for (int s = 0; s < P::STAGES; ++s) {
      mbar_init(&b_full[s], 1);
      mbar_init(&a_full[s], 4);
      mbar_init(&s_free[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
      mbar_init(&gam_full[b], 4);
      mbar_init(&gam_free[b], 4);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == W_TMA && lane == 0) {
    if (ENC) tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmBhi);
    tma_prefetch_desc(&tmBlo);
  }
  if (warp == W_ALLOC) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_launch_dependents();
  griddep_wait();
  if (!ENC && threadIdx.x < 16) {
    // centroid c as hi + lo tf32 terms
    const float c = __ldg(table + threadIdx.x);
    const uint32_t hi = __float_as_uint(c) & 0xFFFFE000u;
    ctab[threadIdx.x] = make_float2(__uint_as_float(hi), __uint_as_float(tf32_rna_bits(c - __uint_as_float(hi))));
  }
  __syncthreads();

  if (warp == W_TMA) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int mb = tile / NNT, nb = tile % NNT;
        for (int kb = 0; kb < NKB; ++kb, ++it) {
          const uint32_t s = it % P::STAGES;
          if (!mbar_wait(&s_free[s], ((it / P::STAGES) & 1u) ^ 1u, abort_flag, status)) {
            ok = false;
            break;
          }
          uint8_t *st = smem + s * P::STAGE;
          mbar_arrive_expect_tx(&b_full[s], P::TX_BYTES);
          if (ENC) tma_load_2d(st + P::OFF_RAW, &tmA, kb * BK, mb * BM, &b_full[s]);
          tma_load_2d(st + P::OFF_BHI, &tmBhi, kb * BK, nb * BN, &b_full[s]);
          tma_load_2d(st + P::OFF_BLO, &tmBlo, kb * BK, nb * BN, &b_full[s]);
        }
      }
      for (uint32_t u = (it > P::STAGES ? it - P::STAGES : 0); u < it; ++u)
        mbar_wait_drain(&b_full[u % P::STAGES], (u / P::STAGES) & 1u, status);
    }
  } else if (warp == W_MMA) {
    if (lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      uint32_t it = 0, t = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++t) {
        const uint32_t b = t & 1u;
        if (!mbar_wait(&acc_empty[b], ((t >> 1) & 1u) ^ 1u, abort_flag, status)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + b * BN;
        for (int kb = 0; kb < NKB; ++kb, ++it) {
          const uint32_t s = it % P::STAGES, ph = (it / P::STAGES) & 1u;
          if (!mbar_wait(&b_full[s], ph, abort_flag, status) || !mbar_wait(&a_full[s], ph, abort_flag, status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = smem_u32(smem + s * P::STAGE);
#pragma unroll
          for (int term = 0; term < 3; ++term) {
            // hi x hi, hi x lo, lo x hi
            const uint32_t a = st + (term == 2 ? P::OFF_ALO : P::OFF_AHI);
            const uint32_t bb = st + (term == 1 ? P::OFF_BLO : P::OFF_BHI);
#pragma unroll
            for (int j = 0; j < BK / 8; ++j)
              mma_tf32(d, umma_desc(a + 32 * j, 16, 1024, kLayoutSw128),
                       umma_desc(bb + 32 * j, 16, 1024, kLayoutSw128), kIdesc,
                       (kb | term | j) != 0 ? 1u : 0u);
          }
          tc_commit(&s_free[s]);
        }
        if (ok) tc_commit(&acc_full[b]);
      }
      tc_commit(mma_done);
      mbar_wait_drain(mma_done, 0, status);
    }
  } else if (warp >= W_PREP0 && warp < W_PREP0 + 4) {
    // ------------------------------------------- split (encode) / expand (decode)
    const int r = (warp - W_PREP0) * 32 + lane;   // tile row
    uint32_t it = 0, t = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++t) {
      const int mb = tile / NNT;
      const int64_t row = static_cast<int64_t>(mb) * BM + r;
      float ss = 0.0f;
      for (int kb = 0; kb < NKB; ++kb, ++it) {
        const uint32_t s = it % P::STAGES;
        if (!mbar_wait(&b_full[s], (it / P::STAGES) & 1u, abort_flag, status)) {
          ok = false;
          break;
        }
        uint8_t *st = smem + s * P::STAGE;
        // row r: 128 bytes, 16-byte chunk c at c ^ (r % 8)
        if constexpr (ENC) {
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint32_t off = r * 128 + ((c ^ (r & 7)) << 4);
            const float4 x = *reinterpret_cast<const float4 *>(st + P::OFF_RAW + off);
            const float xs[4] = {x.x, x.y, x.z, x.w};
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              ss = fmaf(xs[e], xs[e], ss);
              hi[e] = __float_as_uint(xs[e]) & 0xFFFFE000u;
              lo[e] = tf32_rna_bits(xs[e] - __uint_as_float(hi[e]));
            }
            *reinterpret_cast<uint4 *>(st + P::OFF_AHI + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            *reinterpret_cast<uint4 *>(st + P::OFF_ALO + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
          }
        } else {
          // the row's 32 codes of this k-block: 16 bytes (element 2i in the low nibble)
          uint4 w = make_uint4(0u, 0u, 0u, 0u);
          if (row < n) w = __ldg(reinterpret_cast<const uint4 *>(codes_in + row * (kD / 2) + kb * (BK / 2)));
          const uint32_t words[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint32_t off = r * 128 + ((c ^ (r & 7)) << 4);
            float hi[4], lo[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int k = 4 * c + e;   // code of element kb * 32 + k
              const float2 h = row < n ? ctab[(words[k >> 3] >> (4 * (k & 7))) & 15u] : make_float2(0.0f, 0.0f);
              hi[e] = h.x;
              lo[e] = h.y;
            }
            *reinterpret_cast<float4 *>(st + P::OFF_AHI + off) = make_float4(hi[0], hi[1], hi[2], hi[3]);
            *reinterpret_cast<float4 *>(st + P::OFF_ALO + off) = make_float4(lo[0], lo[1], lo[2], lo[3]);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&a_full[s]);
      }
      if (ENC && ok) {
        const uint32_t b = t & 1u;
        if (!mbar_wait(&gam_free[b], ((t >> 1) & 1u) ^ 1u, abort_flag, status)) break;
        gam[b * BM + r] = sqrtf(ss);
        __syncwarp();
        if (lane == 0) mbar_arrive(&gam_full[b]);
      }
    }
  } else if (warp >= W_EPI0) {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const uint32_t tq = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    float bnd[15];
    if (ENC)
#pragma unroll
      for (int k = 0; k < 15; ++k) bnd[k] = __ldg(table + k);
    uint32_t t = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++t) {
      const int mb = tile / NNT, nb = tile % NNT;
      const int64_t row = static_cast<int64_t>(mb) * BM + r;
      const uint32_t b = t & 1u;
      float g;
      if constexpr (ENC) {
        if (!mbar_wait(&gam_full[b], (t >> 1) & 1u, abort_flag, status)) break;
        g = gam[b * BM + r];
        __syncwarp();
        if (lane == 0) mbar_arrive(&gam_free[b]);
        if (nb == 0 && row < n) norms_out[row] = g;
      } else {
        g = row < n ? __ldg(norms_in + row) : 0.0f;
      }
      if (!mbar_wait(&acc_full[b], (t >> 1) & 1u, abort_flag, status)) break;
      tc_fence_after();
      // encode: t_k < D / g  <=>  t_k g < D  (g > 0); g = 0 means y = 0
      float thr[15];
      if constexpr (ENC) {
#pragma unroll
        for (int k = 0; k < 15; ++k) thr[k] = bnd[k] * g;
      }
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tq + b * BN + 32 * c, v);
        tmem_wait_ld();
        if (c == BN / 32 - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[b]);
        }
        if (row >= n) continue;
        const int j0 = nb * BN + 32 * c;
        if constexpr (ENC) {
          uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float y = __uint_as_float(v[e]);
            int code = 0;
            if (g > 0.0f) {
#pragma unroll
              for (int k = 0; k < 15; ++k) code += thr[k] < y ? 1 : 0;
            } else {
              code = 7;   // y = 0: the boundaries below 0
            }
            w[e >> 3] |= static_cast<uint32_t>(code) << (4 * (e & 7));
          }
          *reinterpret_cast<uint4 *>(codes_out + row * (kD / 2) + j0 / 2) = make_uint4(w[0], w[1], w[2], w[3]);
        } else {
          float4 *dst = reinterpret_cast<float4 *>(Y + row * kD + j0);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            __stcs(dst + e, make_float4(__uint_as_float(v[4 * e]) * g, __uint_as_float(v[4 * e + 1]) * g,
                                        __uint_as_float(v[4 * e + 2]) * g, __uint_as_float(v[4 * e + 3]) * g));
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == W_ALLOC) tmem_dealloc(tmem_base, 512);
}

template <bool ENC>
cudaError_t launch_dense(const float *A, const float *Bhi, const float *Blo, const uint8_t *codes_in,
                         const float *norms_in, const float *table, uint8_t *codes_out, float *norms_out,
                         float *Y, int64_t n, cudaStream_t st) {
  using P = DensePlan<ENC>;
  auto kern = tq_dense_kernel<ENC>;
  static ContextCache<bool> attr;
  bool done = false;
  cudaError_t e = attr.get(&done, [&](bool *v) {
    *v = true;
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, P::SMEM);
  });
  if (e != cudaSuccess) return e;
  unsigned int *status = nullptr;
  if ((e = status_word(&status)) != cudaSuccess) return e;
  CUtensorMap ta = {}, tbh, tbl;
  if (ENC && !encode_tensor_map_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, A, kD, static_cast<uint64_t>(n),
                                   kD * 4, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (!encode_tensor_map_2d(&tbh, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, Bhi, kD, kD, kD * 4, BK, BN,
                            CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tensor_map_2d(&tbl, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, Blo, kD, kD, kD * 4, BK, BN,
                            CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const int tiles = static_cast<int>((n + BM - 1) / BM) * NNT;
  const int sms = device_sm_count();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(tiles < sms ? tiles : sms, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = P::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, ta, tbh, tbl, codes_in, norms_in, table, codes_out, norms_out, Y,
                         static_cast<int>(n), status);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Householder QR of the d x d matrix G (row-major, double), sign-fixed so that
// R has a positive diagonal; Pi = Q diag(sign(diag R)) into pi[i * d + j].
// Column k of G is processed as row k of the transpose, so every update is a
// contiguous dot product and axpy.
void householder_rotation(const double *G, int d, std::vector<double> &pi) {
  std::vector<double> at(static_cast<size_t>(d) * d);           // at[j][i] = G[i][j]
  for (int i = 0; i < d; ++i)
    for (int j = 0; j < d; ++j) at[static_cast<size_t>(j) * d + i] = G[static_cast<size_t>(i) * d + j];
  std::vector<double> vs(static_cast<size_t>(d) * d, 0.0);      // reflector k in row k, entries k..d-1
  std::vector<double> diag(d);
  for (int k = 0; k < d; ++k) {
    double *col = &at[static_cast<size_t>(k) * d];
    double nrm = 0.0;
    for (int i = k; i < d; ++i) nrm += col[i] * col[i];
    nrm = std::sqrt(nrm);
    double *v = &vs[static_cast<size_t>(k) * d];
    const double alpha = col[k] >= 0.0 ? -nrm : nrm;   // R[k][k] after the reflection
    diag[k] = alpha;
    for (int i = k; i < d; ++i) v[i] = col[i];
    v[k] -= alpha;
    double vn = 0.0;
    for (int i = k; i < d; ++i) vn += v[i] * v[i];
    vn = std::sqrt(vn);
    if (vn > 0.0)
      for (int i = k; i < d; ++i) v[i] /= vn;
    // apply I - 2 v v^T to the remaining columns j > k
    for (int j = k + 1; j < d; ++j) {
      double *cj = &at[static_cast<size_t>(j) * d];
      double dot = 0.0;
      for (int i = k; i < d; ++i) dot += v[i] * cj[i];
      dot *= 2.0;
      for (int i = k; i < d; ++i) cj[i] -= dot * v[i];
    }
  }
  // Q = H_0 H_1 ... H_{d-1}: column j of Q is H_0 ( ... (H_{d-1} e_j))
  pi.assign(static_cast<size_t>(d) * d, 0.0);
  std::vector<double> q(d);
  for (int j = 0; j < d; ++j) {
    std::fill(q.begin(), q.end(), 0.0);
    q[j] = 1.0;
    for (int k = d - 1; k >= 0; --k) {
      const double *v = &vs[static_cast<size_t>(k) * d];
      double dot = 0.0;
      for (int i = k; i < d; ++i) dot += v[i] * q[i];
      dot *= 2.0;
      for (int i = k; i < d; ++i) q[i] -= dot * v[i];
    }
    const double sgn = diag[j] < 0.0 ? -1.0 : 1.0;   // the sign that makes R[j][j] positive
    for (int i = 0; i < d; ++i) pi[static_cast<size_t>(i) * d + j] = q[i] * sgn;
  }
}

void split_tf32(double v, float *hi, float *lo) {
  const float f = static_cast<float>(v);
  uint32_t b;
  std::memcpy(&b, &f, 4);
  b &= 0xFFFFE000u;
  float h;
  std::memcpy(&h, &b, 4);
  // round the remainder to nearest tf32 (ties away from zero, as cvt.rna)
  const float r = static_cast<float>(v - static_cast<double>(h));
  uint32_t rb;
  std::memcpy(&rb, &r, 4);
  rb = (rb + 0x1000u) & 0xFFFFE000u;
  float l;
  std::memcpy(&l, &rb, 4);
  *hi = h;
  *lo = l;
}

}  // namespace
}  // namespace w4a4

extern "C" {

w4a4_status tq_rotation_qr(const double *G, int32_t d, float *pi_hi, float *pi_lo, float *pit_hi,
                           float *pit_lo) {
  if (d != w4a4::kD) return W4A4_ERR_UNSUPPORTED;
  if (!G || !pi_hi || !pi_lo || !pit_hi || !pit_lo) return W4A4_ERR_ARG;
  std::vector<double> pi;
  w4a4::householder_rotation(G, d, pi);
  for (int i = 0; i < d; ++i)
    for (int j = 0; j < d; ++j) {
      const double v = pi[static_cast<size_t>(i) * d + j];
      w4a4::split_tf32(v, &pi_hi[static_cast<size_t>(i) * d + j], &pi_lo[static_cast<size_t>(i) * d + j]);
      w4a4::split_tf32(v, &pit_hi[static_cast<size_t>(j) * d + i], &pit_lo[static_cast<size_t>(j) * d + i]);
    }
  return W4A4_OK;
}

static bool tqd_aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

w4a4_status tq_encode_dense(const float *X, int64_t n, int32_t d, const float *pi_hi, const float *pi_lo,
                            const float *boundaries, uint8_t *codes, float *norms, void *stream) {
  if (d != w4a4::kD) return W4A4_ERR_UNSUPPORTED;
  if (n < 0 || n >= (int64_t(1) << 31)) return W4A4_ERR_SHAPE;
  if (n == 0) return W4A4_OK;
  if (!X || !pi_hi || !pi_lo || !boundaries || !codes || !norms) return W4A4_ERR_ARG;
  if (!tqd_aligned16(X) || !tqd_aligned16(pi_hi) || !tqd_aligned16(pi_lo) || !tqd_aligned16(codes) ||
      !tqd_aligned16(norms) || !tqd_aligned16(boundaries))
    return W4A4_ERR_ALIGN;
  const cudaError_t e = w4a4::launch_dense<true>(X, pi_hi, pi_lo, nullptr, nullptr, boundaries, codes, norms,
                                                 nullptr, n, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? W4A4_OK : W4A4_ERR_CUDA;
}

w4a4_status tq_decode_dense(const uint8_t *codes, const float *norms, int64_t n, int32_t d,
                            const float *pit_hi, const float *pit_lo, const float *centroids, float *Y,
                            void *stream) {
  if (d != w4a4::kD) return W4A4_ERR_UNSUPPORTED;
  if (n < 0 || n >= (int64_t(1) << 31)) return W4A4_ERR_SHAPE;
  if (n == 0) return W4A4_OK;
  if (!codes || !norms || !pit_hi || !pit_lo || !centroids || !Y) return W4A4_ERR_ARG;
  if (!tqd_aligned16(codes) || !tqd_aligned16(norms) || !tqd_aligned16(pit_hi) || !tqd_aligned16(pit_lo) ||
      !tqd_aligned16(centroids) || !tqd_aligned16(Y))
    return W4A4_ERR_ALIGN;
  const cudaError_t e = w4a4::launch_dense<false>(nullptr, pit_hi, pit_lo, codes, norms, centroids, nullptr,
                                                  nullptr, Y, n, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? W4A4_OK : W4A4_ERR_CUDA;
}

}  // extern "C"
