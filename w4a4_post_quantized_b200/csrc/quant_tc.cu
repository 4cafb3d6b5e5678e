// quant_tc.cu -- the DSFQ activation quantizer with the Hadamard rotation on
// the tensor cores (sm_100a tcgen05).
//
// What it computes is the rotate -> smooth -> per-token int4 step of page
// "十亿参数的三维重建模型，能塞进手机吗？" (sections 预全局旋转, 后局部平滑,
// 训练后量化（PTQ）, 细粒度量化粒度): for each token row x of K values,
// y = x H_K (Sylvester Hadamard, natural order; the 1/sqrt(K) goes into the
// stored step), y_j *= mult_j, step = max|y| / sqrt(K) / 7, codes
// round-half-even(7 y / max|y|).  The CUDA-core version (quant.cu) spends most
// of its instructions on the butterflies; here the rotation is two small
// matrix products on the tensor cores, using the Kronecker structure of the
// Sylvester matrix: with K = R^2 (R = 32 for K = 1024, R = 64 for K = 4096)
// and a token row folded as X[a][b] = x[R a + b],
//     y[R a' + b'] = sum_{a, b} H_R[a][a'] X[a][b] H_R[b][b'].
//
//   stage 1 (kind::f16, bf16 inputs, exact products, fp32 accumulators):
//     Z[b][a'] = sum_a X[a][b] H_R[a][a'].  The MMA's A operand is the bf16
//     token tile exactly as TMA loads it (rows a, columns b), read MN-major
//     (M = b, contiguous; K = a); 128 / R tokens form one 128-row MMA.
//   stage 2 (kind::tf32, fp32 accumulators):
//     Y[a'][b'] = sum_b Z[b][a'] H_R[b][b'].  Z leaves tensor memory one row
//     (one b, all a') per thread, which is one K-row of the MN-major A
//     operand (M = a'); each value goes in as two tf32 terms, hi = Z with the
//     low 13 mantissa bits cleared and lo = tf32-round(Z - hi), whose sum
//     carries Z to a relative 2^-22.
//   finish: thread (token, a') reads Y[a'][0..R) = y[R a' .. R a' + R) from
//     tensor memory: R consecutive outputs, multiplied by mult, absmax over
//     the token (warp shuffles, plus one exchange between the two warps of a
//     token when R = 64), codes formed and stored as the CUDA-core kernel
//     does (codes.cuh).
//
// Warp roles (one persistent CTA of 384 threads per SM, 128-row groups
// round-robin over the CTAs):
//   warp 0      TMA producer: one 128 x R bf16 box per group (TOK tokens)
//   warp 1      MMA issuer (one thread): stage 1 of group i, then stage 2 of i-1
//   warp 2      tensor-memory allocator
//   warps 4..7  split: stage-1 accumulators -> hi / lo tf32 operand tiles
//   warps 8..11 finish: stage-2 accumulators -> smoothing, absmax, codes
// warp % 4 selects the 32 tensor-memory lanes a warp may access: lane
// 32 q + l holds row (token t, index rho) with t = (32 q + l) / R.
//
// Every wait is bounded (ptx.cuh): a stuck pipeline sets the device status
// word, the CTA lets its copies land and its MMAs finish, frees its tensor
// memory and returns.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "codes.cuh"
#include "ctxcache.h"
#include "kernels.h"
#include "ptx.cuh"

namespace w4a4 {
namespace {

constexpr int kTcThreads = 384;
constexpr int W_PROD = 0, W_MMA = 1, W_ALLOC = 2, W_SPLIT0 = 4, W_FIN0 = 8;

template <int K>
struct TcPlan {
  static constexpr int R = K == 1024 ? 32 : 64;      // H_K = H_R (x) H_R
  static constexpr int TOK = 128 / R;                // tokens per 128-row MMA group
  static constexpr int Q = R / 32;                   // lane quadrants (warps) per token
  static constexpr int XST = K == 1024 ? 6 : 3;      // token-tile stages
  static constexpr int D1S = K == 1024 ? 4 : 2;      // stage-1 accumulator slots (R columns)
  static constexpr int D2S = K == 1024 ? 4 : 2;      // stage-2 accumulator slots (R columns)
  static constexpr int A2B = 2;                      // stage-2 operand buffers
  static constexpr int NT = 2;                       // tf32 terms per value (hi, lo)
  static constexpr int X_BYTES = 128 * R * 2;        // one group's bf16 tile
  static constexpr uint32_t LAYOUT1 = R == 32 ? kLayoutSw64 : kLayoutSw128;  // 2R-byte rows
  static constexpr int SW1 = 2 * R;                  // swizzle width of the bf16 tiles (bytes)
  static constexpr int A1_LBO = 2 * K;               // tokens (MN atoms) apart in the tile
  static constexpr int A1_SBO = 8 * 2 * R;           // 8 rows a apart
  static constexpr int B1_BYTES = R * R * 2;
  static constexpr int B1_SBO = 8 * 2 * R;
  static constexpr int TERM = 128 * R * 4;           // one tf32 term of the stage-2 A operand
  static constexpr int A2_BYTES = NT * TERM;
  static constexpr int A2_LBO = (R / 8) * 1024;      // MN atoms (32 values of a') apart
  static constexpr int B2_BYTES = R * R * 4;
  static constexpr int OFF_X = 0;
  static constexpr int OFF_A2 = OFF_X + XST * X_BYTES;
  static constexpr int OFF_B1 = OFF_A2 + A2B * A2_BYTES;
  static constexpr int OFF_B2 = OFF_B1 + (B1_BYTES + 1023) / 1024 * 1024;
  static constexpr int OFF_TAB = OFF_B2 + B2_BYTES;  // multipliers, K floats
  static constexpr int OFF_PAIR = OFF_TAB + 4 * K;   // [D2S][4] per-warp absmax (R = 64)
  static constexpr int OFF_BAR = OFF_PAIR + D2S * 4 * 4;
  static constexpr int NUM_BARS = 2 * XST + 2 * D1S + 2 * A2B + 2 * D2S + D2S * TOK + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;  // + slack to align the base to 1024
  static constexpr uint32_t TMEM_COLS = 256;
  static_assert(D1S * R + D2S * R <= static_cast<int>(TMEM_COLS), "tensor-memory budget");
  static_assert(SMEM <= 232448, "shared-memory budget");
  static_assert(OFF_A2 % 1024 == 0 && OFF_B1 % 1024 == 0 && OFF_B2 % 1024 == 0 && X_BYTES % 1024 == 0,
                "swizzled tiles need 1024-byte alignment");
  static constexpr uint32_t IDESC1 = idesc_f32acc<128, R, false, true>();
  static constexpr uint32_t IDESC2 = idesc_f32acc<128, R, true, true>();
};

// Physical offset of a logical byte offset inside a tile whose 16-byte chunks
// are XOR-swizzled by address bits 7.. (64-byte: 2 bits, 128-byte: 3 bits).
__device__ __forceinline__ uint32_t swz(uint32_t off, int width) {
  const uint32_t mask = width == 64 ? 3u : 7u;
  return off ^ (((off >> 7) & mask) << 4);
}

__device__ __forceinline__ uint32_t tf32_rna(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}

template <int K, int CODE>
__global__ void __launch_bounds__(kTcThreads, 1)
    quant_tc_kernel(const __grid_constant__ CUtensorMap tmX, int64_t M, const float *__restrict__ mult,
                    uint8_t *__restrict__ q, float *__restrict__ scale, unsigned int *__restrict__ status,
                    int num_groups) {
  using P = TcPlan<K>;
  constexpr int R = P::R;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + P::OFF_BAR);
  uint64_t *x_full = bars;                      // a group's token tile landed
  uint64_t *x_free = x_full + P::XST;           // stage-1 MMAs reading it completed
  uint64_t *d1_full = x_free + P::XST;          // stage-1 accumulators complete
  uint64_t *d1_free = d1_full + P::D1S;         // split warps read them (4 arrivals)
  uint64_t *a2_full = d1_free + P::D1S;         // stage-2 operand written (4 arrivals)
  uint64_t *a2_free = a2_full + P::A2B;         // stage-2 MMAs reading it completed
  uint64_t *d2_full = a2_free + P::A2B;         // stage-2 accumulators complete
  uint64_t *d2_free = d2_full + P::D2S;         // finish warps read them (4 arrivals)
  uint64_t *pair_bar = d2_free + P::D2S;        // [D2S][TOK]: the two warps of a token (R = 64)
  uint64_t *mma_done = pair_bar + P::D2S * P::TOK;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + P::OFF_MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + P::OFF_MISC + 4);
  float *pairmax = reinterpret_cast<float *>(smem + P::OFF_PAIR);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < P::XST; ++s) {
      mbar_init(&x_full[s], 1);
      mbar_init(&x_free[s], 1);
    }
    for (int s = 0; s < P::D1S; ++s) {
      mbar_init(&d1_full[s], 1);
      mbar_init(&d1_free[s], 4);
    }
    for (int s = 0; s < P::A2B; ++s) {
      mbar_init(&a2_full[s], 4);
      mbar_init(&a2_free[s], 1);
    }
    for (int s = 0; s < P::D2S; ++s) {
      mbar_init(&d2_full[s], 1);
      mbar_init(&d2_free[s], 4);
    }
    for (int s = 0; s < P::D2S * P::TOK; ++s) mbar_init(&pair_bar[s], 2);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == W_PROD && lane == 0) tma_prefetch_desc(&tmX);
  if (warp == W_ALLOC) {
    tmem_alloc(tmem_slot, P::TMEM_COLS);
    tmem_relinquish();
  }
  // The two Hadamard operands, +-1 in bf16 (stage 1) and tf32 (stage 2),
  // K-major: row n holds H_R[k][n] over k (H_R is symmetric).
  {
    uint8_t *b1 = smem + P::OFF_B1;
    uint8_t *b2 = smem + P::OFF_B2;
    for (int idx = threadIdx.x; idx < R * R; idx += kTcThreads) {
      const int n = idx / R, k = idx % R;
      const bool neg = (__popc(n & k) & 1) != 0;
      *reinterpret_cast<uint16_t *>(b1 + swz(n * 2 * R + 2 * k, P::SW1)) = neg ? 0xBF80u : 0x3F80u;
      // tf32 rows are 4R bytes: K halves of 32 values, each a 128-byte swizzled tile
      const uint32_t off2 = (k / 32) * (R * 128) + n * 128 + (k % 32) * 4;
      *reinterpret_cast<uint32_t *>(b2 + swz(off2, 128)) = neg ? 0xBF800000u : 0x3F800000u;
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Everything above may overlap the tail of the previous kernel of the
  // stream; X and mult are read only after it has completed.
  griddep_launch_dependents();
  griddep_wait();
  {
    // multiplier table: float4 (c, rho) at c * R + rho holds mult[R rho + 4c .. + 3]
    // (the finishing thread rho reads its R consecutive multipliers; a warp's
    // 16-byte reads of one c are consecutive: conflict-free)
    float4 *tab = reinterpret_cast<float4 *>(smem + P::OFF_TAB);
    for (int idx = threadIdx.x; idx < K / 4; idx += kTcThreads) {
      const int c = idx / R, rho = idx % R;
      tab[idx] = __ldg(reinterpret_cast<const float4 *>(mult + R * rho + 4 * c));
    }
  }
  __syncthreads();

  if (warp == W_PROD) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      uint32_t it = 0;
      for (int g = blockIdx.x; g < num_groups; g += gridDim.x, ++it) {
        const uint32_t s = it % P::XST;
        if (!mbar_wait(&x_free[s], ((it / P::XST) & 1u) ^ 1u, abort_flag, status)) break;
        mbar_arrive_expect_tx(&x_full[s], P::X_BYTES);
        tma_load_2d(smem + P::OFF_X + s * P::X_BYTES, &tmX, 0, g * 128, &x_full[s]);
      }
      // let every issued copy land before the CTA can exit
      for (uint32_t u = (it > P::XST ? it - P::XST : 0); u < it; ++u)
        mbar_wait_drain(&x_full[u % P::XST], (u / P::XST) & 1u, status);
    }
  } else if (warp == W_MMA) {
    if (lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      const uint32_t x0 = smem_u32(smem + P::OFF_X);
      const uint32_t a20 = smem_u32(smem + P::OFF_A2);
      const uint32_t b1 = smem_u32(smem + P::OFF_B1);
      const uint32_t b2 = smem_u32(smem + P::OFF_B2);
      // stage 2 of the i-th group of this CTA
      auto stage2 = [&](uint32_t i) -> bool {
        const uint32_t ab = i % P::A2B, d2 = i % P::D2S;
        if (!mbar_wait(&a2_full[ab], (i / P::A2B) & 1u, abort_flag, status)) return false;
        if (!mbar_wait(&d2_free[d2], ((i / P::D2S) & 1u) ^ 1u, abort_flag, status)) return false;
        tc_fence_after();
        const uint32_t d = tmem_base + P::D1S * R + d2 * R;
#pragma unroll
        for (int term = 0; term < P::NT; ++term)
#pragma unroll
          for (int j = 0; j < R / 8; ++j)
            mma_tf32(d,
                     umma_desc(a20 + ab * P::A2_BYTES + term * P::TERM + j * 1024, P::A2_LBO, 1024,
                               kLayoutSw128),
                     umma_desc(b2 + (j / 4) * (R * 128) + (j % 4) * 32, 16, 1024, kLayoutSw128),
                     P::IDESC2, (term | j) != 0 ? 1u : 0u);
        tc_commit(&a2_free[ab]);
        tc_commit(&d2_full[d2]);
        return true;
      };
      uint32_t it = 0;
      bool ok = true;
      for (int g = blockIdx.x; g < num_groups; g += gridDim.x, ++it) {
        const uint32_t s = it % P::XST, d1 = it % P::D1S;
        if (!mbar_wait(&x_full[s], (it / P::XST) & 1u, abort_flag, status) ||
            !mbar_wait(&d1_free[d1], ((it / P::D1S) & 1u) ^ 1u, abort_flag, status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + d1 * R;
#pragma unroll
        for (int j = 0; j < R / 16; ++j)
          mma_f16(d, umma_desc(x0 + s * P::X_BYTES + j * 2 * P::A1_SBO, P::A1_LBO, P::A1_SBO, P::LAYOUT1),
                  umma_desc(b1 + j * 32, 16, P::B1_SBO, P::LAYOUT1), P::IDESC1, j != 0 ? 1u : 0u);
        tc_commit(&x_free[s]);
        tc_commit(&d1_full[d1]);
        if (it > 0 && !stage2(it - 1)) {
          ok = false;
          break;
        }
      }
      if (ok && it > 0) stage2(it - 1);
      // every MMA issued must finish before tensor memory is freed
      tc_commit(mma_done);
      mbar_wait_drain(mma_done, 0, status);
    }
  } else if (warp >= W_SPLIT0 && warp < W_SPLIT0 + 4) {
    // ------------------------------------------------------------------ split
    const int qd = warp & 3;
    const int t = qd / P::Q;                 // token of the group
    const int rho = (qd % P::Q) * 32 + lane; // b: one K-row of the stage-2 operand
    const uint32_t taddr0 = tmem_base + (static_cast<uint32_t>(qd * 32) << 16);
    const uint32_t a2base = smem_u32(smem + P::OFF_A2);
    uint32_t it = 0;
    for (int g = blockIdx.x; g < num_groups; g += gridDim.x, ++it) {
      const uint32_t d1 = it % P::D1S, ab = it % P::A2B;
      if (!mbar_wait(&d1_full[d1], (it / P::D1S) & 1u, abort_flag, status)) break;
      tc_fence_after();
      uint32_t z[R];
      tmem_ld_32x32b_x32(taddr0 + d1 * R, *reinterpret_cast<uint32_t(*)[32]>(&z[0]));
      if constexpr (R == 64)
        tmem_ld_32x32b_x32(taddr0 + d1 * R + 32, *reinterpret_cast<uint32_t(*)[32]>(&z[32]));
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&d1_free[d1]);
      if (!mbar_wait(&a2_free[ab], ((it / P::A2B) & 1u) ^ 1u, abort_flag, status)) break;
      // row rho of atom (t, ah): logical offset atom * LBO + (rho / 8) * 1024 + (rho % 8) * 128,
      // 16-byte chunk c (values a' = 32 ah + 4c .. + 3) at c ^ (rho % 8)
      const uint32_t rowb = a2base + ab * P::A2_BYTES + (rho >> 3) * 1024 + (rho & 7) * 128;
#pragma unroll
      for (int ah = 0; ah < P::Q; ++ah) {
        const uint32_t atom = rowb + (t * P::Q + ah) * P::A2_LBO;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint32_t x = z[32 * ah + 4 * c + e];
            hi[e] = x & 0xFFFFE000u;
            lo[e] = tf32_rna(__uint_as_float(x) - __uint_as_float(hi[e]));
          }
          const uint32_t a = atom + ((c ^ (rho & 7)) << 4);
          st_shared_v4(a, hi[0], hi[1], hi[2], hi[3]);
          st_shared_v4(a + P::TERM, lo[0], lo[1], lo[2], lo[3]);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&a2_full[ab]);
    }
  } else if (warp >= W_FIN0) {
    // ----------------------------------------------------------------- finish
    const int qd = warp & 3;
    const int t = qd / P::Q;
    const int rho = (qd % P::Q) * 32 + lane;  // a': outputs R rho .. R rho + R - 1
    const uint32_t taddr0 = tmem_base + (static_cast<uint32_t>(qd * 32) << 16) + P::D1S * R;
    const float4 *tab = reinterpret_cast<const float4 *>(smem + P::OFF_TAB);
    constexpr float kQmax = CODE == kCodeBytes8 ? 127.0f : 7.0f;
    constexpr float kInvSqrtK = K == 1024 ? 0.03125f : 0.015625f;
    uint32_t it = 0;
    for (int g = blockIdx.x; g < num_groups; g += gridDim.x, ++it) {
      const uint32_t d2 = it % P::D2S;
      if (!mbar_wait(&d2_full[d2], (it / P::D2S) & 1u, abort_flag, status)) break;
      tc_fence_after();
      uint32_t yb[R];
      tmem_ld_32x32b_x32(taddr0 + d2 * R, *reinterpret_cast<uint32_t(*)[32]>(&yb[0]));
      if constexpr (R == 64)
        tmem_ld_32x32b_x32(taddr0 + d2 * R + 32, *reinterpret_cast<uint32_t(*)[32]>(&yb[32]));
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&d2_free[d2]);
      float y[R];
#pragma unroll
      for (int c = 0; c < R / 4; ++c) {
        const float4 m = tab[c * R + rho];
        y[4 * c + 0] = __uint_as_float(yb[4 * c + 0]);
        y[4 * c + 1] = __uint_as_float(yb[4 * c + 1]);
        y[4 * c + 2] = __uint_as_float(yb[4 * c + 2]);
        y[4 * c + 3] = __uint_as_float(yb[4 * c + 3]);
        mul_x2(y[4 * c + 0], y[4 * c + 1], m.x, m.y);
        mul_x2(y[4 * c + 2], y[4 * c + 3], m.z, m.w);
      }
      float am[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int r = 0; r < R; r += 8)
#pragma unroll
        for (int a = 0; a < 4; ++a) am[a] = fmax3(am[a], fabsf(y[r + 2 * a]), fabsf(y[r + 2 * a + 1]));
      float amax = fmax3(am[0], am[1], fmaxf(am[2], am[3]));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      if constexpr (P::Q == 2) {
        // the other warp of this token holds the other half of its outputs
        uint64_t *pb = &pair_bar[d2 * P::TOK + t];
        if (lane == 0) {
          pairmax[d2 * 4 + qd] = amax;
          mbar_arrive(pb);
        }
        if (!mbar_wait(pb, (it / P::D2S) & 1u, abort_flag, status)) break;
        amax = fmaxf(amax, pairmax[d2 * 4 + (qd ^ 1)]);
      }
      const int64_t tok = static_cast<int64_t>(g) * P::TOK + t;
      if (tok < M) {
        if (lane == 0 && (qd % P::Q) == 0) scale[tok] = amax * kInvSqrtK / kQmax;
        store_codes<R, CODE>(y, amax, q + tok * code_bytes_of<CODE>(K) + rho * code_bytes_of<CODE>(R));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == W_ALLOC) tmem_dealloc(tmem_base, P::TMEM_COLS);
}

// Tokens per launch: the TMA row coordinate (token * R) must stay below 2^31.
constexpr int64_t kTcMaxTokens = int64_t(1) << 24;

template <int K, int CODE>
cudaError_t launch_tc_k(const uint16_t *X, int64_t M, const float *mult, uint8_t *q, float *scale,
                        cudaStream_t st) {
  using P = TcPlan<K>;
  auto kern = quant_tc_kernel<K, CODE>;
  static ContextCache<bool> attr;
  bool done = false;
  cudaError_t e = attr.get(&done, [&](bool *v) {
    *v = true;
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, P::SMEM);
  });
  if (e != cudaSuccess) return e;
  unsigned int *status = nullptr;
  if ((e = status_word(&status)) != cudaSuccess) return e;
  for (int64_t m0 = 0; m0 < M; m0 += kTcMaxTokens) {
    const int64_t m = (M - m0 < kTcMaxTokens) ? M - m0 : kTcMaxTokens;
    // the token rows as m R rows of R bf16 values (row a of every token)
    CUtensorMap tm;
    if (!encode_tensor_map_2d(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X + m0 * K, P::R,
                              static_cast<uint64_t>(m) * P::R, 2 * P::R, P::R, 128,
                              P::R == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
    const int groups = static_cast<int>((m + P::TOK - 1) / P::TOK);
    const int sms = device_sm_count();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(groups < sms ? groups : sms, 1, 1);
    cfg.blockDim = dim3(kTcThreads, 1, 1);
    cfg.dynamicSmemBytes = P::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, tm, m, mult, q + m0 * code_bytes_of<CODE>(K), scale + m0, status,
                           groups);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

template <int CODE>
cudaError_t launch_tc_c(const uint16_t *X, int64_t M, int K, const float *mult, uint8_t *q, float *scale,
                        cudaStream_t st) {
  return K == 1024 ? launch_tc_k<1024, CODE>(X, M, mult, q, scale, st)
                   : launch_tc_k<4096, CODE>(X, M, mult, q, scale, st);
}

}  // namespace

cudaError_t launch_quantize_rows_tc(const uint16_t *X, int64_t M, int K, const float *mult, uint8_t *q,
                                    float *scale, CodeFormat code, cudaStream_t st) {
  if (M <= 0) return cudaSuccess;
  switch (code) {
    case kCodeBytes4: return launch_tc_c<kCodeBytes4>(X, M, K, mult, q, scale, st);
    case kCodeBytes8: return launch_tc_c<kCodeBytes8>(X, M, K, mult, q, scale, st);
    default: return launch_tc_c<kCodePacked4>(X, M, K, mult, q, scale, st);
  }
}

}  // namespace w4a4
