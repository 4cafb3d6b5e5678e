// quant_tc.cu -- the DSFQ activation quantizer with most of the Hadamard
// rotation on the tensor cores (sm_100a tcgen05).
//
// What it computes is the rotate -> smooth -> per-token int4 step of page
// "十亿参数的三维重建模型，能塞进手机吗？" (sections 预全局旋转, 后局部平滑,
// 训练后量化（PTQ）, 细粒度量化粒度): for each token row x of K values,
// y = x H_K (Sylvester Hadamard, natural order; the 1/sqrt(K) goes into the
// stored step), y_j *= mult_j, step = max|y| / sqrt(K) / 7, codes
// round-half-even(7 y / max|y|).
//
// The Sylvester matrix factors as H_K = H_128 (x) H_S with S = K / 128 (8 at
// K = 1024, 32 at K = 4096).  Folding a token row as X[a][b] = x[S a + b]
// (a < 128, b < S),
//     y[S a' + b'] = sum_b H_S[b][b'] Z[b][a'],   Z[b][a'] = sum_a H_128[a'][a] X[a][b].
//   * Z on the tensor cores (kind::f16: bf16 inputs, exact +-1 products, fp32
//     accumulators): D[a'][n] = sum_a H_128[a'][a] B[n][a] with A = H_128
//     (128 x 128, K-major) and B the bf16 token tile read MN-major: column
//     n = S t + b of token t of the tile, contiguous in b, exactly as the
//     tokens lie in memory.  One 128 x 128 x 16 MMA covers 128 / S tokens;
//     eight cover the 128 values of a.  (Few large MMAs: a tcgen05.mma takes
//     about 100 cycles to issue whatever its size, so a factorisation into
//     small products -- H_32 (x) H_32 as two N = 32 stages -- is bound by the
//     issuing thread.)
//   * H_S in registers: thread a' (tensor-memory lane a') holds Z[b][a'] for
//     every b of each token, so the remaining log2(S) butterfly stages run on
//     values the thread already has, and the thread ends with S consecutive
//     outputs y[S a' .. S a' + S) -- their codes go out as one contiguous
//     store, with no transpose.
//   * absmax: a token's outputs are spread over the 128 lanes (4 warps), so
//     each tile goes through tensor memory twice: pass 1 applies H_S and the
//     multipliers, writes the values back in place (tcgen05.st) and forms the
//     per-token maxima (warp shuffles, then one exchange between the 4 warps
//     through shared memory); pass 2 reads the values again and forms the
//     codes with each token's reciprocal step, computed once by one lane.
//     Each pass reads its 128 columns in four 32-column loads; at K = 4096
//     the next load is issued before the current chunk is worked on.
//
// Warp roles (one persistent CTA of 512 threads per SM; tiles of 128 / S
// tokens round-robin over the CTAs):
//   warp 0        producer: one bulk copy (K = 1024) or two TMA boxes (K = 4096)
//                 per tile into a ring of stages
//   warp 1        MMA issuer (one thread): 8 MMAs per tile into one of four
//                 128-column accumulator slots of tensor memory
//   warp 2        tensor-memory allocator
//   warps 4..15   three finishing sets of 4 warps (one per lane quadrant);
//                 successive tiles go to the sets in turn (a set's passes
//                 wait on tensor-memory loads, so several tiles in flight
//                 hide that latency)
//
// Every wait is bounded (ptx.cuh): a stuck pipeline sets the device status
// word, the CTA lets its copies land and its MMAs finish, frees its tensor
// memory and returns.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <type_traits>

#include "codes.cuh"
#include "ctxcache.h"
#include "fwht.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace w4a4 {
namespace {

constexpr int kTcThreads = 512;
constexpr int W_PROD = 0, W_MMA = 1, W_ALLOC = 2, W_FIN0 = 4;
constexpr int kFinSets = 3;  // (with two, the 32-frame K = 1024 layers ran 8 % slower)
constexpr int kSlots = 4;        // accumulator slots (128 columns each)
constexpr int kHBytes = 128 * 128 * 2;

template <int K>
struct TcPlan {
  static constexpr int S = K / 128;                  // H_K = H_128 (x) H_S
  static constexpr int LOGS = S == 8 ? 3 : 5;
  static constexpr int TOKT = 128 / S;               // tokens per tile (N = 128 columns)
  static constexpr int X_BYTES = TOKT * K * 2;       // one tile of bf16 tokens (32 KB)
  static constexpr int XST = 4;                      // tile stages
  // B operand (the token tile, MN-major): K = 1024: no swizzle, 8-row groups
  // of 16-byte rows, tokens (MN atoms of 8 values) 2 KB apart; K = 4096:
  // 64-byte swizzle (the TMA boxes' layout), atoms of 32 values, tokens 8 KB
  // apart, 8-row groups 512 bytes apart.
  static constexpr uint32_t B_LAYOUT = S == 8 ? 0u : kLayoutSw64;
  static constexpr uint32_t B_LBO = S == 8 ? 128u : static_cast<uint32_t>(2 * K);
  static constexpr uint32_t B_SBO = S == 8 ? static_cast<uint32_t>(2 * K) : 512u;
  static constexpr uint32_t B_KSTEP = S == 8 ? 256u : 1024u;  // 16 rows of a
  static constexpr int OFF_X = 0;
  static constexpr int OFF_H = OFF_X + XST * X_BYTES;
  static constexpr int OFF_TM = OFF_H + kHBytes;     // [kSlots][TOKT][4] warp maxima
  static constexpr int OFF_BAR = OFF_TM + kSlots * TOKT * 4 * 4;
  static constexpr int NUM_BARS = 2 * XST + 3 * kSlots + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;  // + slack to align the base to 1024
  static_assert(SMEM <= 232448, "shared-memory budget");
  static_assert(OFF_H % 1024 == 0 && X_BYTES % 1024 == 0, "tile alignment");
  // kind::f16, bf16 A and B, fp32 D, A K-major, B MN-major, M = N = 128
  static constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                                    ((128u >> 3) << 17) | ((128u >> 4) << 24);
};

template <int K, int CODE>
__global__ void __launch_bounds__(kTcThreads, 1)
    quant_tc_kernel(const __grid_constant__ CUtensorMap tmX, const uint16_t *__restrict__ X, int64_t M,
                    const float *__restrict__ mult, uint8_t *__restrict__ q, float *__restrict__ scale,
                    unsigned int *__restrict__ status, int num_tiles) {
  using P = TcPlan<K>;
  constexpr int S = P::S, TOKT = P::TOKT;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + P::OFF_BAR);
  uint64_t *x_full = bars;                 // a tile's tokens landed
  uint64_t *x_free = x_full + P::XST;      // the MMAs reading it completed
  uint64_t *d_full = x_free + P::XST;      // an accumulator slot complete
  uint64_t *d_free = d_full + kSlots;      // its 4 finishing warps are done with it
  uint64_t *tm_bar = d_free + kSlots;      // its 4 finishing warps wrote their maxima
  uint64_t *mma_done = tm_bar + kSlots;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + P::OFF_MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + P::OFF_MISC + 4);
  float *tmax = reinterpret_cast<float *>(smem + P::OFF_TM);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < P::XST; ++s) {
      mbar_init(&x_full[s], 1);
      mbar_init(&x_free[s], 1);
    }
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&d_full[s], 1);
      mbar_init(&d_free[s], 4);
      mbar_init(&tm_bar[s], 4);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == W_PROD && lane == 0 && S != 8) tma_prefetch_desc(&tmX);
  if (warp == W_ALLOC) {
    tmem_alloc(tmem_slot, kSlots * 128);
    tmem_relinquish();
  }
  {
    // H_128 in bf16, K-major with the 128-byte swizzle: row a' holds
    // H[a'][a] over a, in two 64-value halves of 16 KB (row a' at 128 a',
    // 16-byte chunk c at c ^ (a' % 8)).  One 16-byte store per chunk of 8
    // values a = 8c + i: H[a'][a] = (-1)^(popc(a' & 8c) + popc(a' & i)), the
    // row of H_8 selected by a' % 8, negated when a' & 8c has odd parity.
    uint8_t *h = smem + P::OFF_H;
    for (int q = threadIdx.x; q < 128 * 16; q += kTcThreads) {
      const int ap = q >> 4, c = q & 15;
      const uint32_t flip = (__popc(ap & (8 * c)) & 1) ? 0x80008000u : 0u;
      uint32_t w[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t lo = (__popc(ap & 7 & (2 * k)) & 1) ? 0xBF80u : 0x3F80u;
        const uint32_t hi = (__popc(ap & 7 & (2 * k + 1)) & 1) ? 0xBF80u : 0x3F80u;
        w[k] = (lo | (hi << 16)) ^ flip;
      }
      *reinterpret_cast<uint4 *>(h + (c >> 3) * 16384 + ap * 128 + (((c & 7) ^ (ap & 7)) << 4)) =
          make_uint4(w[0], w[1], w[2], w[3]);
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

  if (warp == W_PROD) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      // K = 4096: X is read once, and its lines are made the first to go when
      // L2 needs room (87936 tokens: 199 -> 195 us alone, 249 -> 241 us
      // inside the stack step).  At K = 1024 the same hint made the kernel
      // alone slower (44 -> 48 us) and left it unchanged in the step.
      const uint64_t x_policy = S == 8 ? 0 : l2_policy_evict_first();
      uint32_t it = 0;
      for (int g = blockIdx.x; g < num_tiles; g += gridDim.x, ++it) {
        const uint32_t s = it % P::XST;
        if (!mbar_wait(&x_free[s], ((it / P::XST) & 1u) ^ 1u, abort_flag, status)) break;
        uint8_t *dst = smem + P::OFF_X + s * P::X_BYTES;
        const int64_t tok0 = static_cast<int64_t>(g) * TOKT;
        if constexpr (S == 8) {
          // the tile's tokens are contiguous: one bulk copy of the valid ones
          // (the rest of the stage keeps old bytes; their columns are not stored)
          const int64_t valid = (M - tok0 < TOKT) ? M - tok0 : TOKT;
          const uint32_t bytes = static_cast<uint32_t>(valid) * 2 * K;
          mbar_arrive_expect_tx(&x_full[s], bytes);
          bulk_load(dst, X + tok0 * K, bytes, &x_full[s]);
        } else {
          // rows (token, a) of S values through the 64-byte swizzle, 256 rows
          // (two tokens) per box; rows past the end are filled with zeros
          mbar_arrive_expect_tx(&x_full[s], P::X_BYTES);
          tma_load_2d_hint(dst, &tmX, 0, static_cast<int>(g * 512), &x_full[s], x_policy);
          tma_load_2d_hint(dst + P::X_BYTES / 2, &tmX, 0, static_cast<int>(g * 512 + 256), &x_full[s],
                           x_policy);
        }
      }
      // let every issued copy land before the CTA can exit
      for (uint32_t u = (it > P::XST ? it - P::XST : 0); u < it; ++u)
        mbar_wait_drain(&x_full[u % P::XST], (u / P::XST) & 1u, status);
    }
  } else if (warp == W_MMA) {
    if (lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      const uint32_t x0 = smem_u32(smem + P::OFF_X);
      const uint32_t h0 = smem_u32(smem + P::OFF_H);
      uint32_t it = 0;
      for (int g = blockIdx.x; g < num_tiles; g += gridDim.x, ++it) {
        const uint32_t s = it % P::XST, d = it % kSlots;
        if (!mbar_wait(&x_full[s], (it / P::XST) & 1u, abort_flag, status) ||
            !mbar_wait(&d_free[d], ((it / kSlots) & 1u) ^ 1u, abort_flag, status))
          break;
        tc_fence_after();
#pragma unroll
        for (int j = 0; j < 8; ++j)
          mma_f16(tmem_base + d * 128,
                  umma_desc(h0 + (j >> 2) * 16384 + (j & 3) * 32, 16, 1024, kLayoutSw128),
                  umma_desc(x0 + s * P::X_BYTES + j * P::B_KSTEP, P::B_LBO, P::B_SBO, P::B_LAYOUT),
                  P::IDESC, j != 0 ? 1u : 0u);
        tc_commit(&x_free[s]);
        tc_commit(&d_full[d]);
      }
      // every MMA issued must finish before tensor memory is freed
      tc_commit(mma_done);
      mbar_wait_drain(mma_done, 0, status);
    }
  } else if (warp >= W_FIN0 && warp < W_FIN0 + 4 * kFinSets) {
    // ----------------------------------------------------------------- finish
    const int qd = warp & 3;
    const int set = (warp - W_FIN0) >> 2;
    const int ap = 32 * qd + lane;               // a': outputs S a' .. S a' + S - 1
    const uint32_t tq = tmem_base + (static_cast<uint32_t>(32 * qd) << 16);
    constexpr float kQmax = CODE == kCodeBytes8 ? 127.0f : 7.0f;
    constexpr float kInvSqrtK = K == 1024 ? 0.03125f : 0.015625f;
    float m[S];                                  // this thread's multipliers
#pragma unroll
    for (int c = 0; c < S / 4; ++c) {
      const float4 v = __ldg(reinterpret_cast<const float4 *>(mult + S * ap) + c);
      m[4 * c] = v.x;
      m[4 * c + 1] = v.y;
      m[4 * c + 2] = v.z;
      m[4 * c + 3] = v.w;
    }
    // token u of a 32-column load: its S values for this lane, transformed
    // by H_S and smoothed
    auto token_values = [&](const uint32_t (&r)[32], int j0, float (&y)[S]) {
#pragma unroll
      for (int b = 0; b < S; ++b) y[b] = __uint_as_float(r[j0 + b]);
      butterflies<S, 0, P::LOGS>(y);
#pragma unroll
      for (int b = 0; b < S; b += 2) mul_x2(y[b], y[b + 1], m[b], m[b + 1]);
    };
    auto local_max = [&](const float (&y)[S]) {
      float am = 0.0f;
#pragma unroll
      for (int b = 0; b < S; b += 2) am = fmax3(am, fabsf(y[b]), fabsf(y[b + 1]));
      return am;
    };
    for (uint32_t it = set; blockIdx.x + it * gridDim.x < static_cast<uint32_t>(num_tiles);
         it += kFinSets) {
      const int g = static_cast<int>(blockIdx.x + it * gridDim.x);
      const uint32_t d = it % kSlots;
      if (!mbar_wait(&d_full[d], (it / kSlots) & 1u, abort_flag, status)) break;
      tc_fence_after();
      const uint32_t taddr = tq + d * 128;
      // pass 1: H_S and the multipliers, written back in place (tcgen05.st),
      // and the per-token maxima over this warp's 32 lanes
      float tok_max[TOKT];
      auto pass1_chunk = [&](int c, uint32_t(&r)[32]) {
#pragma unroll
        for (int u = 0; u < 32 / S; ++u) {
          float y[S];
          token_values(r, u * S, y);
          tok_max[c * (32 / S) + u] = local_max(y);
#pragma unroll
          for (int b = 0; b < S; ++b) r[u * S + b] = __float_as_uint(y[b]);
        }
        tmem_st_32x32b_x32(taddr + 32 * c, r);
      };
      if constexpr (S == 32) {
        // one token per chunk: chunk c + 1's load is in flight while chunk c
        // is transformed (87936 tokens: 201 -> 199 us at K = 4096; at
        // K = 1024 the second buffer cost more than the overlap gained,
        // 44 -> 50 us, so S = 8 keeps one load at a time)
        uint32_t ra[32], rb[32];
        tmem_ld_32x32b_x32(taddr, ra);
        tmem_wait_ld();
        tmem_ld_32x32b_x32(taddr + 32, rb);
        pass1_chunk(0, ra);
        tmem_wait_ld();
        tmem_ld_32x32b_x32(taddr + 64, ra);
        pass1_chunk(1, rb);
        tmem_wait_ld();
        tmem_ld_32x32b_x32(taddr + 96, rb);
        pass1_chunk(2, ra);
        tmem_wait_ld();
        pass1_chunk(3, rb);
      } else {
#pragma unroll
        for (int c = 0; c < 4; ++c) {              // 32 columns = 32 / S tokens
          uint32_t r[32];
          tmem_ld_32x32b_x32(taddr + 32 * c, r);
          tmem_wait_ld();
          pass1_chunk(c, r);
        }
      }
      // maxima over the warp, reduce-scattered: at the step with lane offset
      // o a lane keeps the half of its remaining tokens that its lane bit
      // selects and sends the other half, so lane l ends with the warp's
      // maximum of token l / (32 / TOKT)
#pragma unroll
      for (int step = 0; step < 5; ++step) {
        const int o = 16 >> step;
        const int half = (TOKT >> step) / 2;     // tokens sent at this step (0: plain reduce)
        const bool upper = (lane & o) != 0;
        if (half > 0) {
#pragma unroll
          for (int j = 0; j < (half > 0 ? half : 1); ++j) {
            const float keep = upper ? tok_max[j + half] : tok_max[j];
            const float send = upper ? tok_max[j] : tok_max[j + half];
            tok_max[j] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, o));
          }
        } else {
          tok_max[0] = fmaxf(tok_max[0], __shfl_xor_sync(0xffffffffu, tok_max[0], o));
        }
      }
      // exchange with the other three warps of the set
      float *tm = tmax + d * TOKT * 4;
      constexpr int kLanesPerTok = 32 / TOKT;
      if (lane % kLanesPerTok == 0) tm[(lane / kLanesPerTok) * 4 + qd] = tok_max[0];
      __syncwarp();
      if (lane == 0) mbar_arrive(&tm_bar[d]);
      if (!mbar_wait(&tm_bar[d], (it / kSlots) & 1u, abort_flag, status)) break;
      // lane t < TOKT: token t's maximum, step and reciprocal step (the same
      // binary32 arithmetic as store_codes: a maximum below 2^-100 is first
      // scaled by 2^64, exactly, to keep kQmax / amax finite)
      const int64_t tok0 = static_cast<int64_t>(g) * TOKT;
      float inv_l = 0.0f, pre_l = 1.0f;
      if (lane < TOKT) {
        const float4 w = reinterpret_cast<const float4 *>(tm)[lane];
        float amax = fmaxf(fmaxf(w.x, w.y), fmaxf(w.z, w.w));
        if (qd == 0 && tok0 + lane < M) scale[tok0 + lane] = amax * kInvSqrtK / kQmax;
        if (amax < 0x1p-100f) {
          amax *= 0x1p+64f;
          pre_l = 0x1p+64f;
        }
        inv_l = amax > 0.0f ? kQmax / amax : 0.0f;
      }
      tmem_wait_st();
      // pass 2: codes.  The common tile (every token present, no step so
      // small that it needs the 2^64 rescale) runs without the per-token
      // rescale and bounds tests.
      const unsigned long long magic2 = pack2(12582912.0f, 12582912.0f);
      const bool plain_tile = !__any_sync(0xffffffffu, pre_l != 1.0f) && tok0 + TOKT <= M;
      auto release_slot = [&]() {                // the slot is no longer read
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&d_free[d]);
      };
      auto pass2 = [&](auto plain) {
        constexpr bool PLAIN = decltype(plain)::value;
        auto codes_chunk = [&](int c, const uint32_t(&r)[32]) {
#pragma unroll
          for (int u = 0; u < 32 / S; ++u) {
            const int t = c * (32 / S) + u;
            const float inv = __shfl_sync(0xffffffffu, inv_l, t);
            const int64_t tok = tok0 + t;
            if (PLAIN || tok < M) {
              float y[S];
#pragma unroll
              for (int b = 0; b < S; ++b) y[b] = __uint_as_float(r[u * S + b]);
              if constexpr (!PLAIN) {
                const float pre = __shfl_sync(0xffffffffu, pre_l, t);
                if (pre != 1.0f) {
#pragma unroll
                  for (int b = 0; b < S; ++b) y[b] *= pre;
                }
              }
              const unsigned long long inv2 = pack2(inv, inv);
#pragma unroll
              for (int b = 0; b < S; b += 2) fma_x2(y[b], y[b + 1], inv2, magic2);
              store_code_words<S, CODE>(y, q + tok * code_bytes_of<CODE>(K) + ap * code_bytes_of<CODE>(S));
            }
          }
        };
        if constexpr (S == 32) {                 // loads overlapped as in pass 1
          uint32_t ra[32], rb[32];
          tmem_ld_32x32b_x32(taddr, ra);
          tmem_wait_ld();
          tmem_ld_32x32b_x32(taddr + 32, rb);
          codes_chunk(0, ra);
          tmem_wait_ld();
          tmem_ld_32x32b_x32(taddr + 64, ra);
          codes_chunk(1, rb);
          tmem_wait_ld();
          tmem_ld_32x32b_x32(taddr + 96, rb);
          codes_chunk(2, ra);
          tmem_wait_ld();
          release_slot();
          codes_chunk(3, rb);
        } else {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t r[32];
            tmem_ld_32x32b_x32(taddr + 32 * c, r);
            tmem_wait_ld();
            if (c == 3) release_slot();
            codes_chunk(c, r);
          }
        }
      };
      if (plain_tile)
        pass2(std::true_type{});
      else
        pass2(std::false_type{});
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == W_ALLOC) tmem_dealloc(tmem_base, kSlots * 128);
}

// Tokens per launch: the TMA row coordinate (token * 128) must stay below 2^31.
constexpr int64_t kTcMaxTokens = int64_t(1) << 23;

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
    CUtensorMap tm = {};
    // K = 4096: the tokens as rows (token, a) of 32 bf16 values
    if (P::S != 8 &&
        !encode_tensor_map_2d(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X + m0 * K, P::S,
                              static_cast<uint64_t>(m) * 128, 2 * P::S, P::S, 256,
                              CU_TENSOR_MAP_SWIZZLE_64B))
      return cudaErrorInvalidValue;
    const int tiles = static_cast<int>((m + P::TOKT - 1) / P::TOKT);
    const int sms = device_sm_count();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(tiles < sms ? tiles : sms, 1, 1);
    cfg.blockDim = dim3(kTcThreads, 1, 1);
    cfg.dynamicSmemBytes = P::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, tm, X + m0 * K, m, mult, q + m0 * code_bytes_of<CODE>(K),
                           scale + m0, status, tiles);
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
