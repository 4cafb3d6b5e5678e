// gemm.cu -- the tensor-core half of the DSFQ W4A4 linear on sm_100a.
//
//   Y[m, n] = bf16( (sum_k qx[m, k] qw[n, k]) * scale_tok[m] * scale_ch[n] + bias[n] )
//
// qx [M, K/2] and qw [N, K/2] hold int4 codes packed two per byte (page
// "十亿参数的三维重建模型，能塞进手机吗？", section 训练后量化（PTQ）: symmetric
// 4-bit codes; section 细粒度量化粒度 read as per-token x per-channel steps).
// tcgen05 has no 4-bit integer MMA, so the kernel
//   1. stages packed tiles in shared memory with TMA (one warp, one thread),
//   2. unpacks them to int8 (4 warps) straight into the 128-byte-swizzled
//      K-major layout the tensor core reads,
//   3. issues tcgen05.mma kind::i8 (one thread) with s32 accumulators in tensor
//      memory, double-buffered so the epilogue of one tile overlaps the main
//      loop of the next,
//   4. reads the accumulators back with tcgen05.ld (4 warps), applies the
//      per-token x per-channel steps and the bias in fp32, rounds to bf16 and
//      writes the tile with TMA stores from a swizzled staging buffer.
// The CTA is persistent (one per SM, tiles assigned round-robin, M-major so
// that concurrently running CTAs share activation rows through L2).
//
// Unpacking permutes K inside every group of 8 codes (even codes first, then
// odd ones).  A and B are unpacked identically, so every dot product sums the
// same pairs and the integer result is exact and unchanged.
//
// Every wait is bounded (ptx.cuh): a stuck pipeline sets the device status word
// and the CTA drains its in-flight copies and MMAs, frees its tensor memory and
// returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "kernels.h"
#include "ptx.cuh"

namespace w4a4 {

// Device status word (bits W4A4_DEV_* of include/w4a4.h): the only state the
// library keeps between calls.
__device__ unsigned int g_status = 0;

namespace {

constexpr int BM = 128;   // tile rows (tokens)
constexpr int BN = 256;   // tile columns (output channels)
constexpr int BK = 128;   // int8 elements per k-block = one 128-byte swizzle row
constexpr int BKP = 64;   // packed bytes per row per k-block
constexpr int PST = 4;    // packed (TMA) stages
constexpr int UST = 2;    // unpacked (MMA operand) stages
constexpr int A_PK = BM * BKP;
constexpr int B_PK = BN * BKP;
constexpr int A_UN = BM * BK;
constexpr int B_UN = BN * BK;
constexpr int EPI_BYTES = 32 * 32 * 2;  // one warp's 32 x 32 bf16 staging tile
constexpr int NUM_THREADS = 384;        // 12 warps, roles below
constexpr uint32_t TMEM_COLS = 512;     // two 128 x 256 s32 accumulators
constexpr int OFF_A_UN = 0;
constexpr int OFF_B_UN = OFF_A_UN + UST * A_UN;
constexpr int OFF_A_PK = OFF_B_UN + UST * B_UN;
constexpr int OFF_B_PK = OFF_A_PK + PST * A_PK;
constexpr int OFF_EPI = OFF_B_PK + PST * B_PK;
constexpr int OFF_BAR = OFF_EPI + 4 * 2 * EPI_BYTES;
constexpr int NUM_BARS = 2 * PST + 2 * UST + 2 * 2 + 1;
constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + slack to align the base to 1024
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(OFF_B_UN % 1024 == 0 && OFF_A_PK % 1024 == 0 && OFF_EPI % 1024 == 0, "alignment");

constexpr uint32_t IDESC = idesc_i8<BM, BN>();

// Warp roles.
constexpr int W_TMA = 0, W_MMA = 1, W_TMEM = 2;
constexpr int W_UNPACK0 = 4;  // warps 4..7
constexpr int W_EPI0 = 8;     // warps 8..11 (warp % 4 selects its 32 TMEM lanes)

// 4 nibbles (one per byte, values 0..15 = two's-complement int4) -> 4 int8.
__device__ __forceinline__ uint32_t sext4x4(uint32_t n) {
  return ((n ^ 0x08080808u) + 0x78787878u) ^ 0x80808080u;
}

// Packed 16-byte chunk (32 codes) -> two 16-byte int8 chunks.  Word t holds
// codes 8t..8t+7; its even codes go first, then its odd codes.
__device__ __forceinline__ void unpack_chunk(uint4 v, uint4 &o0, uint4 &o1) {
  o0.x = sext4x4(v.x & 0x0F0F0F0Fu);
  o0.y = sext4x4((v.x >> 4) & 0x0F0F0F0Fu);
  o0.z = sext4x4(v.y & 0x0F0F0F0Fu);
  o0.w = sext4x4((v.y >> 4) & 0x0F0F0F0Fu);
  o1.x = sext4x4(v.z & 0x0F0F0F0Fu);
  o1.y = sext4x4((v.z >> 4) & 0x0F0F0F0Fu);
  o1.z = sext4x4(v.w & 0x0F0F0F0Fu);
  o1.w = sext4x4((v.w >> 4) & 0x0F0F0F0Fu);
}

// Unpack NCH packed chunks of a tile (rows of 64 packed bytes) into the
// 128-byte swizzled int8 tile.  Chunk q covers row q/4, codes 32(q%4)..+31.
template <int NCH>
__device__ __forceinline__ void unpack_tile(const uint8_t *__restrict__ src, uint8_t *__restrict__ dst,
                                            int t) {
  uint4 v[NCH];
#pragma unroll
  for (int i = 0; i < NCH; ++i) v[i] = *reinterpret_cast<const uint4 *>(src + (t + 128 * i) * 16);
#pragma unroll
  for (int i = 0; i < NCH; ++i) {
    const int q = t + 128 * i;
    const int r = q >> 2, c = q & 3;
    uint4 o0, o1;
    unpack_chunk(v[i], o0, o1);
    uint8_t *row = dst + r * 128;
    *reinterpret_cast<uint4 *>(row + (((2 * c) ^ (r & 7)) << 4)) = o0;
    *reinterpret_cast<uint4 *>(row + (((2 * c + 1) ^ (r & 7)) << 4)) = o1;
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&h);
}

template <bool OUT_S32>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    w4a4_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmY, const float *__restrict__ scale_tok,
                     const float *__restrict__ scale_ch, const float *__restrict__ bias,
                     int32_t *__restrict__ acc_out, int M, int N, int num_n_tiles, int num_tiles,
                     int num_kb) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
  uint64_t *pk_full = bars;
  uint64_t *pk_empty = pk_full + PST;
  uint64_t *un_full = pk_empty + PST;
  uint64_t *un_empty = un_full + UST;
  uint64_t *acc_full = un_empty + UST;
  uint64_t *acc_empty = acc_full + 2;
  uint64_t *mma_done = acc_empty + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + OFF_MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < PST; ++s) {
      mbar_init(&pk_full[s], 1);
      mbar_init(&pk_empty[s], 128);
    }
    for (int u = 0; u < UST; ++u) {
      mbar_init(&un_full[u], 128);
      mbar_init(&un_empty[u], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == W_TMA && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (!OUT_S32) tma_prefetch_desc(&tmY);
  }
  if (warp == W_TMEM) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == W_TMA) {
    if (lane == 0) {
      // ---------------------------------------------------------------- producer
      uint32_t issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int mb = tile / num_n_tiles, nb = tile % num_n_tiles;
        for (int kb = 0; kb < num_kb; ++kb) {
          const uint32_t s = issued % PST, ph = (issued / PST) & 1u;
          if (!mbar_wait(&pk_empty[s], ph ^ 1u, abort_flag, &g_status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&pk_full[s], A_PK + B_PK);
          tma_load_2d(smem + OFF_A_PK + s * A_PK, &tmA, kb * BKP, mb * BM, &pk_full[s]);
          tma_load_2d(smem + OFF_B_PK + s * B_PK, &tmB, kb * BKP, nb * BN, &pk_full[s]);
          ++issued;
        }
      }
      // let every issued copy land before the CTA can exit
      for (uint32_t t = (issued > PST ? issued - PST : 0); t < issued; ++t)
        mbar_wait_drain(&pk_full[t % PST], (t / PST) & 1u, &g_status);
    }
  } else if (warp == W_MMA) {
    if (lane == 0) {
      // ------------------------------------------------------------- MMA issuer
      uint32_t consumed = 0;
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++it) {
        const uint32_t b = it & 1, pb = (it >> 1) & 1;
        if (!mbar_wait(&acc_empty[b], pb ^ 1u, abort_flag, &g_status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + b * BN;
        for (int kb = 0; kb < num_kb; ++kb) {
          const uint32_t u = consumed % UST, pu = (consumed / UST) & 1u;
          if (!mbar_wait(&un_full[u], pu, abort_flag, &g_status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + OFF_A_UN + u * A_UN);
          const uint32_t b0 = smem_u32(smem + OFF_B_UN + u * B_UN);
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk)
            mma_i8(d_tmem, umma_desc_sw128(a0 + kk * 32), umma_desc_sw128(b0 + kk * 32), IDESC,
                   (kb | kk) != 0 ? 1u : 0u);
          tc_commit(&un_empty[u]);
          ++consumed;
        }
        if (ok) tc_commit(&acc_full[b]);
      }
      // every MMA issued must finish before tensor memory is freed
      tc_commit(mma_done);
      mbar_wait_drain(mma_done, 0, &g_status);
    }
  } else if (warp >= W_UNPACK0 && warp < W_UNPACK0 + 4) {
    // ------------------------------------------------------------------ unpack
    const int t = threadIdx.x - W_UNPACK0 * 32;
    uint32_t n = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      for (int kb = 0; kb < num_kb; ++kb, ++n) {
        const uint32_t s = n % PST, ps = (n / PST) & 1u;
        const uint32_t u = n % UST, pu = (n / UST) & 1u;
        if (!mbar_wait(&pk_full[s], ps, abort_flag, &g_status) || !mbar_wait(&un_empty[u], pu ^ 1u, abort_flag, &g_status)) {
          ok = false;
          break;
        }
        unpack_tile<A_PK / 16 / 128>(smem + OFF_A_PK + s * A_PK, smem + OFF_A_UN + u * A_UN, t);
        unpack_tile<B_PK / 16 / 128>(smem + OFF_B_PK + s * B_PK, smem + OFF_B_UN + u * B_UN, t);
        fence_proxy_async_smem();
        mbar_arrive(&pk_empty[s]);
        mbar_arrive(&un_full[u]);
      }
    }
  } else if (warp >= W_EPI0) {
    // ---------------------------------------------------------------- epilogue
    const int ew = warp - W_EPI0;  // == warp % 4: owns TMEM lanes 32 ew .. 32 ew + 31
    int it = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      const uint32_t b = it & 1, pb = (it >> 1) & 1;
      if (!mbar_wait(&acc_full[b], pb, abort_flag, &g_status)) break;
      tc_fence_after();
      const int mb = tile / num_n_tiles, nb = tile % num_n_tiles;
      const int row0 = mb * BM + ew * 32;
      const int m = row0 + lane;
      const float st = (!OUT_S32 && m < M) ? __ldg(scale_tok + m) : 0.0f;
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(ew * 32) << 16) + b * BN;
#pragma unroll 1
      for (int ch = 0; ch < BN / 32; ++ch) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tbase + ch * 32, r);
        tmem_wait_ld();
        if (ch == BN / 32 - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[b]);
        }
        const int n0 = nb * BN + ch * 32;
        if (OUT_S32) {
          if (m < M) {
            int4 *dst = reinterpret_cast<int4 *>(acc_out + static_cast<int64_t>(m) * N + n0);
#pragma unroll
            for (int c = 0; c < 8; ++c)
              dst[c] = make_int4(static_cast<int>(r[4 * c]), static_cast<int>(r[4 * c + 1]),
                                 static_cast<int>(r[4 * c + 2]), static_cast<int>(r[4 * c + 3]));
          }
        } else {
          uint32_t pk[16];
          const float4 *sc4 = reinterpret_cast<const float4 *>(scale_ch + n0);
          const float4 *bi4 = reinterpret_cast<const float4 *>(bias + n0);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const float4 sc = __ldg(sc4 + c), bi = __ldg(bi4 + c);
            const float y0 = fmaf(static_cast<float>(static_cast<int>(r[4 * c + 0])), st * sc.x, bi.x);
            const float y1 = fmaf(static_cast<float>(static_cast<int>(r[4 * c + 1])), st * sc.y, bi.y);
            const float y2 = fmaf(static_cast<float>(static_cast<int>(r[4 * c + 2])), st * sc.z, bi.z);
            const float y3 = fmaf(static_cast<float>(static_cast<int>(r[4 * c + 3])), st * sc.w, bi.w);
            pk[2 * c] = pack_bf16x2(y0, y1);
            pk[2 * c + 1] = pack_bf16x2(y2, y3);
          }
          uint8_t *stg = smem + OFF_EPI + (ew * 2 + (ch & 1)) * EPI_BYTES;
          if (lane == 0) bulk_wait_read<1>();  // the store that last read this buffer is done
          __syncwarp();
#pragma unroll
          for (int c = 0; c < 4; ++c)
            *reinterpret_cast<uint4 *>(stg + lane * 64 + ((c ^ ((lane >> 1) & 3)) << 4)) =
                make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && row0 < M) {
            tma_store_2d(&tmY, stg, n0, row0);
            bulk_commit();
          }
        }
      }
    }
    if (!OUT_S32 && lane == 0) bulk_wait<0>();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == W_TMEM) tmem_dealloc(tmem_base, TMEM_COLS);
}

// --------------------------------------------------------------- host side
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool make_map_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t inner,
                 uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                 CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool OUT_S32>
cudaError_t launch_t(const GemmArgs &a, cudaStream_t st) {
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(w4a4_gemm_kernel<OUT_S32>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  });
  if (attr_err != cudaSuccess) return attr_err;
  CUtensorMap tmA, tmB, tmY;
  const uint64_t kp = static_cast<uint64_t>(a.K / 2);
  if (!make_map_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.qx, kp, a.M, kp, BKP, BM,
                   CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_map_2d(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.qw, kp, a.N, kp, BKP, BN,
                   CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  if (OUT_S32) {
    tmY = tmA;  // unused
  } else if (!make_map_2d(&tmY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.y, a.N, a.M,
                          static_cast<uint64_t>(a.N) * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B)) {
    return cudaErrorInvalidValue;
  }
  const int num_m = static_cast<int>((a.M + BM - 1) / BM);
  const int num_n = a.N / BN;
  const int tiles = num_m * num_n;
  const int grid = tiles < device_sm_count() ? tiles : device_sm_count();
  w4a4_gemm_kernel<OUT_S32><<<grid, NUM_THREADS, SMEM_BYTES, st>>>(
      tmA, tmB, tmY, a.scale_tok, a.scale_ch, a.bias, a.acc, static_cast<int>(a.M), a.N, num_n,
      tiles, a.K / BK);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm(const GemmArgs &a, cudaStream_t st) {
  if (a.M <= 0) return cudaSuccess;
  return a.acc ? launch_t<true>(a, st) : launch_t<false>(a, st);
}

cudaError_t read_status(unsigned int *out, cudaStream_t st) {
  cudaError_t e = cudaMemcpyFromSymbolAsync(out, g_status, sizeof(unsigned int), 0,
                                            cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return e;
  return cudaStreamSynchronize(st);
}

cudaError_t clear_status(cudaStream_t st) {
  static const unsigned int zero = 0;
  return cudaMemcpyToSymbolAsync(g_status, &zero, sizeof(unsigned int), 0, cudaMemcpyHostToDevice, st);
}

}  // namespace w4a4
