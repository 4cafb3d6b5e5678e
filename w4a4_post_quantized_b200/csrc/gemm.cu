// gemm.cu -- the tensor-core half of the DSFQ W4A4 linear on sm_100a.
//
//   Y[m, n] = bf16( (sum_k qx[m, k] qw[n, k]) * scale_tok[m] * scale_ch[n] + bias[n] )
//
// qx [M, K/2] and qw [N, K/2] hold int4 codes packed two per byte (page
// "十亿参数的三维重建模型，能塞进手机吗？", section 训练后量化（PTQ）: symmetric
// 4-bit codes; section 细粒度量化粒度 read as per-token x per-channel steps).
// tcgen05 has no 4-bit integer MMA, so the int4 codes are widened to 8 bits
// and multiplied with tcgen05.mma kind::i8 (s32 accumulators in tensor
// memory).  Three ways of feeding the operands:
//
//   * expanded B (packed activation codes, weights that carry qw8): the weights
//     are static, so their int4 codes are widened once, at preparation time,
//     into qw8 [N, K] int8 in exactly the order the kernel widens A.  The
//     kernel TMA-loads B tiles straight into the 128-byte swizzled operand
//     layout.  A is TMA-staged packed; the widen warps turn each row into the
//     unsigned values code + 8 (a nibble XOR, 3 integer ops per 8 codes) in
//     registers and store them into tensor memory (tcgen05.st), and the MMA
//     reads A from there, so shared memory carries only the packed A and B.
//     sum_k (qa + 8) qb = acc + 8 * colsum[n], so the epilogue subtracts
//     8 * colsum[n] (colsum = per-output-channel sum of the weight codes,
//     prepared with qw8).  The result is exact.  Tiles are 128 x 192 (the
//     last column tile of an N that is not a multiple of 192 is partly
//     outside the matrix: TMA fills those B rows with zeros and clips the
//     stores).
//   * packed B (qw8 == NULL): both operands are TMA-staged packed and
//     sign-extended to int8 in shared memory on every tile (no extra weight
//     memory, more shared-memory traffic and integer work); tiles 128 x 256.
//   * bytes (a8): activations and weights carry one code per byte in the
//     same order: the int4 codes the quantize kernel writes one per byte in
//     qw8's operand order (the fused call's default route), or the W8A8
//     setting's 8-bit codes in natural order.  TMA loads both straight into
//     the 128-byte swizzled operand layout and the MMA reads them there
//     (signed x signed); no widening at all.  With enough tiles a cluster of
//     two CTAs shares a 256 x 256 tile (cta_group::2: each CTA loads its 128
//     rows of A and of B, the leader issues the MMAs, each CTA drains its own
//     128 rows); small shapes take 128 x 128 tiles of one CTA.
//
// Warp roles (one persistent CTA, or CTA pair, per SM, tiles round-robin, M-major):
//   warp 0      TMA producer (one thread)
//   warp 1      tcgen05.mma issuer (one thread)
//   warp 2      tensor-memory allocator
//   warps 4..7  widen packed int4 -> int8 (into tensor memory, or into the
//               swizzled shared-memory operand tiles of the packed-B path);
//               with byte operands, a second epilogue warp per lane quadrant
//               when the GELU is on the output or the CTAs work in pairs
//   warps 8..11 epilogue: tcgen05.ld accumulators (64 columns at a time),
//               subtract the code-offset term, scale by scale_tok[m] *
//               scale_ch[n], add bias in fp32, round to bf16, TMA-store
//               32 x 64 tiles through a 128-byte-swizzled staging buffer.
//               The expanded-B path loads the accumulators in the 16x256b
//               fragment layout (each thread: 4 rows, 2 of every 8 columns),
//               so a thread reads only its own columns' constants (8-byte
//               loads instead of 16-byte broadcasts of every column, which
//               kept the shared-memory pipe busy), and writes the bf16 pairs
//               with stmatrix.
// Accumulators are double-buffered in tensor memory so the epilogue of one
// tile overlaps the main loop of the next.
//
// Widening permutes K inside every group of 8 codes (even codes first, then
// odd ones).  A and B use the same order, so every dot product sums the same
// pairs and the integer result is unchanged.
//
// Every wait is bounded (ptx.cuh): a stuck pipeline sets the device status
// word and the CTA drains its in-flight copies and MMAs, frees its tensor
// memory and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "ctxcache.h"
#include "gelu.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace w4a4 {

// Device status word (bits W4A4_DEV_* of include/w4a4.h): the only state the
// library keeps between calls.
__device__ unsigned int g_status = 0;

namespace {

constexpr int BM = 128;   // tile rows (tokens)
constexpr int BN = 256;   // tile columns (output channels) of the packed-B path
constexpr int BK = 128;   // int8 elements per k-block = one 128-byte swizzle row
constexpr int BKP = 64;   // packed bytes per row per k-block
constexpr int A_PK = BM * BKP;   // 8 KB
constexpr int B_PK = BN * BKP;   // 16 KB
constexpr int A_UN = BM * BK;    // 16 KB
constexpr int B_UN = BN * BK;    // 32 KB
constexpr int EPI_COLS = 64;             // output columns per epilogue store
constexpr int EPI_BYTES = 32 * EPI_COLS * 2;  // one warp's 32 x 64 bf16 staging tile (128-byte rows)
constexpr int NUM_EPI_WARPS = 4;        // one per TMEM lane quadrant
constexpr int NUM_THREADS = (8 + NUM_EPI_WARPS) * 32;
constexpr uint32_t TMEM_COLS = 512;     // the whole tensor memory of the SM

// Shared-memory and tensor-memory plan.  TMA stages hold what comes from L2
// (A packed or int8, B int8 or packed).
//   expanded B: A is widened into tensor memory (the MMA reads A there), so
//     shared memory carries only B and the packed A.  Tiles are 128 x 192:
//     two 192-column accumulators and two widened-A slots of KG k-blocks
//     (32 columns each) fill the 512 columns.
//   packed B: A and B are widened into a ring of shared-memory slots; tiles
//     are 128 x 256.
//   int8: A and B arrive as int8 operand tiles; tiles are 128 x 256, two
//     256-column accumulators.  The narrow variant (128 x 128 tiles, 6 stages
//     of 32 KB) serves shapes whose 128 x 256 tiles would leave more than
//     half of the SMs idle (a single frame: 44 tiles), doubling the tiles.
//   int8 pair: the same operands for a CTA pair (a cluster of 2) sharing a
//     256 x 256 tile: each CTA loads its 128 rows of A and 128 rows of B
//     (6 stages of 32 KB), the leader issues cta_group::2 MMAs that read both
//     CTAs' halves, and each CTA's tensor memory holds its 128 rows x 256
//     columns (two buffers), drained by its own epilogue.  Per multiply-add a
//     CTA loads and the tensor cores read a third less shared memory than a
//     128 x 256 tile of one CTA, and the same stage bytes cover 1.5x the time.
//     The pair synchronises through barriers at CTA scope (the other CTA's
//     arrivals publish completed tensor-memory reads, the copies and MMAs
//     complete through their own mechanisms): cluster-scope release /
//     acquire on those waits and arrivals made the pair slower than one CTA
//     per tile wherever the epilogue bounds the kernel (K = 1024).
enum : int { kExpanded = 0, kPacked = 1, kInt8 = 2, kInt8Narrow = 3, kInt8Pair = 4 };

template <int MODE>
struct Plan {
  static constexpr bool B_PACKED = MODE == kPacked;
  static constexpr bool A_TMEM = MODE == kExpanded;
  static constexpr bool NARROW = MODE == kInt8Narrow;
  static constexpr bool PAIR = MODE == kInt8Pair;
  static constexpr bool A8 = MODE == kInt8 || NARROW || PAIR;  // both operands one code per byte
  static constexpr bool EPI16 = !B_PACKED;           // 16x256b epilogue fragments
  static constexpr int TN = A_TMEM ? 192 : (NARROW ? 128 : BN);  // tile columns
  static constexpr int TNL = PAIR ? TN / 2 : TN;     // B rows a CTA loads
  static constexpr int TM = PAIR ? 2 * BM : BM;      // tile rows (of the pair)
  static constexpr int STAGES = B_PACKED ? 3 : ((NARROW || PAIR) ? 6 : (A8 ? 4 : 5));  // TMA stages
  // staging buffers (32 x 64 bf16) per epilogue lane quadrant (a CTA pair's
  // eight epilogue warps take one each: 6 stages and 2 buffers measured 3 %
  // faster on the K = 1024 layers than 5 and 4)
  static constexpr int EPI_NB = 2;
  static constexpr int KG = A_TMEM ? 2 : 1;          // k-blocks per widen -> MMA handshake
  static constexpr int WSLOTS = A8 ? 0 : 2;          // widened operand slots
  static constexpr int A_ST = A8 ? A_UN : A_PK;      // A bytes of a stage
  static constexpr int OFF_ST_A = 0;                 // A: packed [BM x 64 B] or int8 [BM x 128 B] (swizzled)
  static constexpr int OFF_ST_B = A_ST;              // B: int8 [TN x 128 B] (swizzled) or packed
  static constexpr int STAGE_BYTES = A_ST + (B_PACKED ? B_PK : TNL * BK);
  static constexpr int OFF_W = STAGES * STAGE_BYTES;
  static constexpr int OFF_W_A = 0;                  // widened A [BM x 128 B] (swizzled)
  static constexpr int OFF_W_B = A_UN;               // widened B (B_PACKED only)
  static constexpr int WSLOT_BYTES = B_PACKED ? A_UN + B_UN : 0;
  static constexpr uint32_t TMEM_A0 = 2 * TN;        // first widened-A column (A_TMEM)
  static_assert(!A_TMEM || TMEM_A0 + WSLOTS * KG * 32 <= 512, "tensor-memory budget");
  static constexpr int OFF_EPI = OFF_W + WSLOTS * WSLOT_BYTES;
  static constexpr int OFF_COL = OFF_EPI + NUM_EPI_WARPS * EPI_NB * EPI_BYTES;  // per-warp constants
  static constexpr int COL_WORDS = A8 ? 0 : 3 * TN;  // (int8: no code offset, no table)
  static constexpr int OFF_BAR = OFF_COL + NUM_EPI_WARPS * COL_WORDS * 4;
  static constexpr int NUM_BARS = 2 * STAGES + 2 * (WSLOTS > 0 ? WSLOTS : 1) + 2 * 2 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + slack to align the base to 1024
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(OFF_ST_B % 1024 == 0 && STAGE_BYTES % 1024 == 0 && OFF_W % 1024 == 0 &&
                    WSLOT_BYTES % 1024 == 0 && OFF_EPI % 1024 == 0,
                "swizzled tiles need 1024-byte alignment");
  // tcgen05.mma kind::i8 instruction descriptor: s32 D; A unsigned (code + 8)
  // with expanded B, signed otherwise; B signed; both K-major; TM x TN.
  static constexpr uint32_t IDESC = (2u << 4) | ((A_TMEM ? 0u : 1u) << 7) | (1u << 10) |
                                    (static_cast<uint32_t>(TN >> 3) << 17) |
                                    (static_cast<uint32_t>(TM >> 4) << 24);
};

constexpr int W_TMA = 0, W_MMA = 1, W_TMEM = 2;
constexpr int W_UNPACK0 = 4;  // warps 4..7
constexpr int W_EPI0 = 8;     // warps 8..11: warp % 4 selects its 32 TMEM lanes

// 4 nibbles (one per byte, 0..15 = two's-complement int4) -> 4 signed int8.
__device__ __forceinline__ uint32_t sext4x4(uint32_t n) {
  return ((n ^ 0x08080808u) + 0x78787878u) ^ 0x80808080u;
}

// Widen a 16-byte packed chunk (32 codes) to two 16-byte chunks.  Word t
// holds codes 8t..8t+7; its even codes go first, then its odd codes.
// SIGNED: two's-complement int8; otherwise the unsigned value code + 8.
template <bool SIGNED>
__device__ __forceinline__ void widen_chunk(uint4 v, uint4 &o0, uint4 &o1) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[8];
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const uint32_t lo = w[t] & 0x0F0F0F0Fu, hi = (w[t] >> 4) & 0x0F0F0F0Fu;
    o[2 * t] = SIGNED ? sext4x4(lo) : (lo ^ 0x08080808u);
    o[2 * t + 1] = SIGNED ? sext4x4(hi) : (hi ^ 0x08080808u);
  }
  o0 = make_uint4(o[0], o[1], o[2], o[3]);
  o1 = make_uint4(o[4], o[5], o[6], o[7]);
}

// Widen NCH packed chunks of a tile (rows of 64 packed bytes) into the
// 128-byte swizzled int8 tile.  Chunk q covers row q/4, codes 32(q%4)..+31.
template <int NCH, bool SIGNED>
__device__ __forceinline__ void widen_tile(const uint8_t *__restrict__ src, uint8_t *__restrict__ dst,
                                           int t) {
  uint4 v[NCH];
#pragma unroll
  for (int i = 0; i < NCH; ++i) v[i] = *reinterpret_cast<const uint4 *>(src + (t + 128 * i) * 16);
#pragma unroll
  for (int i = 0; i < NCH; ++i) {
    const int q = t + 128 * i;
    const int r = q >> 2, c = q & 3;
    uint4 o0, o1;
    widen_chunk<SIGNED>(v[i], o0, o1);
    uint8_t *row = dst + r * 128;
    *reinterpret_cast<uint4 *>(row + (((2 * c) ^ (r & 7)) << 4)) = o0;
    *reinterpret_cast<uint4 *>(row + (((2 * c + 1) ^ (r & 7)) << 4)) = o1;
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&h);
}

// Packed fp32x2 arithmetic of sm_100 (each lane rounded as the scalar op).
__device__ __forceinline__ unsigned long long f2_pack(float lo, float hi) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(unsigned long long v, float &lo, float &hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

// Dequantize two accumulators given as biased bit patterns (0x4B400000 + acc,
// i.e. the floats 1.5 * 2^23 + acc, exact for |acc| < 2^22):
//   y = (float(bits) - 1.5 * 2^23) * (st * sc) + bias, all in fp32.
__device__ __forceinline__ uint32_t dequant2_bf16(int32_t b0, int32_t b1, float st, float sc0,
                                                  float sc1, float bi0, float bi1) {
  const unsigned long long x = f2_pack(__int_as_float(b0), __int_as_float(b1));
  const unsigned long long magic = f2_pack(12582912.0f, 12582912.0f);
  const unsigned long long s = f2_pack(st, st), c = f2_pack(sc0, sc1), b = f2_pack(bi0, bi1);
  unsigned long long a, m, y;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(a) : "l"(x), "l"(magic));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(m) : "l"(s), "l"(c));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(y) : "l"(a), "l"(m), "l"(b));
  float y0, y1;
  f2_unpack(y, y0, y1);
  return pack_bf16x2(y0, y1);
}

// The same for plain accumulators of any size (8-bit codes reach 127^2 K,
// beyond the 2^22 the biased bit pattern above can hold): converted with
// round-to-nearest (exact up to 2^24; the relative error stays below 2^-24).
__device__ __forceinline__ uint32_t dequant2_bf16_cvt(int32_t a0, int32_t a1, float st, float sc0,
                                                      float sc1, float bi0, float bi1) {
  const unsigned long long x = f2_pack(__int2float_rn(a0), __int2float_rn(a1));
  const unsigned long long s = f2_pack(st, st), c = f2_pack(sc0, sc1), b = f2_pack(bi0, bi1);
  unsigned long long m, y;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(m) : "l"(s), "l"(c));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(y) : "l"(x), "l"(m), "l"(b));
  float y0, y1;
  f2_unpack(y, y0, y1);
  return pack_bf16x2(y0, y1);
}

template <int MODE, bool OUT_S32, bool GELU_OUT = false, bool ACC22 = false>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    w4a4_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmY, const float *__restrict__ scale_tok,
                     const float *__restrict__ scale_ch, const float *__restrict__ bias,
                     const int32_t *__restrict__ colsum, int32_t *__restrict__ acc_out, int M, int N,
                     int num_n_tiles, int num_tiles, int num_kb, uint32_t stall,
                     unsigned long long wait_ns) {
  using P = Plan<MODE>;
  constexpr bool B_PACKED = P::B_PACKED;
  constexpr int ST = P::STAGES;
  constexpr int WS = P::WSLOTS > 0 ? P::WSLOTS : 1;  // (int8: barriers unused)
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + P::OFF_BAR);
  uint64_t *full = bars;             // TMA bytes of a stage landed
  uint64_t *freed = full + ST;       // MMAs reading a stage completed
  uint64_t *wready = freed + ST;     // widened slot written (one arrival per widen warp)
  uint64_t *wfree = wready + WS;     // MMAs reading a widened slot completed
  uint64_t *acc_full = wfree + WS;   // accumulator buffer complete
  uint64_t *acc_empty = acc_full + 2;  // epilogue drained an accumulator buffer
  uint64_t *mma_done = acc_empty + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + P::OFF_MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + P::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // a CTA pair works on the pair's tiles; rank 0 (the leader) issues the MMAs
  constexpr bool PAIR = P::PAIR;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const int unit0 = PAIR ? static_cast<int>(cluster_id_x()) : static_cast<int>(blockIdx.x);
  const int units = PAIR ? static_cast<int>(nclusters_x()) : static_cast<int>(gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&freed[s], 1);
    }
    for (int u = 0; u < WS; ++u) {
      mbar_init(&wready[u], 4);
      mbar_init(&wfree[u], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      // (a pair's leader counts the epilogue warps of both CTAs)
      mbar_init(&acc_empty[b], ((GELU_OUT || PAIR) && P::A8 ? 2 : 1) * NUM_EPI_WARPS * (PAIR ? 2 : 1));
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
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // TPRE (byte operands, small accumulators): every accumulator starts at the
  // bit pattern of the float 1.5 * 2^23 and the MMAs always accumulate, so an
  // accumulator's bits are the float 1.5 * 2^23 + acc (exact below 2^22) and
  // the epilogue needs no integer add; each epilogue warp refills what it
  // has read before it frees the buffer.  Here the epilogue warps fill both
  // buffers of their lane quadrant once.
  constexpr bool TPRE = ACC22 && P::A8 && !OUT_S32;
  if constexpr (TPRE) {
    constexpr bool E8 = (GELU_OUT || PAIR) && P::A8;
    if (warp >= W_EPI0 || (E8 && warp >= W_UNPACK0)) {
      const int cols_per_warp = E8 ? P::TN : 2 * P::TN;          // E8: each warp one buffer
      const uint32_t c0 = E8 ? (warp >= W_EPI0 ? 0u : static_cast<uint32_t>(P::TN)) : 0u;
      const uint32_t lanes = static_cast<uint32_t>((warp & 3) * 32) << 16;
      for (int c = 0; c < cols_per_warp; c += 32) tmem_fill_32x32b_x32(tmem_base + lanes + c0 + c, 0x4B400000u);
      tmem_wait_st();
    }
  }
  tc_fence_before();
  __syncthreads();
  // (a pair: both CTAs' barriers exist, and both tensor memories are filled,
  // before either CTA signals the other or the leader's MMAs write them)
  if constexpr (PAIR) cluster_sync();
  tc_fence_after();
  // Everything above (barriers, tensor memory, descriptor prefetch) may overlap
  // the tail of the kernel that produced qx and scale_tok; from here on this
  // CTA reads what earlier kernels wrote.
  griddep_launch_dependents();
  griddep_wait();

  if (warp == W_TMA) {
    if (lane == 0) {
      // ---------------------------------------------------------------- producer
      uint32_t issued = 0;
      bool ok = true;
      // stall (a test of the failure path, w4a4_gemm_s32_ex with W4A4_DEBUG_STALL):
      // no copy is ever issued, so the consumers' first waits run out
      for (int tile = unit0; tile < num_tiles && ok && !stall; tile += units) {
        const int mb = tile / num_n_tiles, nb = tile % num_n_tiles;
        for (int kb = 0; kb < num_kb; ++kb) {
          const uint32_t s = issued % ST, ph = (issued / ST) & 1u;
          if (!mbar_wait(&freed[s], ph ^ 1u, abort_flag, &g_status, wait_ns)) {
            ok = false;
            break;
          }
          uint8_t *stage = smem + s * P::STAGE_BYTES;
          if constexpr (PAIR) {
            // both CTAs' bytes land on the leader's barrier, which the leader arms
            if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * P::STAGE_BYTES);
            const uint32_t bar0 = cluster_addr(&full[s], 0);
            tma_load_2d_pair(stage + P::OFF_ST_A, &tmA, kb * BK, mb * P::TM + static_cast<int>(rank) * BM,
                             bar0);
            tma_load_2d_pair(stage + P::OFF_ST_B, &tmB, kb * BK,
                             nb * P::TN + static_cast<int>(rank) * P::TNL, bar0);
          } else {
            mbar_arrive_expect_tx(&full[s], P::STAGE_BYTES);
            tma_load_2d(stage + P::OFF_ST_A, &tmA, P::A8 ? kb * BK : kb * BKP, mb * BM, &full[s]);
            tma_load_2d(stage + P::OFF_ST_B, &tmB, B_PACKED ? kb * BKP : kb * BK, nb * P::TN, &full[s]);
          }
          ++issued;
        }
      }
      // let every issued copy land before the CTA can exit (a pair's copies
      // complete on the leader's barriers: the leader waits for both CTAs',
      // and the closing cluster barrier holds the other CTA until then)
      if (!PAIR || rank == 0)
        for (uint32_t t = (issued > ST ? issued - ST : 0); t < issued; ++t)
          mbar_wait_drain(&full[t % ST], (t / ST) & 1u, &g_status, wait_ns);
    }
  } else if (warp == W_MMA) {
    if (lane == 0 && rank == 0) {
      // ------------------------------------------------------------- MMA issuer
      uint32_t consumed = 0, group = 0;
      int it = 0;
      bool ok = true;
      for (int tile = unit0; tile < num_tiles && ok; tile += units, ++it) {
        const uint32_t b = it & 1, pb = (it >> 1) & 1;
        if (!mbar_wait(&acc_empty[b], pb ^ 1u, abort_flag, &g_status, wait_ns)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + b * P::TN;
        if constexpr (P::A_TMEM) {
          // one handshake per group of KG k-blocks: widened A of the group in
          // slot u, B of each k-block in its TMA stage
          for (int kb = 0; kb < num_kb; kb += P::KG, ++group) {
            const uint32_t u = group % WS, pu = (group / WS) & 1u;
            if (!mbar_wait(&wready[u], pu, abort_flag, &g_status, wait_ns)) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int j = 0; j < P::KG; ++j) {
              const uint32_t s = consumed % ST;
              const uint32_t b0 = smem_u32(smem + s * P::STAGE_BYTES + P::OFF_ST_B);
              const uint32_t ta = tmem_base + P::TMEM_A0 + (u * P::KG + j) * 32;
#pragma unroll
              for (int kk = 0; kk < BK / 32; ++kk)
                mma_i8_ta(d_tmem, ta + kk * 8, umma_desc_sw128(b0 + kk * 32), P::IDESC,
                          ((kb + j) | kk) != 0 ? 1u : 0u);
              tc_commit(&freed[s]);
              ++consumed;
            }
            tc_commit(&wfree[u]);
          }
        } else if constexpr (P::A8) {
          // both operands straight from the TMA stage
          for (int kb = 0; kb < num_kb; ++kb) {
            const uint32_t s = consumed % ST, ps = (consumed / ST) & 1u;
            if (!mbar_wait(&full[s], ps, abort_flag, &g_status, wait_ns)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t a0 = smem_u32(smem + s * P::STAGE_BYTES + P::OFF_ST_A);
            const uint32_t b0 = smem_u32(smem + s * P::STAGE_BYTES + P::OFF_ST_B);
#pragma unroll
            for (int kk = 0; kk < BK / 32; ++kk) {
              // (TPRE: the accumulators start at the float bias, always accumulate)
              if constexpr (PAIR)
                mma_i8_pair(d_tmem, umma_desc_sw128(a0 + kk * 32), umma_desc_sw128(b0 + kk * 32),
                            P::IDESC, (TPRE || (kb | kk) != 0) ? 1u : 0u);
              else
                mma_i8(d_tmem, umma_desc_sw128(a0 + kk * 32), umma_desc_sw128(b0 + kk * 32), P::IDESC,
                       (TPRE || (kb | kk) != 0) ? 1u : 0u);
            }
            if constexpr (PAIR)
              tc_commit_pair(&freed[s], 0x3);  // frees the stage in both CTAs
            else
              tc_commit(&freed[s]);
            ++consumed;
          }
        } else {
          for (int kb = 0; kb < num_kb; ++kb) {
            const uint32_t s = consumed % ST;
            const uint32_t u = consumed % WS, pu = (consumed / WS) & 1u;
            // the widen warps waited for the stage's TMA bytes before signalling wready
            if (!mbar_wait(&wready[u], pu, abort_flag, &g_status, wait_ns)) {
              ok = false;
              break;
            }
            tc_fence_after();
            uint8_t *slot = smem + P::OFF_W + u * P::WSLOT_BYTES;
            const uint32_t a0 = smem_u32(slot + P::OFF_W_A);
            const uint32_t b0 = smem_u32(slot + P::OFF_W_B);
#pragma unroll
            for (int kk = 0; kk < BK / 32; ++kk)
              mma_i8(d_tmem, umma_desc_sw128(a0 + kk * 32), umma_desc_sw128(b0 + kk * 32), P::IDESC,
                     (kb | kk) != 0 ? 1u : 0u);
            tc_commit(&freed[s]);
            tc_commit(&wfree[u]);
            ++consumed;
          }
        }
        if (ok) {
          if constexpr (PAIR)
            tc_commit_pair(&acc_full[b], 0x3);
          else
            tc_commit(&acc_full[b]);
        }
      }
      // every MMA issued must finish before tensor memory is freed (a pair's
      // commit is only issued after pair MMAs: with none, nothing is pending)
      if constexpr (PAIR) {
        if (consumed > 0) {
          tc_commit_pair(mma_done, 0x1);
          mbar_wait_drain(mma_done, 0, &g_status, wait_ns);
        }
      } else {
        tc_commit(mma_done);
        mbar_wait_drain(mma_done, 0, &g_status, wait_ns);
      }
    }
  } else if (!P::A8 && warp >= W_UNPACK0 && warp < W_UNPACK0 + 4) {
    // ------------------------------------------------------------------ widen
    const int t = threadIdx.x - W_UNPACK0 * 32;
    uint32_t n = 0;
    bool ok = true;
    if constexpr (P::A_TMEM) {
      // this warp writes tensor-memory lanes 32 (warp % 4) .. + 31 (its lane quadrant)
      uint32_t grp = 0;
      const uint32_t tq = tmem_base + (static_cast<uint32_t>((warp & 3) * 32) << 16) + P::TMEM_A0;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        for (int kb = 0; kb < num_kb && ok; kb += P::KG, ++grp) {
          const uint32_t u = grp % WS, pu = (grp / WS) & 1u;
          if (!mbar_wait(&wfree[u], pu ^ 1u, abort_flag, &g_status, wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();  // the MMAs that read slot u completed
#pragma unroll 1
          for (int j = 0; j < P::KG; ++j, ++n) {
            const uint32_t s = n % ST, ps = (n / ST) & 1u;
            if (!mbar_wait(&full[s], ps, abort_flag, &g_status, wait_ns)) {
              ok = false;
              break;
            }
            // tile row t: its 64 packed bytes (64-byte swizzled rows: 16-byte
            // chunk c at c ^ ((row / 2) % 4)) -> 128 values code + 8 -> 32
            // tensor-memory columns of lane t
            const uint8_t *src = smem + s * P::STAGE_BYTES + P::OFF_ST_A + t * 64;
            uint32_t o[32];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const uint4 v = *reinterpret_cast<const uint4 *>(src + ((c ^ ((t >> 1) & 3)) << 4));
              uint4 o0, o1;
              widen_chunk<false>(v, o0, o1);
              o[8 * c + 0] = o0.x;
              o[8 * c + 1] = o0.y;
              o[8 * c + 2] = o0.z;
              o[8 * c + 3] = o0.w;
              o[8 * c + 4] = o1.x;
              o[8 * c + 5] = o1.y;
              o[8 * c + 6] = o1.z;
              o[8 * c + 7] = o1.w;
            }
            tmem_st_32x32b_x32(tq + (u * P::KG + j) * 32, o);
          }
          if (!ok) {
            tmem_wait_st();
            break;
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&wready[u]);
        }
      }
    } else if constexpr (P::B_PACKED) {
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        for (int kb = 0; kb < num_kb; ++kb, ++n) {
          const uint32_t s = n % ST, ps = (n / ST) & 1u;
          const uint32_t u = n % WS, pu = (n / WS) & 1u;
          if (!mbar_wait(&full[s], ps, abort_flag, &g_status, wait_ns) ||
              !mbar_wait(&wfree[u], pu ^ 1u, abort_flag, &g_status, wait_ns)) {
            ok = false;
            break;
          }
          uint8_t *stage = smem + s * P::STAGE_BYTES;
          uint8_t *slot = smem + P::OFF_W + u * P::WSLOT_BYTES;
          widen_tile<A_PK / 16 / 128, true>(stage + P::OFF_ST_A, slot + P::OFF_W_A, t);
          widen_tile<B_PK / 16 / 128, true>(stage + P::OFF_ST_B, slot + P::OFF_W_B, t);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&wready[u]);
        }
      }
    }
  } else if (warp >= W_EPI0 || ((GELU_OUT || P::PAIR) && P::A8 && warp >= W_UNPACK0 && warp < W_UNPACK0 + 4)) {
    // ---------------------------------------------------------------- epilogue
    const int ew = warp & 3;  // owns TMEM lanes 32 ew .. 32 ew + 31
    // With the GELU on the output (the epilogue's ALU work then exceeds the
    // main loop's time), and in a CTA pair, the byte-operand mode's idle warps
    // 4..7 join in: the two warps of a lane quadrant take half of the tile's
    // columns each, with one staging buffer each.
    constexpr bool EPI8 = (GELU_OUT || P::PAIR) && P::A8;
    const int half = (EPI8 && warp < W_EPI0) ? 1 : 0;
    constexpr int SC_PER = EPI8 ? P::TN / EPI_COLS / 2 : P::TN / EPI_COLS;
    // this warp's copy of the tile's per-column constants:
    //   off[n] = 0x4B400000 - 8 colsum[n] (the code-offset correction folded
    //   into the exact int -> float bias), sc[n], bias[n]
    constexpr int TN = P::TN;
    int32_t *coff = reinterpret_cast<int32_t *>(smem + P::OFF_COL) + ew * P::COL_WORDS;
    float *csc = reinterpret_cast<float *>(coff + TN);
    float *cbi = csc + TN;
    int it = 0;
    for (int tile = unit0; tile < num_tiles; tile += units, ++it) {
      const uint32_t b = it & 1, pb = (it >> 1) & 1;
      const int mb = tile / num_n_tiles, nb = tile % num_n_tiles;
      __syncwarp();  // every lane is done reading the previous tile's constants
#pragma unroll
      for (int j = lane; j < (((!OUT_S32 && P::EPI16) || P::A8) ? 0 : TN); j += 32) {
        const int n = nb * TN + j;
        const bool in = n < N;  // the last tile of a ragged N
        coff[j] = 0x4B400000 - ((B_PACKED || !in) ? 0 : 8 * __ldg(colsum + n));
        if (!OUT_S32) {
          csc[j] = in ? __ldg(scale_ch + n) : 0.0f;
          cbi[j] = in ? __ldg(bias + n) : 0.0f;
        }
      }
      __syncwarp();
      if (!mbar_wait(&acc_full[b], pb, abort_flag, &g_status, wait_ns)) break;
      tc_fence_after();
      const int row0 = mb * P::TM + static_cast<int>(rank) * BM + ew * 32;
      if constexpr (!OUT_S32 && P::EPI16) {
        // 16x256b fragments: thread t holds rows q = t/4 + 8 i (i < 4) of the
        // warp's 32 rows and, per 8-column group j, columns 8j + 2(t%4) + {0,1};
        // its columns' constants are 8-byte loads, and the bf16 pairs go to the
        // staging tile with stmatrix (one 8 x 8 block per register)
        const int tq = lane >> 2, tc = 2 * (lane & 3);
        float st4[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int m = row0 + tq + 8 * i;
          st4[i] = m < M ? __ldg(scale_tok + m) : 0.0f;
        }
        const uint32_t tbase = tmem_base + (static_cast<uint32_t>(ew * 32) << 16) + b * TN;
#pragma unroll 1
        for (int sc = half * SC_PER; sc < (half + 1) * SC_PER; ++sc) {
          uint32_t r[2][32];  // [16-row half][4 j + k]
          tmem_ld_16x256b_x8(tbase + sc * EPI_COLS, r[0]);
          tmem_ld_16x256b_x8(tbase + (16u << 16) + sc * EPI_COLS, r[1]);
          tmem_wait_ld();
          if constexpr (TPRE) {  // the columns just read start the buffer's next tile at the bias
            tmem_fill_32x32b_x32(tbase + sc * EPI_COLS, 0x4B400000u);
            tmem_fill_32x32b_x32(tbase + sc * EPI_COLS + 32, 0x4B400000u);
          }
          if (sc == (half + 1) * SC_PER - 1) {
            if constexpr (TPRE) tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
              if constexpr (PAIR)
                mbar_arrive_cluster(&acc_empty[b], 0);  // the leader's barrier
              else
                mbar_arrive(&acc_empty[b]);
            }
          }
          const int c0 = sc * EPI_COLS;
          const int n0 = nb * TN + c0;
          uint32_t pk[2][2][8];  // [half][row sub-block][j]: bf16 pair of (row, columns 8j + tc + {0,1})
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int n = nb * TN + c0 + 8 * j + tc;  // N is even: the pair is all in or all out
            int2 o = TPRE ? make_int2(0, 0) : make_int2(0x4B400000, 0x4B400000);
            float2 scl = make_float2(0.0f, 0.0f), bi = make_float2(0.0f, 0.0f);
            if (n < N) {
              if constexpr (P::A_TMEM) {
                const int2 cs2 = __ldg(reinterpret_cast<const int2 *>(colsum + n));
                o = make_int2(0x4B400000 - 8 * cs2.x, 0x4B400000 - 8 * cs2.y);
              }
              scl = __ldg(reinterpret_cast<const float2 *>(scale_ch + n));
              bi = __ldg(reinterpret_cast<const float2 *>(bias + n));
            }
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
              for (int u = 0; u < 2; ++u)
                pk[h][u][j] =
                    (P::A8 && !ACC22) ? dequant2_bf16_cvt(static_cast<int32_t>(r[h][4 * j + 2 * u]),
                                              static_cast<int32_t>(r[h][4 * j + 2 * u + 1]),
                                              st4[2 * h + u], scl.x, scl.y, bi.x, bi.y)
                          : dequant2_bf16(static_cast<int32_t>(r[h][4 * j + 2 * u]) + o.x,
                                          static_cast<int32_t>(r[h][4 * j + 2 * u + 1]) + o.y,
                                          st4[2 * h + u], scl.x, scl.y, bi.x, bi.y);
          }
          if constexpr (GELU_OUT) {
            // the MLP's activation on the rounded output (bf16 in, bf16 out)
#pragma unroll
            for (int j = 0; j < 8; ++j)
#pragma unroll
              for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int u = 0; u < 2; ++u) pk[h][u][j] = gelu_pair_bf16(pk[h][u][j]);
          }
          // this warp's staging buffers: a quadrant's EPI_NB, split between its
          // two warps when eight share the epilogue
          constexpr int NBW = EPI8 ? P::EPI_NB / 2 : P::EPI_NB;
          uint8_t *stg = smem + P::OFF_EPI + ((ew * P::EPI_NB) + (EPI8 ? half * NBW : 0) + (sc % NBW)) * EPI_BYTES;
          if (lane == 0) bulk_wait_read<NBW - 1>();  // the store that last read this buffer is done
          __syncwarp();
          // staging tile: 32 rows of 128 bytes, 16-byte chunk k of row R at k ^ (R % 8);
          // stmatrix x4 #(h, jp): matrices (u, j) = (0, 2jp), (1, 2jp), (0, 2jp+1), (1, 2jp+1)
          const int mi = lane >> 3, mr = lane & 7;
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int jp = 0; jp < 4; ++jp) {
              const int row = 16 * h + 8 * (mi & 1) + mr;
              const int chunk = 2 * jp + (mi >> 1);
              stmatrix_x4(smem_u32(stg + row * 128 + ((chunk ^ (row & 7)) << 4)), pk[h][0][2 * jp],
                          pk[h][1][2 * jp], pk[h][0][2 * jp + 1], pk[h][1][2 * jp + 1]);
            }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && row0 < M && n0 < N) {
            tma_store_2d(&tmY, stg, n0, row0);
            bulk_commit();
          }
        }
        continue;
      }
      const int m = row0 + lane;
      const float st = (!OUT_S32 && m < M) ? __ldg(scale_tok + m) : 0.0f;
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(ew * 32) << 16) + b * TN;
#pragma unroll 1
      for (int sc = 0; sc < TN / EPI_COLS; ++sc) {
        // 64 accumulator columns of this warp's 32 rows: two loads, one wait
        uint32_t r[64];
        tmem_ld_32x32b_x32(tbase + sc * EPI_COLS, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
        tmem_ld_32x32b_x32(tbase + sc * EPI_COLS + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
        tmem_wait_ld();
        if (sc == TN / EPI_COLS - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if constexpr (PAIR)
              mbar_arrive_cluster(&acc_empty[b], 0);
            else
              mbar_arrive(&acc_empty[b]);
          }
        }
        const int c0 = sc * EPI_COLS;
        const int n0 = nb * TN + c0;
        const int4 *off4 = reinterpret_cast<const int4 *>(coff + c0);
        if (OUT_S32) {
          if (m < M && n0 < N) {
            int4 *dst = reinterpret_cast<int4 *>(acc_out + static_cast<int64_t>(m) * N + n0);
#pragma unroll
            for (int c = 0; c < EPI_COLS / 4; ++c) {
              const int4 o = P::A8 ? make_int4(0x4B400000, 0x4B400000, 0x4B400000, 0x4B400000) : off4[c];
              dst[c] = make_int4(static_cast<int32_t>(r[4 * c + 0]) + o.x - 0x4B400000,
                                 static_cast<int32_t>(r[4 * c + 1]) + o.y - 0x4B400000,
                                 static_cast<int32_t>(r[4 * c + 2]) + o.z - 0x4B400000,
                                 static_cast<int32_t>(r[4 * c + 3]) + o.w - 0x4B400000);
            }
          }
        } else {
          uint32_t pk[EPI_COLS / 2];
          const float4 *sc4 = reinterpret_cast<const float4 *>(csc + c0);
          const float4 *bi4 = reinterpret_cast<const float4 *>(cbi + c0);
#pragma unroll
          for (int c = 0; c < EPI_COLS / 4; ++c) {
            const int4 o = off4[c];
            const float4 scl = sc4[c], bi = bi4[c];
            pk[2 * c] = dequant2_bf16(static_cast<int32_t>(r[4 * c + 0]) + o.x,
                                      static_cast<int32_t>(r[4 * c + 1]) + o.y, st, scl.x, scl.y,
                                      bi.x, bi.y);
            pk[2 * c + 1] = dequant2_bf16(static_cast<int32_t>(r[4 * c + 2]) + o.z,
                                          static_cast<int32_t>(r[4 * c + 3]) + o.w, st, scl.z, scl.w,
                                          bi.z, bi.w);
          }
          if constexpr (GELU_OUT) {
#pragma unroll
            for (int c = 0; c < EPI_COLS / 2; ++c) pk[c] = gelu_pair_bf16(pk[c]);
          }
          uint8_t *stg = smem + P::OFF_EPI + (ew * 2 + (sc & 1)) * EPI_BYTES;
          if (lane == 0) bulk_wait_read<1>();  // the store that last read this buffer is done
          __syncwarp();
          // row = lane: 128 bytes = 8 chunks of 16 B, chunk u at (u ^ (row % 8)) (128-byte swizzle)
#pragma unroll
          for (int u = 0; u < 8; ++u)
            *reinterpret_cast<uint4 *>(stg + lane * 128 + ((u ^ (lane & 7)) << 4)) =
                make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && row0 < M && n0 < N) {
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
  if constexpr (PAIR) cluster_sync();  // the leader's MMAs and the other CTA's reads are done
  tc_fence_after();
  if (warp == W_TMEM) {
    if constexpr (PAIR)
      tmem_dealloc_pair(tmem_base, TMEM_COLS);
    else
      tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// Expand packed weight codes to the int8 operand order the kernel above
// widens A in (signed), and sum each row's codes: one warp per row.
__global__ void expand_weights_kernel(const uint8_t *__restrict__ qw, int N, int K,
                                      int8_t *__restrict__ qw8, int32_t *__restrict__ colsum) {
  const int lane = threadIdx.x & 31;
  const int n = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (n >= N) return;
  const uint4 *src = reinterpret_cast<const uint4 *>(qw + static_cast<int64_t>(n) * (K / 2));
  uint4 *dst = reinterpret_cast<uint4 *>(qw8 + static_cast<int64_t>(n) * K);
  int sum = 0;
  for (int c = lane; c < K / 32; c += 32) {
    uint4 o0, o1;
    widen_chunk<true>(src[c], o0, o1);
    dst[2 * c] = o0;
    dst[2 * c + 1] = o1;
    const uint32_t w[8] = {o0.x, o0.y, o0.z, o0.w, o1.x, o1.y, o1.z, o1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) sum = __dp4a(static_cast<int>(w[i]), 0x01010101, sum);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane == 0) colsum[n] = sum;
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
  return encode_tensor_map_2d(map, dt, base, inner, outer, row_bytes, box_inner, box_outer, swz);
}

template <int MODE, bool OUT_S32, bool GELU_OUT = false, bool ACC22 = false>
cudaError_t launch_t(const GemmArgs &a, cudaStream_t st) {
  using P = Plan<MODE>;
  auto kern = w4a4_gemm_kernel<MODE, OUT_S32, GELU_OUT, ACC22>;
  static ContextCache<bool> attr_set;  // the shared-memory attribute, per context
  bool done = false;
  cudaError_t e = attr_set.get(&done, [&](bool *v) {
    *v = true;
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, P::SMEM_BYTES);
  });
  if (e != cudaSuccess) return e;
  CUtensorMap tmA, tmB, tmY;
  const uint64_t kp = static_cast<uint64_t>(a.K / 2);
  const bool okA = P::A8 ? make_map_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.qx, a.K, a.M, a.K, BK,
                                       BM, CU_TENSOR_MAP_SWIZZLE_128B)
                         : make_map_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.qx, kp, a.M, kp, BKP,
                                       BM, P::A_TMEM ? CU_TENSOR_MAP_SWIZZLE_64B
                                                     : CU_TENSOR_MAP_SWIZZLE_NONE);
  if (!okA) return cudaErrorInvalidValue;
  const bool okB = P::B_PACKED ? make_map_2d(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.qw, kp, a.N, kp,
                                          BKP, BN, CU_TENSOR_MAP_SWIZZLE_NONE)
                            : make_map_2d(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.qw8, a.K, a.N,
                                          a.K, BK, P::TNL, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!okB) return cudaErrorInvalidValue;
  if (OUT_S32) {
    tmY = tmA;  // unused
  } else if (!make_map_2d(&tmY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.y, a.N, a.M,
                          static_cast<uint64_t>(a.N) * 2, EPI_COLS, 32, CU_TENSOR_MAP_SWIZZLE_128B)) {
    return cudaErrorInvalidValue;
  }
  const int num_m = static_cast<int>((a.M + P::TM - 1) / P::TM);
  const int num_n = (a.N + P::TN - 1) / P::TN;
  const int tiles = num_m * num_n;
  // programmatic stream serialization: the prologue may overlap the previous
  // kernel's tail (the kernel waits for it before reading any input)
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = P::SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int grid;
  if constexpr (P::PAIR) {
    // persistent CTA pairs: as many clusters of 2 as can be resident at once
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
    static ContextCache<int> clusters;
    int max_clusters = 0;
    e = clusters.get(&max_clusters, [&](int *v) {
      cudaLaunchConfig_t q = cfg;
      q.gridDim = dim3(2 * (device_sm_count() / 2), 1, 1);
      q.attrs = &attr[1];
      q.numAttrs = 1;
      return cudaOccupancyMaxActiveClusters(v, kern, &q);
    });
    if (e != cudaSuccess) return e;
    if (max_clusters <= 0) return cudaErrorInvalidConfiguration;
    grid = 2 * (tiles < max_clusters ? tiles : max_clusters);
  } else {
    grid = tiles < device_sm_count() ? tiles : device_sm_count();
  }
  cfg.gridDim = dim3(grid, 1, 1);
  // a stalled launch (failure-path test) gives every bounded wait 1 ms
  const unsigned long long wait_ns = a.stall ? 1000000ull : kWaitLimitNs;
  e = cudaLaunchKernelEx(&cfg, kern, tmA, tmB, tmY, a.scale_tok, a.scale_ch, a.bias, a.colsum, a.acc,
                         static_cast<int>(a.M), a.N, num_n, tiles, a.K / BK,
                         static_cast<uint32_t>(a.stall ? 1u : 0u), wait_ns);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

bool encode_tensor_map_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t inner,
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

cudaError_t launch_gemm(const GemmArgs &a, cudaStream_t st) {
  if (a.M <= 0) return cudaSuccess;
  // byte operands: 128 x 128 tiles when 128 x 256 ones would fill at most half of the SMs
  const int64_t wide_tiles = ((a.M + BM - 1) / BM) * ((a.N + BN - 1) / BN);
  const bool narrow = a.a8 && 2 * wide_tiles <= device_sm_count();
  // byte operands with small accumulators (4-bit weight codes): exact integer-add conversion
  const bool acc22 = a.acc22 && a.K <= 4096;
  // byte operands and enough tiles: CTA pairs on 256 x 256 tiles (frame QKV
  // 30.8 -> 31.5 us, the 48-block stack's layers 8-10 % faster: QKV 229 ->
  // 208 us, proj 82 -> 73, fc1 with the GELU 384 -> 367, fc2 253 -> 226)
  const bool pair = a.a8 && !narrow;
  if (a.gelu_out) {
    if (a.acc) return cudaErrorInvalidValue;
    if (a.a8 && acc22) {
      if (narrow) return launch_t<kInt8Narrow, false, true, true>(a, st);
      return pair ? launch_t<kInt8Pair, false, true, true>(a, st) : launch_t<kInt8, false, true, true>(a, st);
    }
    if (a.a8) {
      if (narrow) return launch_t<kInt8Narrow, false, true>(a, st);
      return pair ? launch_t<kInt8Pair, false, true>(a, st) : launch_t<kInt8, false, true>(a, st);
    }
    return a.qw8 ? launch_t<kExpanded, false, true>(a, st) : launch_t<kPacked, false, true>(a, st);
  }
  if (!a.acc && a.a8 && acc22) {
    if (narrow) return launch_t<kInt8Narrow, false, false, true>(a, st);
    return pair ? launch_t<kInt8Pair, false, false, true>(a, st) : launch_t<kInt8, false, false, true>(a, st);
  }
  if (narrow) return a.acc ? launch_t<kInt8Narrow, true>(a, st) : launch_t<kInt8Narrow, false>(a, st);
  if (pair) return a.acc ? launch_t<kInt8Pair, true>(a, st) : launch_t<kInt8Pair, false>(a, st);
  if (a.a8) return a.acc ? launch_t<kInt8, true>(a, st) : launch_t<kInt8, false>(a, st);
  const bool packed = (a.qw8 == nullptr);
  if (a.acc) return packed ? launch_t<kPacked, true>(a, st) : launch_t<kExpanded, true>(a, st);
  return packed ? launch_t<kPacked, false>(a, st) : launch_t<kExpanded, false>(a, st);
}

cudaError_t launch_expand_weights(const uint8_t *qw, int N, int K, int8_t *qw8, int32_t *colsum,
                                  cudaStream_t st) {
  expand_weights_kernel<<<(N + 7) / 8, 256, 0, st>>>(qw, N, K, qw8, colsum);
  return cudaGetLastError();
}

cudaError_t status_word(unsigned int **out) {
  static ContextCache<unsigned int *> cache;
  const cudaError_t e = cache.get(out, [](unsigned int **p) {
    void *a = nullptr;
    const cudaError_t r = cudaGetSymbolAddress(&a, g_status);
    *p = static_cast<unsigned int *>(a);
    return r;
  });
  if (e == cudaSuccess && *out == nullptr) return cudaErrorInvalidSymbol;
  return e;
}

unsigned long long current_context_id() {
  using GetCurrentFn = CUresult (*)(CUcontext *);
  using GetIdFn = CUresult (*)(CUcontext, unsigned long long *);
  static GetCurrentFn get_current = nullptr;
  static GetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetIdFn>(p);
  });
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  unsigned long long id = 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
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
