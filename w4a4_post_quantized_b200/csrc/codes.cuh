// codes.cuh -- the per-row quantizer's arithmetic shared by the row kernels
// (quant.cu: the CUDA-core transform; quant_tc.cu: the tensor-core
// transform): packed fp32x2 helpers, and the step / code forming and storing
// of page "十亿参数的三维重建模型，能塞进手机吗？", section 训练后量化（PTQ）
// (symmetric codes, round half to even).
#pragma once

#include <cstdint>

#include "kernels.h"

namespace w4a4 {
namespace {

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ unsigned long long pack2(float lo, float hi) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void unpack2(unsigned long long v, float &lo, float &hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ void mul_x2(float &a0, float &a1, float b0, float b1) {
  unsigned long long d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(pack2(a0, a1)), "l"(pack2(b0, b1)));
  unpack2(d, a0, a1);
}
__device__ __forceinline__ void fma_x2(float &a0, float &a1, unsigned long long b,
                                       unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(pack2(a0, a1)), "l"(b), "l"(c));
  unpack2(d, a0, a1);
}

// Low bytes of a, b, c, d as the bytes 0..3 of one word.
__device__ __forceinline__ uint32_t low_bytes(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

// Per-channel multiplier (from the block's shared table), per-row absmax,
// codes, store for a phase-2 row.  The transform's 1/sqrt(K) is an exact
// power of two, so it changes neither the absmax position nor any code: it is
// applied to the stored step only.  CODE (CodeFormat): kCodePacked4 codes in
// [-7, 7] two per byte; kCodeBytes4 the same codes one per byte in operand
// order; kCodeBytes8 codes in [-127, 127] one per byte.
// Bytes the codes of `elems` elements take in a code format.
template <int CODE>
constexpr int code_bytes_of(int elems) {
  return CODE == kCodePacked4 ? elems / 2 : elems;
}

// Codes of V consecutive elements whose row absmax is amax, stored at dst
// (16-byte aligned, or aligned to the codes' size when that is 4 or 8 bytes).  code = round-half-even(v * kQmax / amax); |v * inv| <=
// kQmax (1 + 2^-24), so no clamp can ever act.  Adding 1.5 * 2^23 in the same
// fused operation rounds the exact product to an integer whose low 8 bits are
// the two's-complement code.
// Stores W 32-bit words at dst with the widest accesses their count allows
// (dst aligned to 16 bytes, or to 4 W bytes when W < 4).
template <int W>
__device__ __forceinline__ void store_words(const uint32_t (&words)[W], uint8_t *__restrict__ dst) {
  if constexpr (W % 4 == 0) {
    uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
    for (int c = 0; c < W / 4; ++c)
      d4[c] = make_uint4(words[4 * c + 0], words[4 * c + 1], words[4 * c + 2], words[4 * c + 3]);
  } else if constexpr (W == 2) {
    *reinterpret_cast<uint2 *>(dst) = make_uint2(words[0], words[1]);
  } else {
    static_assert(W == 1, "word count");
    *reinterpret_cast<uint32_t *>(dst) = words[0];
  }
}

template <int V, int CODE>
__device__ __forceinline__ void store_code_words(const float (&v)[V], uint8_t *__restrict__ dst);

template <int V, int CODE>
__device__ __forceinline__ void store_codes(float (&v)[V], float amax, uint8_t *__restrict__ dst) {
  constexpr float kQmax = CODE == kCodeBytes8 ? 127.0f : 7.0f;
  if (amax < 0x1p-100f) {  // keep kQmax/amax finite: exact power-of-two rescale, same codes
#pragma unroll
    for (int r = 0; r < V; ++r) v[r] *= 0x1p+64f;
    amax *= 0x1p+64f;
  }
  const float inv = (amax > 0.0f) ? kQmax / amax : 0.0f;
  const unsigned long long inv2 = pack2(inv, inv), magic2 = pack2(12582912.0f, 12582912.0f);
#pragma unroll
  for (int k = 0; k < V; k += 2) fma_x2(v[k], v[k + 1], inv2, magic2);
  store_code_words<V, CODE>(v, dst);
}

// The codes of V values already rounded by the fused multiply-add with
// 1.5 * 2^23 (their low bytes are the two's-complement codes), packed in the
// code format and stored at dst.
template <int V, int CODE>
__device__ __forceinline__ void store_code_words(const float (&v)[V], uint8_t *__restrict__ dst) {
  if constexpr (CODE != kCodePacked4) {
    // one byte per code.  Natural order: word w holds elements 4w .. 4w + 3.
    // Operand order: the word pair (2g, 2g + 1) holds elements 8g + 0, 2, 4, 6
    // and 8g + 1, 3, 5, 7.
    uint32_t words[V / 4];
#pragma unroll
    for (int w = 0; w < V / 4; ++w) {
      const int e0 = CODE == kCodeBytes8 ? 4 * w : 8 * (w >> 1) + (w & 1);
      const int d = CODE == kCodeBytes8 ? 1 : 2;
      words[w] = low_bytes(__float_as_uint(v[e0]), __float_as_uint(v[e0 + d]),
                           __float_as_uint(v[e0 + 2 * d]), __float_as_uint(v[e0 + 3 * d]));
    }
    store_words<V / 4>(words, dst);
  } else {
    // word w: codes of elements 8w .. 8w + 7, element 2i in the low nibble of byte i
    uint32_t words[V / 8];
#pragma unroll
    for (int w = 0; w < V / 8; ++w) {
      uint32_t b[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) b[e] = __float_as_uint(v[8 * w + e]);
      const uint32_t even = low_bytes(b[0], b[2], b[4], b[6]);
      const uint32_t odd = low_bytes(b[1], b[3], b[5], b[7]);
      words[w] = (even & 0x0F0F0F0Fu) | ((odd << 4) & 0xF0F0F0F0u);
    }
    store_words<V / 8>(words, dst);
  }
}

}  // namespace
}  // namespace w4a4
