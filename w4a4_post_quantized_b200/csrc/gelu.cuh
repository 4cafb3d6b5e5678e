// gelu.cuh -- the GELU applied to bf16 activations: by the quantize kernel on
// the input of an MLP's second linear (quant.cu), or by the GEMM epilogue on
// the output of the first (gemm.cu).  Both give the same bf16 values.
#pragma once

#include <cuda_bf16.h>

namespace w4a4 {
namespace {

// GELU(x) = x Phi(x) of a bf16 pair, rounded to bf16 (the activation an MLP's
// second linear receives), as
//     GELU(x) = max(x, 0) - a Phi(-a),   a = min(|x|, 5.9375)  (one fma),
// with no cancellation on either side, and Phi(-a) = exp2(c(u)),
// u = a / 2.96875 - 1, c the degree-7 fit of log2 Phi(-a) on [0, 5.9375]
// made by w4a4_post_quantized_b200/gelu_fit.py (the Gaussian's -a^2 / (2 ln 2)
// is part of the polynomial).  For every bf16 input with |x| <= 5.9375 the
// result is the exact GELU rounded to bf16 (checked exhaustively on the host
// with room for ex2.approx's error); above, it rounds to x as the exact GELU
// does, and below -5.9375 it is the constant -5.9375 Phi(-5.9375) = -8.6e-9
// (the exact values lie in (-8.6e-9, 0)).  Pairs share packed fp32x2
// arithmetic: 18 instructions per pair.
__device__ __forceinline__ unsigned long long f2(float a, float b) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2_split(unsigned long long v, float &a, float &b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ unsigned long long fma2(unsigned long long a, unsigned long long b,
                                                   unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// GELU of the two bf16 values of a packed pair (element 0 in the low half),
// bf16 pair out.
__device__ __forceinline__ uint32_t gelu_pair_bf16(uint32_t w) {
  constexpr float kA = 5.9375f;
  constexpr float kC[8] = {-9.38557243347168f,    -13.937207221984863f,   -5.902647495269775f,
                           -0.20142221450805664f, 0.090062215924263f,     -0.039654191583395004f,
                           0.01601894572377205f,  -0.003860969329252839f};
  const float x0 = __uint_as_float(w << 16), x1 = __uint_as_float(w & 0xFFFF0000u);
  // na = -a = max(-|x|, -A)
  const unsigned long long na = f2(fmaxf(-fabsf(x0), -kA), fmaxf(-fabsf(x1), -kA));
  const unsigned long long u = fma2(na, f2(-2.0f / kA, -2.0f / kA), f2(-1.0f, -1.0f));
  unsigned long long p = f2(kC[7], kC[7]);
#pragma unroll
  for (int i = 6; i >= 0; --i) p = fma2(p, u, f2(kC[i], kC[i]));
  float e0, e1;
  f2_split(p, e0, e1);
  // max(x, 0) - a Phi(-a), one rounding
  float g0, g1;
  f2_split(fma2(na, f2(ex2_approx(e0), ex2_approx(e1)), f2(fmaxf(x0, 0.0f), fmaxf(x1, 0.0f))), g0, g1);
  const __nv_bfloat162 h = __floats2bfloat162_rn(g0, g1);
  return *reinterpret_cast<const uint32_t *>(&h);
}

// The same on two floats holding bf16 values; the results are bf16 values.
__device__ __forceinline__ void gelu2_bf16(float &x0, float &x1) {
  const uint32_t w = (__float_as_uint(x1) & 0xFFFF0000u) | (__float_as_uint(x0) >> 16);
  const uint32_t g = gelu_pair_bf16(w);
  x0 = __uint_as_float(g << 16);
  x1 = __uint_as_float(g & 0xFFFF0000u);
}

}  // namespace
}  // namespace w4a4
