// gelu.cuh -- the GELU applied to bf16 activations: by the quantize kernel on
// the input of an MLP's second linear (quant.cu), or by the GEMM epilogue on
// the output of the first (gemm.cu).  Both give the same bf16 values.
#pragma once

#include <cuda_bf16.h>

namespace w4a4 {
namespace {

// GELU(x) = x Phi(x) of two bf16 inputs, rounded to bf16 (the activation an
// MLP's second linear receives).  Phi(-|x|) = erfc(z) / 2, z = |x| / sqrt 2,
// is evaluated as exp2(-log2(e) z^2 + c(u)), u = z / 2.1 - 1, for z <= 4.2: the
// exp(-z^2 + polynomial) form of Numerical Recipes' erfcc (section 6.2), with
// c a degree-11 fit in z by w4a4_post_quantized_b200/gelu_fit.py (relative
// error of erfc 6.5e-8 in fp64; factor 1/2 folded in).  For z > 4.2,
// Phi(-|x|) < 1.4e-9 is taken as 0.  Then GELU = x - x Phi(-x) for x >= 0 and
// x Phi(-|x|) for x < 0, with no cancellation on either side.  Pairs of inputs
// share packed fp32x2 arithmetic.
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
__device__ __forceinline__ unsigned long long mul2(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void gelu2_bf16(float &x0, float &x1) {
  constexpr float kZ = 4.2f;
  constexpr float kC[12] = {-3.02844500541687f,     -1.222137451171875f,   0.4550056755542755f,
                            -0.20184531807899475f,  0.09051182866096497f,  -0.03863636031746864f,
                            0.0148030836135149f,    -0.004897787235677242f, 0.0015472964150831103f,
                            -5.184028486837633e-05f, -0.0006587805110029876f, 0.0003328344027977437f};
  const float z0 = fabsf(x0) * 0.70710678118654752f, z1 = fabsf(x1) * 0.70710678118654752f;
  const unsigned long long z = f2(z0, z1);
  const unsigned long long u = fma2(z, f2(2.0f / kZ, 2.0f / kZ), f2(-1.0f, -1.0f));
  unsigned long long p = f2(kC[11], kC[11]);
#pragma unroll
  for (int i = 10; i >= 0; --i) p = fma2(p, u, f2(kC[i], kC[i]));
  const float nl2e = -1.4426950408889634f;
  float a0, a1;
  f2_split(fma2(mul2(z, z), f2(nl2e, nl2e), p), a0, a1);
  const float ph0 = z0 <= kZ ? ex2_approx(a0) : 0.0f;  // Phi(-|x|)
  const float ph1 = z1 <= kZ ? ex2_approx(a1) : 0.0f;
  const unsigned long long ph = f2(ph0, ph1), x = f2(x0, x1);
  float pos0, pos1, neg0, neg1;
  f2_split(fma2(f2(-x0, -x1), ph, x), pos0, pos1);  // x - x Phi(-x)
  f2_split(mul2(x, ph), neg0, neg1);                 // x Phi(x), x < 0
  const float g0 = x0 >= 0.0f ? pos0 : neg0, g1 = x1 >= 0.0f ? pos1 : neg1;
  const __nv_bfloat162 h = __floats2bfloat162_rn(g0, g1);
  x0 = __low2float(h);
  x1 = __high2float(h);
}

}  // namespace
}  // namespace w4a4
