"""Coefficients of the GELU the kernels evaluate (csrc/gelu.cuh, gelu2_bf16:
the quantize kernel on an MLP's fc2 input, or the GEMM epilogue on its fc1
output), and a check of how its bf16 results compare with the exact GELU.

The kernel computes Phi(-|x|) = erfc(z) / 2, z = |x| / sqrt 2, as
exp2(log2(e) (-z^2) + c(u)) with u = z / (Z/2) - 1 on 0 <= z <= Z = 4.2
(|x| <= 5.94): the scaled complementary error function erfc(z) exp(z^2) is
smooth there and its logarithm is well matched by a polynomial (the
exp(-z^2 + polynomial) form of Numerical Recipes' erfcc, Press et al.,
section 6.2, here fitted in z instead of 1 / (1 + z / 2), which saves a
reciprocal).  c is our own least-squares fit of degree 11 at Chebyshev nodes,
scaled by log2(e), with the factor 1/2 of Phi folded into its constant term.
Beyond Z, Phi(-|x|) < 1.4e-9: the kernel takes it as 0, so GELU(x) = x for
x > 5.94 (exact in bf16) and -0 for x < -5.94 (the exact value is below
1e-8 |x|, far under any step the per-token quantizer can resolve).

    python -m w4a4_post_quantized_b200.gelu_fit        # prints the coefficients
"""
import math

import numpy as np

DEG = 11
Z = 4.2


def _g(z: float) -> float:
    return math.log(math.erfc(z)) + z * z


def coefficients():
    n = 800
    k = np.arange(n)
    us = np.cos((2 * k + 1) * np.pi / (2 * n))
    zs = (us + 1.0) * (Z / 2)
    c = np.polynomial.polynomial.polyfit(us, [_g(z) for z in zs], DEG) / math.log(2.0)
    c[0] -= 1.0  # Phi = erfc / 2: exp2(... - 1)
    return [float(np.float32(x)) for x in c]


def max_fit_error() -> float:
    """Largest |fit - log(erfc(z) exp(z^2))| on 0 <= z <= Z: the relative error of erfc (fp64)."""
    c = np.array(coefficients(), dtype=np.float64)
    c[0] += 1.0
    c *= math.log(2.0)
    zz = np.linspace(0.0, Z, 20001)
    return float(np.max(np.abs(np.polynomial.polynomial.polyval(zz / (Z / 2) - 1.0, c)
                               - np.array([_g(z) for z in zz]))))


if __name__ == "__main__":
    for i, c in enumerate(coefficients()):
        print(f"  c{i} = {c!r}f")
    print("max relative error of erfc on [0, Z] (fp64):", max_fit_error())
