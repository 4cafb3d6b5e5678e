"""Coefficients of the GELU the kernels evaluate (csrc/gelu.cuh: the quantize
kernel on an MLP's fc2 input, or the GEMM epilogue on its fc1 output), and a
check of how its bf16 results compare with the exact GELU.

GELU(x) = x Phi(x) = max(x, 0) - |x| Phi(-|x|), with no cancellation on
either side.  The kernel evaluates Phi(-a), a = min(|x|, A), A = 5.9375, as
exp2(c(u)) with u = a / (A / 2) - 1 in [-1, 1]: log2 Phi(-a) is smooth on
[0, A] (it is -a^2 / (2 ln 2) plus the logarithm of the scaled complementary
error function, the exp(-z^2 + polynomial) form of Numerical Recipes' erfcc,
Press et al., section 6.2), so one polynomial c of degree 7 in u carries the
whole exponent, the Gaussian's quadratic included (to 6e-6 in log2 units,
far inside what the bf16 result can resolve; degree 7 is the lowest for
which every bf16 input still rounds to the exact GELU's bf16 value).  c is our own
least-squares fit at Chebyshev nodes, rounded to binary32.

Beyond A, Phi(-a) is held at Phi(-A) = 1.45e-9: GELU(x) for x > A rounds to
x in bf16 (as the exact GELU does), and for x < -A the result is the
constant -A Phi(-A) = -8.6e-9, where the exact GELU lies in (-8.6e-9, 0):
far under any step the per-token quantizer of the next linear can resolve.

    python -m w4a4_post_quantized_b200.gelu_fit        # prints the coefficients
"""
import math

import numpy as np

DEG = 7
A = 5.9375        # exactly representable in bf16 (0x40BE)


def _log2_phi_neg(a: float) -> float:
    """log2 Phi(-a) = log2(erfc(a / sqrt 2) / 2)."""
    return math.log2(0.5 * math.erfc(a / math.sqrt(2.0)))


def coefficients():
    n = 2000
    k = np.arange(n)
    us = np.cos((2 * k + 1) * np.pi / (2 * n))
    a = (us + 1.0) * (A / 2)
    c = np.polynomial.polynomial.polyfit(us, [_log2_phi_neg(v) for v in a], DEG)
    return [float(np.float32(x)) for x in c]


def max_fit_error() -> float:
    """Largest |fit - log2 Phi(-a)| on 0 <= a <= A in fp64 (log2 units: times
    ln 2, the relative error of Phi(-a))."""
    c = np.array(coefficients(), dtype=np.float64)
    aa = np.linspace(0.0, A, 20001)
    return float(np.max(np.abs(np.polynomial.polynomial.polyval(aa / (A / 2) - 1.0, c)
                               - np.array([_log2_phi_neg(v) for v in aa]))))


if __name__ == "__main__":
    for i, c in enumerate(coefficients()):
        print(f"  c{i} = {c!r}f")
    print("max error of log2 Phi(-a) on [0, A] (fp64):", max_fit_error())
