"""The GELU the kernels evaluate (csrc/gelu.cuh, gelu_pair_bf16) against its fit
script and against the oracle's exact-erf GELU, on the CPU.

  * the coefficients compiled into gelu.cuh are the ones
    w4a4_post_quantized_b200/gelu_fit.py produces, and the fit describes
    log2 Phi(-a) on [0, 5.9375] to within 1e-5 (a relative error of Phi
    under 7e-6, some 300 times finer than a bf16 step);
  * for every bf16 input x with 1e-30 <= |x| <= 5.9375, an emulation of the
    kernel's binary32 arithmetic gives the oracle's GELU rounded to bf16 bit
    for bit, whatever value within 3e-7 relative of 2^arg the hardware's
    ex2.approx returns: the rounding steps after it are monotone, so the two
    ends of that range bound every possible result, and both ends round to
    the oracle's bf16 value;
  * above 5.9375 the result is x (as the exact GELU's), below -5.9375 it is
    the constant -5.9375 Phi(-5.9375) (-8.6e-9; the exact values lie between
    it and 0).
"""
import math
import os
import re

import numpy as np

import oracle
from w4a4_post_quantized_b200 import gelu_fit, synth

HDR = os.path.join(os.path.dirname(__file__), os.pardir, "w4a4_post_quantized_b200", "csrc", "gelu.cuh")
A = np.float32(5.9375)
EX2_REL = 3e-7      # bound on ex2.approx.ftz.f32's relative error (2^-22 = 2.4e-7)


def _header_coefficients():
    text = open(HDR).read()
    m = re.search(r"kC\[(\d+)\]\s*=\s*\{([^}]*)\}", text)
    assert m, "coefficient table not found in gelu.cuh"
    c = [float(v.strip().rstrip("f")) for v in m.group(2).split(",")]
    assert len(c) == int(m.group(1)) == gelu_fit.DEG + 1
    return c


def test_header_coefficients_are_the_fit():
    assert _header_coefficients() == gelu_fit.coefficients()
    assert gelu_fit.max_fit_error() < 1e-5
    # the fit is log2 Phi(-a): Phi(0) = 1/2 and Phi(-1) = 0.158655...
    c = np.array(gelu_fit.coefficients(), dtype=np.float64)
    assert abs(np.polynomial.polynomial.polyval(-1.0, c) + 1.0) < 1e-5
    u1 = 1.0 / (gelu_fit.A / 2) - 1.0
    assert abs(2.0 ** np.polynomial.polynomial.polyval(u1, c) / (0.5 * math.erfc(1 / math.sqrt(2))) - 1) < 1e-5


def _f32(x):
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def _fma(a, b, c):
    """binary32 fused multiply-add: the exact a*b (48 bits) plus c, rounded once."""
    return _f32(a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64))


def _bf16(g32):
    """binary32 -> bf16 bits, round to nearest even."""
    b = g32.view(np.uint32).astype(np.uint64)
    return ((b + 0x7FFF + ((b >> 16) & 1)) >> 16).astype(np.uint16)


def _kernel_gelu(x32, ex2_scale=1.0):
    """The arithmetic of gelu_pair_bf16 on binary32 inputs, element by element,
    with exp2 evaluated exactly and scaled by ex2_scale (then rounded)."""
    c = [np.float32(v) for v in _header_coefficients()]
    na = np.maximum(-np.abs(x32), -A).astype(np.float32)
    u = _fma(na, np.full_like(na, -(np.float32(2.0) / A)), np.full_like(na, np.float32(-1.0)))
    p = np.full_like(na, c[-1])
    for i in range(len(c) - 2, -1, -1):
        p = _fma(p, u, np.full_like(na, c[i]))
    ph = _f32(np.exp2(p.astype(np.float64)) * ex2_scale)
    relu = np.maximum(x32, np.float32(0.0)).astype(np.float32)
    return _bf16(_fma(na, ph, relu))


def _all_bf16():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    x = synth.bf16_bits_to_f32(bits)
    fin = np.isfinite(x)
    return bits[fin], x[fin]


def test_every_bf16_input_matches_the_exact_gelu():
    bits, x = _all_bf16()
    # below 1e-30 (bf16 subnormals among them) GELU(x) = x/2 + 0.4 x^2 sits
    # within 1e-60 relative of x/2, where the oracle's fp64 sees a rounding
    # tie; those inputs are checked apart below
    inside = (np.abs(x) <= A) & (np.abs(x) >= 1e-30)
    bits, x = bits[inside], x[inside]
    assert bits.size > 26000
    want = oracle.gelu_bf16(bits)
    # ph_hw within (1 +- EX2_REL) of 2^arg: the rounded fma is monotone in ph,
    # so the two ends bound every result the hardware can give
    lo = _kernel_gelu(x, 1.0 - EX2_REL - 1e-12)
    hi = _kernel_gelu(x, 1.0 + EX2_REL + 1e-12)
    mid = _kernel_gelu(x, 1.0)
    for got in (lo, hi, mid):
        bad = np.nonzero(got != want)[0]
        assert bad.size == 0, [(float(x[i]), hex(got[i]), hex(want[i])) for i in bad[:5]]


def test_outside_the_fitted_range():
    bits, x = _all_bf16()
    pos, neg = x > A, x < -A
    got = _kernel_gelu(x)
    # x > 5.9375: x itself, which is also the exact GELU rounded to bf16
    assert np.array_equal(got[pos], bits[pos])
    assert np.array_equal(oracle.gelu_bf16(bits[pos]), bits[pos])
    # x < -5.9375: one constant, -A Phi(-A), between the exact values and -1e-8 |x|
    const = set(got[neg].tolist())
    assert len(const) == 1
    v = float(synth.bf16_bits_to_f32(np.array(sorted(const), np.uint16))[0])
    phA = 0.5 * math.erfc(float(A) / math.sqrt(2.0))
    assert abs(v / (-float(A) * phA) - 1.0) < 1e-2
    exact = oracle.bf16_to_f64(oracle.gelu_bf16(bits[neg]))
    assert np.all(v <= exact) and np.all(np.abs(v) <= 1e-8 * np.abs(x[neg]))


def test_tiny_inputs_give_half_of_x():
    bits, x = _all_bf16()
    tiny = (np.abs(x) < 1e-30)
    got = synth.bf16_bits_to_f32(_kernel_gelu(x[tiny])).astype(np.float64)
    half = x[tiny].astype(np.float64) / 2
    quantum = 2.0 ** -133          # the smallest bf16 subnormal
    assert np.all(np.abs(got - half) <= np.maximum(quantum, np.abs(half) * 2.0 ** -8))
