"""The GELU the kernels evaluate (csrc/gelu.cuh, gelu2_bf16) against its fit
script and against the oracle's exact-erf GELU, on the CPU.

  * the coefficients compiled into gelu.cuh are the ones
    w4a4_post_quantized_b200/gelu_fit.py produces, and the fit's relative
    error of erfc on [0, 4.2] is below 1e-7;
  * an emulation of the kernel's fp32 formula (every fused multiply-add
    rounded once to binary32, exp2 correctly rounded) gives, for every bf16
    input x with 1e-30 <= |x| <= 5.9, the oracle's GELU rounded to bf16 bit
    for bit;
  * and it does so with room for the hardware's ex2.approx (a few ulp, below
    3e-7 relative): for every such input the emulated value's relative error
    plus 3e-7 stays below the exact GELU's relative distance to the nearest
    bf16 rounding boundary, so the rounded result cannot change.
"""
import math
import os
import re

import numpy as np

import oracle
from w4a4_post_quantized_b200 import gelu_fit, synth

HDR = os.path.join(os.path.dirname(__file__), os.pardir, "w4a4_post_quantized_b200", "csrc", "gelu.cuh")


def _header_coefficients():
    text = open(HDR).read()
    m = re.search(r"kC\[12\]\s*=\s*\{([^}]*)\}", text)
    assert m, "coefficient table not found in gelu.cuh"
    return [float(v.strip().rstrip("f")) for v in m.group(1).split(",")]


def test_header_coefficients_are_the_fit():
    assert _header_coefficients() == gelu_fit.coefficients()
    assert gelu_fit.max_fit_error() < 1e-7


def _f32(x):
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def _fma(a, b, c):
    """binary32 fused multiply-add: the exact a*b (48 bits) plus c, rounded once."""
    return _f32(a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64))


def _kernel_gelu(x32):
    """The arithmetic of gelu2_bf16 on binary32 inputs, element by element."""
    kZ = np.float32(4.2)
    c = [np.float32(v) for v in _header_coefficients()]
    z = _f32(np.abs(x32).astype(np.float64) * np.float64(np.float32(0.70710678118654752)))
    u = _fma(z, np.full_like(z, np.float32(2.0) / kZ), np.full_like(z, np.float32(-1.0)))
    p = np.full_like(z, c[11])
    for i in range(10, -1, -1):
        p = _fma(p, u, np.full_like(z, c[i]))
    zz = _f32(z.astype(np.float64) * z.astype(np.float64))
    a = _fma(zz, np.full_like(z, np.float32(-1.4426950408889634)), p)
    ph = np.where(z <= kZ, _f32(np.exp2(a.astype(np.float64))), np.float32(0.0))
    pos = _fma(-x32, ph, x32)
    neg = _f32(x32.astype(np.float64) * ph.astype(np.float64))
    g = np.where(x32 >= 0, pos, neg).astype(np.float32)
    # round to bf16, nearest even
    b = g.view(np.uint32).astype(np.uint64)
    r = ((b + 0x7FFF + ((b >> 16) & 1)) >> 16).astype(np.uint16)
    return r


def test_every_bf16_input_matches_the_exact_gelu():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    x = synth.bf16_bits_to_f32(bits)
    with np.errstate(invalid="ignore"):
        keep = np.isfinite(x) & (np.abs(x) >= 1e-30) & (np.abs(x) <= 5.9)
    bits, x = bits[keep], x[keep]
    assert bits.size > 25000
    got = _kernel_gelu(x)
    want = oracle.gelu_bf16(bits)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, [(float(x[i]), hex(got[i]), hex(want[i])) for i in bad[:5]]
    # room for the hardware exp2: error + 3e-7 below the distance to a rounding boundary
    xe = x.astype(np.float64)
    ge = np.array([v * 0.5 * math.erfc(-v / math.sqrt(2.0)) for v in xe])
    ph = _ph64(x)
    em = np.where(x >= 0, xe - xe * ph, xe * ph)
    err = np.abs(em - ge) / np.abs(ge)
    b32 = ge.astype(np.float32).view(np.uint32) & np.uint32(0xFFFF0000)
    lo = b32.view(np.float32).astype(np.float64)                 # bf16 value at or toward zero from ge
    ulp = np.ldexp(1.0, np.frexp(np.abs(lo))[1] - 8)
    mids = np.stack([lo - np.sign(ge) * ulp / 2, lo + np.sign(ge) * ulp / 2])
    gap = np.min(np.abs(ge[None, :] - mids), axis=0) / np.abs(ge)
    assert np.all(err + 3e-7 < gap), float(np.min(gap - err))


def _ph64(x32):
    """The kernel's Phi(-|x|) before the final products, in binary32 steps."""
    kZ = np.float32(4.2)
    c = [np.float32(v) for v in _header_coefficients()]
    z = _f32(np.abs(x32).astype(np.float64) * np.float64(np.float32(0.70710678118654752)))
    u = _fma(z, np.full_like(z, np.float32(2.0) / kZ), np.full_like(z, np.float32(-1.0)))
    p = np.full_like(z, c[11])
    for i in range(10, -1, -1):
        p = _fma(p, u, np.full_like(z, c[i]))
    zz = _f32(z.astype(np.float64) * z.astype(np.float64))
    a = _fma(zz, np.full_like(z, np.float32(-1.4426950408889634)), p)
    return np.where(z <= kZ, _f32(np.exp2(a.astype(np.float64))), np.float32(0.0)).astype(np.float64)
