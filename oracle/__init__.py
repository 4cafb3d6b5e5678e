"""CPU oracle for the DSFQ W4A4 linear layer -- TEST INFRASTRUCTURE ONLY.

What it is: a plain, slow, obviously correct fp64 / int64 statement of what
the DSFQ (Dual-Smoothed Fine-Grained Quantization) W4A4 linear layer computes,
written from the QuantVGGT pages:

  [PTQ]    page "十亿参数的三维重建模型，能塞进手机吗？", section "训练后量化（PTQ）"
  [ROT]    same page, "双平滑细粒度量化（DSFQ）" / "预全局旋转（Pre-Global-Rotation）"
  [SMOOTH] same page, "后局部平滑（Post-Local-Smooth）"
  [GRAN]   same page, "细粒度量化粒度（Fine-Grained Quantization Granularity）"

The arithmetic lives in w4a4_oracle.c (compiled by oracle/build.py); this
module only marshals numpy arrays and composes the steps in the pages' order.
Who may use it: tests/, __graft_entry__.smoke() and bench.py's CPU baseline and
reference arm.  The CUDA library never imports it, and it imports nothing from
the library.

Pins (tests/test_oracle_pins.py): Hadamard vs the closed form
(-1)^popcount(i&j) and scipy.linalg.hadamard; orthonormality; matmul
invariance under rotation; one-hot outlier dispersion; the smoothing identity;
quantizer range / error / tie / zero-row cases; int4 packing round trip; the
integer GEMM against brute force; a hand-derived worked example
(tests/golden/).  No page prints a worked numeric example, so the end-to-end
composition is pinned only through those step pins.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os

import numpy as np

from .build import LIB, build_oracle

_lib = None

_d = ctypes.POINTER(ctypes.c_double)
_i8 = ctypes.POINTER(ctypes.c_int8)
_u8 = ctypes.POINTER(ctypes.c_uint8)
_u16 = ctypes.POINTER(ctypes.c_uint16)
_i64 = ctypes.POINTER(ctypes.c_int64)


def lib():
    """Load (building if needed) the oracle's shared object."""
    global _lib
    if _lib is None:
        path = os.environ.get("W4A4_ORACLE_LIB") or (LIB if os.path.exists(LIB) else build_oracle())
        L = ctypes.CDLL(path)
        i64, i32, dbl = ctypes.c_int64, ctypes.c_int32, ctypes.c_double
        sig = {
            "oracle_bf16_to_double": [_u16, i64, _d],
            "oracle_double_to_bf16": [_d, i64, _u16],
            "oracle_gelu_bf16": [_u16, i64, _u16],
            "oracle_hadamard": [i32, _d],
            "oracle_rotate": [_d, i64, i32, _d],
            "oracle_smooth_factors": [_d, i64, _d, i32, i32, dbl, _d],
            "oracle_quantize_rows": [_d, i64, i32, i32, _i8, _d],
            "oracle_pack_int4": [_i8, i64, i32, _u8],
            "oracle_unpack_int4": [_u8, i64, i32, _i8],
            "oracle_int_gemm": [_i8, _i8, i64, i32, i32, _i64],
            "oracle_dequant": [_i64, _d, _d, _d, i64, i32, _d],
            "oracle_matmul_nt": [_d, _d, _d, i64, i32, i32, _d],
        }
        for name, argt in sig.items():
            fn = getattr(L, name)
            fn.argtypes = argt
            fn.restype = ctypes.c_int
        L.oracle_set_threads.argtypes = [ctypes.c_int]
        L.oracle_set_threads.restype = None
        L.oracle_max_threads.argtypes = []
        L.oracle_max_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def _p(a, t):
    return a.ctypes.data_as(t)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle: {what} rejected its arguments (rc={rc})")


def set_threads(n: int) -> None:
    lib().oracle_set_threads(int(n))


def max_threads() -> int:
    return int(lib().oracle_max_threads())


# ----------------------------------------------------------------- elementary
def bf16_to_f64(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.uint16)
    y = np.empty(x.shape, np.float64)
    _check(lib().oracle_bf16_to_double(_p(x, _u16), x.size, _p(y, _d)), "bf16_to_double")
    return y


def f64_to_bf16(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.empty(x.shape, np.uint16)
    _check(lib().oracle_double_to_bf16(_p(x, _d), x.size, _p(y, _u16)), "double_to_bf16")
    return y


def gelu_bf16(x: np.ndarray) -> np.ndarray:
    """Exact-erf GELU of bf16 values, rounded to bf16 (input of an MLP's
    second linear)."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    y = np.empty(x.shape, np.uint16)
    _check(lib().oracle_gelu_bf16(_p(x, _u16), x.size, _p(y, _u16)), "gelu_bf16")
    return y


def hadamard(d: int) -> np.ndarray:
    """[ROT] Sylvester Hadamard matrix of order d, entries +-1, natural order."""
    H = np.empty((d, d), np.float64)
    _check(lib().oracle_hadamard(d, _p(H, _d)), "hadamard")
    return H


def rotate(X: np.ndarray) -> np.ndarray:
    """[ROT] X . H / sqrt(d) along the last (feature) dimension, dense."""
    X = np.ascontiguousarray(X, dtype=np.float64)
    rows, d = X.reshape(-1, X.shape[-1]).shape
    out = np.empty_like(X)
    _check(lib().oracle_rotate(_p(X, _d), rows, d, _p(out, _d)), "rotate")
    return out


def smooth_factors(Xt: np.ndarray, Wt: np.ndarray, alpha: float = 0.5) -> np.ndarray:
    """[SMOOTH] s_j = max|Xt[:,j]|^alpha / max|Wt[:,j]|^(1-alpha) (1 if a max is 0)."""
    Xt = np.ascontiguousarray(Xt, dtype=np.float64)
    Wt = np.ascontiguousarray(Wt, dtype=np.float64)
    K = Xt.shape[1]
    assert Wt.shape[1] == K
    s = np.empty(K, np.float64)
    _check(lib().oracle_smooth_factors(_p(Xt, _d), Xt.shape[0], _p(Wt, _d), Wt.shape[0], K,
                                       float(alpha), _p(s, _d)), "smooth_factors")
    return s


def quantize_rows(Y: np.ndarray, bits: int = 4, decision: str = "f64"):
    """[PTQ][GRAN] per-row symmetric quantization; returns (codes int8, delta).

    decision="f64": the method as written, in fp64.
    decision="f32": the same quantizer with the rounding decision taken in
    binary32, the precision the CUDA kernels decide in: the values are first
    rounded to binary32, the step's reciprocal is the binary32 quotient
    (2^(bits-1)-1)/absmax, and the code is round-half-even of the exact
    product value*reciprocal.  delta is then the binary32 quotient
    absmax/(2^(bits-1)-1).
    """
    Y = np.ascontiguousarray(Y, dtype=np.float64)
    rows, K = Y.shape
    if decision == "f64":
        q = np.empty((rows, K), np.int8)
        delta = np.empty(rows, np.float64)
        _check(lib().oracle_quantize_rows(_p(Y, _d), rows, K, bits, _p(q, _i8), _p(delta, _d)),
               "quantize_rows")
        return q, delta
    if decision != "f32":
        raise ValueError(decision)
    qmax = (1 << (bits - 1)) - 1
    y32 = Y.astype(np.float32)
    amax = np.max(np.abs(y32), axis=1) if K else np.zeros(rows, np.float32)
    with np.errstate(divide="ignore"):
        inv = np.where(amax > 0, np.float32(qmax) / amax, np.float32(0)).astype(np.float32)
    delta = (amax / np.float32(qmax)).astype(np.float32)
    ratio = y32.astype(np.float64) * inv.astype(np.float64)[:, None]   # exact (24+24 bits)
    q = np.clip(np.rint(ratio), -(qmax + 1), qmax).astype(np.int8)
    return q, delta.astype(np.float64)


def pack_int4(q: np.ndarray) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.int8)
    rows, K = q.shape
    out = np.empty((rows, K // 2), np.uint8)
    _check(lib().oracle_pack_int4(_p(q, _i8), rows, K, _p(out, _u8)), "pack_int4")
    return out


def unpack_int4(p: np.ndarray, K: int) -> np.ndarray:
    p = np.ascontiguousarray(p, dtype=np.uint8)
    rows = p.shape[0]
    assert p.shape[1] * 2 == K
    q = np.empty((rows, K), np.int8)
    _check(lib().oracle_unpack_int4(_p(p, _u8), rows, K, _p(q, _i8)), "unpack_int4")
    return q


def int_gemm(A: np.ndarray, B: np.ndarray) -> np.ndarray:
    """acc[m, n] = sum_k A[m, k] B[n, k], exact int64."""
    A = np.ascontiguousarray(A, dtype=np.int8)
    B = np.ascontiguousarray(B, dtype=np.int8)
    M, K = A.shape
    N = B.shape[0]
    assert B.shape[1] == K
    acc = np.empty((M, N), np.int64)
    _check(lib().oracle_int_gemm(_p(A, _i8), _p(B, _i8), M, N, K, _p(acc, _i64)), "int_gemm")
    return acc


def dequant(acc, delta_tok, delta_ch, bias=None) -> np.ndarray:
    acc = np.ascontiguousarray(acc, dtype=np.int64)
    dt = np.ascontiguousarray(delta_tok, dtype=np.float64)
    dc = np.ascontiguousarray(delta_ch, dtype=np.float64)
    M, N = acc.shape
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float64)
    Y = np.empty((M, N), np.float64)
    _check(lib().oracle_dequant(_p(acc, _i64), _p(dt, _d), _p(dc, _d),
                                None if b is None else _p(b, _d), M, N, _p(Y, _d)), "dequant")
    return Y


def matmul_nt(X, W, bias=None) -> np.ndarray:
    X = np.ascontiguousarray(X, dtype=np.float64)
    W = np.ascontiguousarray(W, dtype=np.float64)
    M, K = X.shape
    N = W.shape[0]
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float64)
    Y = np.empty((M, N), np.float64)
    _check(lib().oracle_matmul_nt(_p(X, _d), _p(W, _d), None if b is None else _p(b, _d),
                                  M, N, K, _p(Y, _d)), "matmul_nt")
    return Y


# ------------------------------------------------------------ the method, composed
@dataclasses.dataclass
class PreparedWeights:
    """Offline result of DSFQ weight preparation for one linear layer."""
    qw: np.ndarray        # int8 [N, K] codes of W_hat = rotate(W) * s (bits-bit)
    delta_ch: np.ndarray  # fp64 [N] per-output-channel step
    bias: np.ndarray      # fp64 [N]
    s: np.ndarray         # fp64 [K] smoothing factors
    Wt: np.ndarray        # fp64 [N, K] rotated weights (kept for tests)


def prepare_weights(W_bf16, bias_bf16, Xcal_bf16, alpha: float = 0.5,
                    decision: str = "f64", plain: bool = False, bits: int = 4) -> PreparedWeights:
    """Offline weight side of DSFQ, in the pages' order:
    rotate W along its input features [ROT]; smoothing factors from the
    rotated calibration activations and rotated weights [SMOOTH]; scale the
    rotated weights by s (rotate first, then scale [SMOOTH]); per-output-
    channel symmetric int4 quantization [PTQ][GRAN].

    plain=True is the baseline without DSFQ (no rotation, s = 1), used only
    for the ablation of the pages' "rotation + scaling" claim.

    bits=8 is the W8A8 setting the results of the summary page of
    "量化視覺幾何基礎變換器" (lsdiaocha.cn, camera-pose paragraph) report
    beside W4A4: the same steps with the symmetric 8-bit quantizer of [PTQ]
    (step = absmax / 127)."""
    W = bf16_to_f64(W_bf16)
    N, K = W.shape
    bias = np.zeros(N) if bias_bf16 is None else bf16_to_f64(bias_bf16)
    if plain:
        Wt = W
        s = np.ones(K)
    else:
        Wt = rotate(W)
        Xt = rotate(bf16_to_f64(Xcal_bf16))
        s = smooth_factors(Xt, Wt, alpha)
    qw, dc = quantize_rows(Wt * s[None, :], bits, decision)
    return PreparedWeights(qw=qw, delta_ch=dc, bias=bias, s=s, Wt=Wt)


def act_hat(X_bf16, s, gelu: bool = False, plain: bool = False) -> np.ndarray:
    """Activation side before rounding: (optional GELU in bf16), rotation
    [ROT], division by the smoothing factors [SMOOTH]."""
    Xb = gelu_bf16(X_bf16) if gelu else np.asarray(X_bf16, np.uint16)
    X = bf16_to_f64(Xb)
    if plain:
        return X
    return rotate(X) / np.asarray(s, np.float64)[None, :]


def quantize_act(X_bf16, s, gelu: bool = False, decision: str = "f64", plain: bool = False,
                 bits: int = 4):
    """Per-token symmetric bits-bit codes (int4 by default, int8 for W8A8) of
    the rotated, smoothed activations; returns (codes int8 [M, K], delta_tok [M])."""
    return quantize_rows(act_hat(X_bf16, s, gelu, plain), bits, decision)


def linear(X_bf16, pw: PreparedWeights, gelu: bool = False, decision: str = "f64",
           plain: bool = False, bits: int = 4):
    """The quantized linear end to end: Y = (Qx Qw^T) * delta_tok * delta_ch + b.
    bits must equal the bit width pw was prepared with.
    Returns (Y fp64 [M, N], qx, delta_tok, acc)."""
    qx, dt = quantize_act(X_bf16, pw.s, gelu, decision, plain, bits)
    acc = int_gemm(qx, pw.qw)
    Y = dequant(acc, dt, pw.delta_ch, pw.bias)
    return Y, qx, dt, acc


def linear_ablation(X_bf16, W_bf16, bias_bf16, Xcal_bf16, rotate_on: bool, smooth_on: bool,
                    alpha: float = 0.5) -> np.ndarray:
    """The quantized linear with either half of DSFQ switched off, for the
    pages' ablation of "rotation + scaling" [ROT][SMOOTH]: rotation of X and W
    along the input features (rotate_on), then smoothing factors computed on
    the (rotated or not) calibration activations and weights (smooth_on, else
    s = 1), then per-token / per-channel symmetric int4 [PTQ][GRAN], the
    integer product and the dequantization.  Both on is DSFQ, both off is
    plain quantization.  Returns Y fp64 [M, N]."""
    W = bf16_to_f64(W_bf16)
    N, K = W.shape
    bias = np.zeros(N) if bias_bf16 is None else bf16_to_f64(bias_bf16)
    X = bf16_to_f64(np.asarray(X_bf16, np.uint16))
    Xc = bf16_to_f64(np.asarray(Xcal_bf16, np.uint16))
    if rotate_on:
        W, X, Xc = rotate(W), rotate(X), rotate(Xc)
    s = smooth_factors(Xc, W, alpha) if smooth_on else np.ones(K)
    qw, dc = quantize_rows(W * s[None, :], 4)
    qx, dt = quantize_rows(X / s[None, :], 4)
    return dequant(int_gemm(qx, qw), dt, dc, bias)


def reference_fp(X_bf16, W_bf16, bias_bf16, gelu: bool = False) -> np.ndarray:
    """Unquantized layer X W^T + b in fp64 from the same bf16 inputs (for SQNR)."""
    Xb = gelu_bf16(X_bf16) if gelu else np.asarray(X_bf16, np.uint16)
    b = None if bias_bf16 is None else bf16_to_f64(bias_bf16)
    return matmul_nt(bf16_to_f64(Xb), bf16_to_f64(W_bf16), b)


def sqnr_db(ref: np.ndarray, test: np.ndarray) -> float:
    ref = np.asarray(ref, np.float64)
    err = np.asarray(test, np.float64) - ref
    return float(10.0 * np.log10(np.sum(ref * ref) / max(np.sum(err * err), 1e-300)))
