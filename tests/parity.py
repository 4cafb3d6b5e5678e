"""Comparison rules shared by the GPU parity tests.

Integer codes.  The CUDA path forms each rotated value in binary32 (an fp32
transform of the bf16 inputs, on the tensor cores or the CUDA cores: see
tie_bound), multiplies it by the binary32 reciprocal step
qmax/absmax and rounds the exact product half to even.  The oracle is compared
in two modes:
  * decision="f64" -- the method as the pages define it: exact fp64 rotation,
    fp64 step absmax/qmax, round(value/step);
  * decision="f32" -- the same quantizer with the rounding decision taken in
    binary32 (the oracle's fp64 values rounded to binary32, the binary32
    reciprocal step).
Where the exact ratio value/step lies within the GPU's error bound of a
rounding boundary (x.5), both codes are correct.  So a code may differ from
the oracle's only
  * by +-1,
  * at an element whose fp64 ratio is within `tie_bound` of a half-integer,
  * on at most 1e-4 of the elements (checked on the large cases).
Everything else must be bit-exact.

tie_bound, the bound on |ratio_gpu - ratio_oracle| (u = 2^-24):
  * the rotated value, e_val = c * sum_i|x_i| / sqrt(K) times the largest
    multiplier, with c fixed by the transform that formed it:
      - "fwht", the CUDA-core fast Walsh-Hadamard transform: a +-sum of K
        inputs formed through log2(K) round-to-nearest levels, c = log2(K) u;
      - "tc", the tensor-core kernel through H_K = H_128 (x) H_S
        (S = K / 128): the tensor cores sum 128 exact +-products in fp32,
        then log2(S) round-to-nearest butterfly levels finish in registers.
        The summation order and rounding inside the tensor core are not
        specified, so its sum of 128 terms is bounded as 128 sequential
        additions that may each lose a full unit in the last place (2u) of
        the running sum; its errors pass through the +-1 butterflies
        unchanged in size: c = (256 + log2 S) u;
    in the ratio that is e_ratio = qmax e_val / absmax;
  * the absmax is one of those values, so it carries the same absolute error
    e_val; through the reciprocal step it moves every ratio of the row by at
    most |ratio| e_val / absmax <= e_ratio;
  * relative roundings: the smoothing multiply (1 u), the binary32 reciprocal
    (1 u) and, against the fp64 oracle, the binary32 rounding of the value
    and of the absmax (2 u): at most 4 u |ratio|, plus the 8 u qmax slack kept
    from the binary32 comparison;
and the sum is taken with a factor 4 of margin.
"""
import numpy as np

U = 2.0 ** -24


def transform_error_coefficient(K: int, transform: str) -> float:
    """c in e_val = c * sum|x| / sqrt(K) (module docstring)."""
    if transform == "fwht":
        return np.log2(K) * U
    if transform == "tc":
        return (256 + np.log2(K // 128)) * U
    raise ValueError(transform)


def tie_bound(x_in: np.ndarray, mult: np.ndarray, ratio: np.ndarray, amax: np.ndarray, K: int,
              qmax: float = 7.0, transform: str = "fwht") -> np.ndarray:
    """Per-row bound on |ratio_cuda - ratio_exact| (rows of x_in are the
    transform's inputs, mult the per-channel multipliers, qmax the largest
    code: 7 for int4, 127 for int8; transform: "fwht" or "tc", the kernel
    that rotated the values)."""
    l1 = np.sum(np.abs(x_in), axis=1)
    e_val = transform_error_coefficient(K, transform) * l1 / np.sqrt(K) * np.max(np.abs(mult))
    with np.errstate(divide="ignore", invalid="ignore"):
        e_ratio = np.where(amax > 0, qmax * e_val / amax, 0.0)
    rmax = np.max(np.abs(ratio), axis=1)
    return 4.0 * (2.0 * e_ratio + 4 * U * rmax + 8 * U * qmax * (1 + rmax / qmax))


def compare_codes(got: np.ndarray, want: np.ndarray, ratio: np.ndarray, bound_row: np.ndarray,
                  max_frac: float | None = 1e-4):
    """got, want: int codes [rows, K]; ratio: fp64 value/step [rows, K];
    bound_row: tie_bound per row.  Returns the number of flips."""
    diff = got.astype(np.int32) - want.astype(np.int32)
    bad = np.nonzero(diff)
    n = len(bad[0])
    if n:
        assert np.all(np.abs(diff[bad]) == 1), f"code differs by more than 1: {np.unique(diff[bad])}"
        r = ratio[bad]
        dist = np.abs(np.abs(r - np.floor(r)) - 0.5)
        allowed = bound_row[bad[0]]
        assert np.all(dist <= allowed), (
            f"{int(np.sum(dist > allowed))} of {n} flips are not at rounding ties "
            f"(worst distance {dist.max():.3e}, bound {allowed.min():.3e})")
    if max_frac is not None:
        assert n <= max_frac * got.size, f"{n} flips > {max_frac} of {got.size}"
    return n


def rel_fro(got, want) -> float:
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    return float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-300))


def act_transform(flags: int) -> str:
    """Which kernel rotated the activations for these w4a4_quantize_act /
    w4a4_linear_fused flags: the tensor cores for DSFQ without GELU, unless
    W4A4_FLAG_FWHT (0x100); the CUDA-core transform otherwise."""
    plain, gelu, fwht = flags & 0x2, flags & 0x1, flags & 0x100
    return "tc" if not (plain or gelu or fwht) else "fwht"
