"""CPU oracle for the 3DTurboQuant vector codec -- TEST INFRASTRUCTURE ONLY.

A plain fp64 statement of what the codec computes, written from page
"3DTurboQuant: Training-Free Near-Optimal Quantization for 3D Reconstruction
Models" (gist.science), technical summary:
  [TQ-FLOW]  section 2.2 (流程): norm separation gamma = ||theta||, rotation of the
             unit direction by a random orthogonal matrix Pi, per-coordinate b-bit
             scalar quantization with a codebook precomputed for the coordinates'
             Beta distribution, reconstruction gamma * Pi^T * centroids.
  [TQ-BETA]  section 2.1: after a random rotation the coordinates of a d-dimensional
             unit vector follow a known Beta distribution; Lloyd-Max quantizers for it
             are precomputed.
  [TQ-MSE]   section 3.2: E||theta - theta~||^2 <= gamma^2 * C * 4^-b, "about 2.7
             times" the information-theoretic 4^-b (section 2.1).
  [TQ-KV]    section 4.2: the DUSt3R KV cache, d = 1024, b = 4, 7.9x smaller.

Readings (the page prints no codebook, no storage format, and of the
rotation only that it is a random orthogonal matrix obtained by QR of a
Gaussian matrix):
  * Pi = Q diag(sign(diag(R))) for the QR factorisation G = Q R of a d x d
    matrix G of independent standard normal entries (an input, seeded): the
    sign fix makes the factorisation unique (R with a positive diagonal), and
    Pi is then Haar-distributed (rotation_qr).
  * a fast variant, not the page's matrix: Pi = H diag(s) / sqrt(d), H the
    Sylvester Hadamard matrix, s a seeded random sign vector -- orthogonal and
    applied in O(d log d) (rotation); the codec kernels offer it beside the
    dense Pi, and it is judged only on the MSE bound and the distortion.
  * the coordinate density of a uniformly random unit vector:
    f(x) = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)) (1 - x^2)^((d-3)/2) on [-1, 1]
    ((x + 1)/2 ~ Beta((d-1)/2, (d-1)/2)).
  * Lloyd-Max iteration: boundaries at the midpoints of adjacent centroids,
    centroids at the conditional means of their cells, started from the
    quantiles of f; the density is even, so the codebook is solved on the
    positive half (boundary 0 in the middle) and mirrored; integrals by
    Gauss-Legendre quadrature written out here.
  * the bound's constant: the formula prints sqrt(3 pi)/2 (= 1.53), which the
    exact Lloyd-Max distortion already exceeds for b >= 2 (b = 4: 1.53 * 4^-4
    = 0.0060 < 0.0095), while the text puts the factor at about 2.7; the
    reading is C = sqrt(3) pi / 2 = 2.72, a sqrt that lost its closing brace.
  * code k in 0 .. 2^b - 1 = the number of boundaries strictly below the
    coordinate; codes stored two per byte for b = 4 (element 2i in the low
    nibble).

Who may use it: tests/, __graft_entry__.smoke() and bench.py's CPU baseline and
reference arm.  It shares no code with the CUDA library.
"""
from __future__ import annotations

import math

import numpy as np

from . import hadamard


def coord_log_norm(d: int) -> float:
    """log of the normalising constant Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2))."""
    return math.lgamma(d / 2.0) - 0.5 * math.log(math.pi) - math.lgamma((d - 1) / 2.0)


def coord_density(x, d: int):
    """[TQ-BETA] density of one coordinate of a uniformly random unit vector in R^d."""
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    inside = np.abs(x) < 1.0
    out[inside] = np.exp(coord_log_norm(d) + 0.5 * (d - 3) * np.log1p(-x[inside] ** 2))
    return out


def _gauss_legendre(a: float, b: float, n: int = 64, pieces: int = 8):
    """Nodes and weights of a composite n-point Gauss-Legendre rule on [a, b]."""
    t, w = np.polynomial.legendre.leggauss(n)
    edges = np.linspace(a, b, pieces + 1)
    xs, ws = [], []
    for lo, hi in zip(edges[:-1], edges[1:]):
        xs.append(0.5 * (hi - lo) * t + 0.5 * (hi + lo))
        ws.append(0.5 * (hi - lo) * w)
    return np.concatenate(xs), np.concatenate(ws)


def _cell_moments(lo: float, hi: float, d: int):
    """Integral of f and of x f over [lo, hi]."""
    x, w = _gauss_legendre(lo, hi)
    fx = coord_density(x, d)
    return float(np.sum(w * fx)), float(np.sum(w * x * fx))


def lloyd_max(d: int, b: int, iters: int = 100000, tol: float = 1e-16):
    """[TQ-BETA] b-bit Lloyd-Max quantizer of the coordinate density (b >= 1).
    Returns (centroids [2^b], boundaries [2^b - 1]), both increasing."""
    half = (1 << b) // 2
    # the density lives within a few 1/sqrt(d) of 0: integrate over [0, R]
    R = min(1.0, 12.0 / math.sqrt(d))
    # start: centroids at the conditional medians of equal-probability cells
    grid = np.linspace(0.0, R, 20001)
    cdf = np.cumsum(coord_density(grid, d))
    cdf /= cdf[-1]
    c = np.interp((np.arange(half) + 0.5) / half, cdf, grid)
    tg, wg = np.polynomial.legendre.leggauss(96)
    for _ in range(iters):
        edges = np.concatenate([[0.0], 0.5 * (c[1:] + c[:-1]), [R]])
        lo, hi = edges[:-1, None], edges[1:, None]
        x = 0.5 * (hi - lo) * tg[None, :] + 0.5 * (hi + lo)
        w = 0.5 * (hi - lo) * wg[None, :]
        fx = coord_density(x, d)
        new = np.sum(w * x * fx, axis=1) / np.sum(w * fx, axis=1)
        done = np.max(np.abs(new - c)) < tol
        c = new
        if done:
            break
    cent = np.concatenate([-c[::-1], c])
    return cent, 0.5 * (cent[1:] + cent[:-1])


def distortion(d: int, centroids, boundaries) -> float:
    """E[(X - q(X))^2] of the scalar quantizer under the coordinate density."""
    R = min(1.0, 12.0 / math.sqrt(d))
    edges = np.concatenate([[-R], boundaries, [R]])
    total = 0.0
    for k, ck in enumerate(centroids):
        x, w = _gauss_legendre(edges[k], edges[k + 1])
        total += float(np.sum(w * (x - ck) ** 2 * coord_density(x, d)))
    return total


def rotation_qr(G) -> np.ndarray:
    """[TQ-FLOW] the page's random orthogonal matrix: Pi = Q diag(sign(diag R))
    for G = Q R (numpy's Householder QR, LAPACK), G a d x d Gaussian matrix."""
    G = np.asarray(G, dtype=np.float64)
    Q, R = np.linalg.qr(G)
    sg = np.sign(np.diag(R))
    sg[sg == 0] = 1.0
    return Q * sg[None, :]


def rotation(signs) -> np.ndarray:
    """The fast variant's orthogonal matrix Pi = H diag(s) / sqrt(d) (not the
    page's: see the module docstring)."""
    s = np.asarray(signs, dtype=np.float64)
    d = s.shape[0]
    return hadamard(d) * s[None, :] / math.sqrt(d)


def _as_rotation(Pi_or_signs) -> np.ndarray:
    a = np.asarray(Pi_or_signs, dtype=np.float64)
    return rotation(a) if a.ndim == 1 else a


def encode(X, Pi, boundaries):
    """[TQ-FLOW] gamma = ||x||, y = Pi x / gamma, code = #{boundaries < y}.
    Pi: the rotation matrix [d, d] (rotation_qr), or a sign vector [d] for the
    fast variant's H diag(s) / sqrt(d).
    Returns (codes uint8 [n, d], gamma [n], y [n, d])."""
    X = np.asarray(X, dtype=np.float64)
    gamma = np.sqrt(np.sum(X * X, axis=1))
    P = _as_rotation(Pi)
    with np.errstate(divide="ignore", invalid="ignore"):
        U = np.where(gamma[:, None] > 0, X / gamma[:, None], 0.0)
    Y = U @ P.T
    codes = np.searchsorted(np.asarray(boundaries, np.float64), Y, side="left").astype(np.uint8)
    return codes, gamma, Y


def decode(codes, gamma, Pi, centroids):
    """[TQ-FLOW] theta~ = gamma * Pi^T * centroids[codes] (Pi as for encode)."""
    P = _as_rotation(Pi)
    Yq = np.asarray(centroids, np.float64)[np.asarray(codes, np.int64)]
    return np.asarray(gamma, np.float64)[:, None] * (Yq @ P)


def pack4(codes) -> np.ndarray:
    """Two 4-bit codes per byte, element 2i in the low nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    assert c.shape[1] % 2 == 0 and c.max(initial=0) < 16
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def unpack4(packed, d: int) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty((p.shape[0], d), np.uint8)
    out[:, 0::2] = p & 0x0F
    out[:, 1::2] = p >> 4
    return out


def mse_bound(b: int) -> float:
    """[TQ-MSE] bound on E||theta - theta~||^2 / gamma^2 (constant sqrt(3) pi / 2,
    the reading above)."""
    return math.sqrt(3.0) * math.pi / 2.0 * 4.0 ** (-b)
