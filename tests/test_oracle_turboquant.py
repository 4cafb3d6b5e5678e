"""Pins of the 3DTurboQuant oracle (oracle/turboquant.py) against things other
than itself: scipy's Beta distribution and adaptive quadrature, closed forms
of the coordinate density's moments and of the 1-bit quantizer, the classical
Gaussian Lloyd-Max tables (the d -> infinity limit), orthogonality, and the
page's MSE bound (page "3DTurboQuant: Training-Free Near-Optimal Quantization
for 3D Reconstruction Models", technical summary sections 2.1, 2.2, 3.2)."""
import math

import numpy as np
import pytest
import scipy.integrate
import scipy.linalg
import scipy.stats

from oracle import turboquant as tq


@pytest.mark.parametrize("d", [16, 45, 1024])
def test_coordinate_density_is_the_scaled_beta(d):
    """(x + 1)/2 ~ Beta((d-1)/2, (d-1)/2): density and normalisation."""
    a = (d - 1) / 2.0
    x = np.linspace(-0.95, 0.95, 77) * min(1.0, 6.0 / math.sqrt(d))
    want = scipy.stats.beta.pdf((x + 1) / 2, a, a) / 2
    np.testing.assert_allclose(tq.coord_density(x, d), want, rtol=1e-10)
    total, _ = scipy.integrate.quad(lambda t: tq.coord_density(np.array([t]), d)[0], -1, 1, limit=200)
    assert abs(total - 1.0) < 1e-9


@pytest.mark.parametrize("d", [16, 1024])
def test_coordinate_moments_closed_form(d):
    """A coordinate of a uniform unit vector: E x^2 = 1/d, E x^4 = 3/(d(d+2))."""
    f = lambda t, k: t ** k * tq.coord_density(np.array([t]), d)[0]
    m2, _ = scipy.integrate.quad(f, -1, 1, args=(2,), limit=200)
    m4, _ = scipy.integrate.quad(f, -1, 1, args=(4,), limit=200)
    assert abs(m2 - 1.0 / d) < 1e-12 * d
    assert abs(m4 - 3.0 / (d * (d + 2))) < 1e-12


@pytest.mark.parametrize("d", [16, 45, 1024])
def test_one_bit_quantizer_closed_form(d):
    """b = 1: boundary 0, centroids +-E|x| = +-Gamma(d/2) / (sqrt(pi) Gamma((d+1)/2))."""
    c, t = tq.lloyd_max(d, 1)
    e_abs = math.exp(math.lgamma(d / 2) - 0.5 * math.log(math.pi) - math.lgamma((d + 1) / 2))
    np.testing.assert_allclose(c, [-e_abs, e_abs], rtol=1e-10)
    assert t.tolist() == [0.0]


@pytest.mark.parametrize("b", [2, 3, 4])
def test_lloyd_max_conditions_with_independent_quadrature(b):
    """Optimality conditions of Lloyd-Max checked with scipy's adaptive
    quadrature: each centroid is its cell's conditional mean, each boundary
    the midpoint of its neighbours; the codebook is odd-symmetric."""
    d = 1024
    c, t = tq.lloyd_max(d, b)
    assert np.all(np.diff(c) > 0)
    np.testing.assert_allclose(c, -c[::-1], atol=1e-15)
    np.testing.assert_allclose(t, 0.5 * (c[1:] + c[:-1]), atol=1e-15)
    edges = np.concatenate([[-1.0], t, [1.0]])
    pdf = lambda x: scipy.stats.beta.pdf((x + 1) / 2, (d - 1) / 2, (d - 1) / 2) / 2
    for k in range(len(c)):
        m0, _ = scipy.integrate.quad(pdf, edges[k], edges[k + 1], limit=200, epsabs=1e-14)
        m1, _ = scipy.integrate.quad(lambda x: x * pdf(x), edges[k], edges[k + 1], limit=200, epsabs=1e-16)
        assert abs(m1 / m0 - c[k]) < 1e-9 / math.sqrt(d), (k, m1 / m0, c[k])


# Lloyd-Max quantizers of the unit Gaussian (Max 1960): positive centroids and
# the mean squared error; the coordinate density tends to N(0, 1/d).
GAUSS_LM = {
    2: ([0.4528, 1.510], 0.1175),
    3: ([0.2451, 0.7560, 1.344, 2.152], 0.03454),
    4: ([0.1284, 0.3881, 0.6568, 0.9423, 1.256, 1.618, 2.069, 2.733], 0.009497),
}


@pytest.mark.parametrize("b", [2, 3, 4])
def test_high_dimension_limit_is_the_gaussian_lloyd_max(b):
    d = 1 << 16
    c, t = tq.lloyd_max(d, b)
    want_c, want_D = GAUSS_LM[b]
    half = c[len(c) // 2:] * math.sqrt(d)
    np.testing.assert_allclose(half, want_c, atol=2e-3)
    assert abs(tq.distortion(d, c, t) * d - want_D) < 3e-4 * max(1.0, want_D * 10)


def test_rotation_is_orthogonal_and_a_signed_hadamard():
    d = 256
    s = np.where(np.random.default_rng(3).random(d) < 0.5, -1.0, 1.0)
    P = tq.rotation(s)
    np.testing.assert_allclose(P @ P.T, np.eye(d), atol=1e-13)
    np.testing.assert_array_equal(P * math.sqrt(d), scipy.linalg.hadamard(d) * s[None, :])


def test_codes_count_the_boundaries_below():
    c, t = tq.lloyd_max(64, 2)
    X = np.zeros((1, 64))
    X[0, 0] = 1.0                        # gamma = 1, y = first column of Pi
    s = np.ones(64)
    codes, gamma, Y = tq.encode(X, s, t)
    assert gamma[0] == 1.0
    brute = np.array([[sum(1 for b_ in t if b_ < y) for y in row] for row in Y])
    assert np.array_equal(codes.astype(int), brute)
    p = tq.pack4(np.array([[1, 2, 15, 0]], np.uint8))
    assert p.tolist() == [[0x21, 0x0F]]
    assert tq.unpack4(p, 4).tolist() == [[1, 2, 15, 0]]


@pytest.mark.parametrize("b", [2, 3, 4])
def test_mse_of_random_directions_matches_the_quantizer_and_the_bound(b):
    """For isotropic Gaussian vectors the rotated unit direction is uniform on
    the sphere, so E||theta - theta~||^2 / gamma^2 = d * D(b) exactly; the
    sample mean agrees within sampling error and stays under the page's bound."""
    d, n = 1024, 400
    rng = np.random.default_rng(11 + b)
    X = rng.standard_normal((n, d)) * rng.uniform(0.5, 3.0, (n, 1))
    s = np.where(rng.random(d) < 0.5, -1.0, 1.0)
    c, t = tq.lloyd_max(d, b)
    codes, gamma, _ = tq.encode(X, s, t)
    Xr = tq.decode(codes, gamma, s, c)
    rel = np.sum((X - Xr) ** 2, axis=1) / gamma ** 2
    D = tq.distortion(d, c, t) * d
    assert abs(rel.mean() - D) < 4 * rel.std() / math.sqrt(n) + 1e-4 * D
    assert rel.mean() <= tq.mse_bound(b)
    # fewer bits, more error: the bound and the distortion both fall by about 4 per bit
    assert 3.0 < (tq.distortion(d, *tq.lloyd_max(d, b - 1)) * d) / D < 4.5


def test_qr_rotation_is_the_sign_fixed_q_factor():
    """rotation_qr(G) is orthogonal and is the Q of the unique QR
    factorisation of G with a positive diagonal in R: Pi^T G is upper
    triangular with a positive diagonal, and Pi (Pi^T G) = G."""
    from w4a4_post_quantized_b200 import synth
    d = 256
    G = synth.gaussian_matrix(d, seed=5)
    P = tq.rotation_qr(G)
    np.testing.assert_allclose(P @ P.T, np.eye(d), atol=1e-12)
    R = P.T @ G
    assert np.max(np.abs(np.tril(R, -1))) < 1e-11 * np.max(np.abs(R))
    assert np.all(np.diag(R) > 0)
    np.testing.assert_allclose(P @ np.triu(R), G, atol=1e-11)
    # a Householder QR written out here (not LAPACK's) gives the same matrix
    A = G.copy()
    Q = np.eye(d)
    for k in range(d - 1):
        x = A[k:, k].copy()
        v = x.copy()
        v[0] += math.copysign(np.linalg.norm(x), x[0])
        v /= np.linalg.norm(v)
        A[k:, :] -= 2.0 * np.outer(v, v @ A[k:, :])
        Q[:, k:] -= 2.0 * np.outer(Q[:, k:] @ v, v)
    Q = Q * np.sign(np.diag(A))[None, :]
    np.testing.assert_allclose(Q, P, atol=1e-10)


def test_qr_rotation_spreads_a_basis_vector_like_a_uniform_direction():
    """Haar-distributed Pi: the image of a fixed unit vector is a uniform
    direction, whose coordinates follow the Beta coordinate density (a
    Kolmogorov-Smirnov test over the d coordinates of one column, and the
    fourth moment 3 / (d (d + 2)) within sampling error).  An identity or a
    signed permutation would fail both."""
    from w4a4_post_quantized_b200 import synth
    d = 1024
    P = tq.rotation_qr(synth.gaussian_matrix(d, seed=9))
    a = (d - 1) / 2.0
    for col in (0, 517):
        y = P[:, col]
        assert abs(np.sum(y * y) - 1.0) < 1e-12
        p = scipy.stats.kstest((y + 1) / 2, scipy.stats.beta(a, a).cdf).pvalue
        assert p > 1e-3, p
        m4 = np.mean(y ** 4)
        # Var(y^4) ~ 105/d^4 - (3/d^2)^2 = 96/d^4: 6 standard errors
        assert abs(m4 - 3.0 / (d * (d + 2))) < 6 * math.sqrt(96.0 / d ** 4 / d)


@pytest.mark.parametrize("b", [3, 4])
def test_mse_with_the_qr_rotation_matches_the_quantizer_and_the_bound(b):
    """The page's pipeline with its rotation: for isotropic inputs the
    normalised error is d * D(b) within sampling error, under the bound."""
    from w4a4_post_quantized_b200 import synth
    d, n = 1024, 300
    rng = np.random.default_rng(21 + b)
    X = rng.standard_normal((n, d)) * rng.uniform(0.5, 3.0, (n, 1))
    P = tq.rotation_qr(synth.gaussian_matrix(d, seed=3))
    c, t = tq.lloyd_max(d, b)
    codes, gamma, _ = tq.encode(X, P, t)
    Xr = tq.decode(codes, gamma, P, c)
    rel = np.sum((X - Xr) ** 2, axis=1) / gamma ** 2
    D = tq.distortion(d, c, t) * d
    assert abs(rel.mean() - D) < 4 * rel.std() / math.sqrt(n) + 1e-4 * D
    assert rel.mean() <= tq.mse_bound(b)
