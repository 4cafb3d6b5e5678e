"""Parity of the 3DTurboQuant codec kernels (include/tq.h) with the oracle
(oracle/turboquant.py), page "3DTurboQuant: Training-Free Near-Optimal
Quantization for 3D Reconstruction Models", technical summary 2.2 / 3.2 / 4.2.

Bars:
  * norms: relative 1e-6 (fp32 sum of squares of the same inputs);
  * codes: equal to the oracle's (same fp32 codebook) except where the oracle's
    exact coordinate lies within the fp32 error bound of the transform from a
    boundary, and then only the neighbouring code; at most 1e-3 of the codes;
  * decode on identical codes: relative Frobenius error 1e-6 against the fp64
    reconstruction;
  * end to end: E||x - x~||^2 / ||x||^2 at most the page's bound, and on
    isotropic inputs within sampling error of d * D(b).
"""
import math

import numpy as np
import pytest
import torch

from oracle import turboquant as tq
from w4a4_post_quantized_b200 import synth

pytestmark = pytest.mark.gpu
D_ = 1024
U = 2.0 ** -24


@pytest.fixture(scope="module")
def w4():
    from w4a4_post_quantized_b200 import w4a4
    return w4a4


@pytest.fixture(scope="module")
def book(w4):
    c, t = w4.tq_codebook(D_, 4)
    return c, t, torch.from_numpy(c).cuda(), torch.from_numpy(t).cuda()


def _encode(w4, book, X, s):
    c, t, cd, td = book
    codes, norms = w4.tq_encode(torch.from_numpy(X).cuda(), torch.from_numpy(s).cuda(), td)
    return tq.unpack4(codes.cpu().numpy(), D_), norms.cpu().numpy(), codes, norms


def _code_flips_allowed(X, Y, codes_gpu, codes_or, t):
    """Every differing code is a neighbour and its coordinate lies within the
    fp32 error bound of the boundary between the two codes."""
    diff = codes_gpu.astype(int) - codes_or.astype(int)
    bad = np.nonzero(diff)
    if len(bad[0]) == 0:
        return 0
    assert np.all(np.abs(diff[bad]) == 1)
    gamma = np.sqrt(np.sum(X.astype(np.float64) ** 2, axis=1))
    l1 = np.sum(np.abs(X.astype(np.float64)), axis=1)
    # |y32 - y| <= (log2 d + 4) u ||x||_1 / (gamma sqrt d) + 4 u |y|  (transform, norm, product)
    bound = 4 * ((math.log2(D_) + 4) * U * l1[bad[0]] / (gamma[bad[0]] * math.sqrt(D_))
                 + 4 * U * np.abs(Y[bad]))
    k = np.minimum(codes_gpu[bad], codes_or[bad]).astype(int)  # the boundary between them
    dist = np.abs(Y[bad] - t.astype(np.float64)[k])
    assert np.all(dist <= bound), (dist.max(), bound.min())
    return len(bad[0])


@pytest.mark.parametrize("n", [1, 37, 1000])
def test_encode_matches_oracle(w4, book, n):
    c, t, _, _ = book
    X = synth.kv_vectors(n, D_, seed=n)
    s = synth.random_signs(D_, seed=7)
    codes_gpu, norms, _, _ = _encode(w4, book, X, s)
    codes_or, gamma, Y = tq.encode(X, s, t.astype(np.float64))
    np.testing.assert_allclose(norms, gamma, rtol=1e-6)
    flips = _code_flips_allowed(X, Y, codes_gpu, codes_or, t)
    assert flips <= max(2, 1e-3 * codes_gpu.size)


def test_decode_matches_oracle_on_identical_codes(w4, book):
    c, t, cd, td = book
    n = 777
    X = synth.kv_vectors(n, D_, seed=21)
    s = synth.random_signs(D_, seed=22)
    codes_u, norms, codes, norms_d = _encode(w4, book, X, s)
    Yg = w4.tq_decode(codes, norms_d, torch.from_numpy(s).cuda(), cd).cpu().numpy().astype(np.float64)
    Yo = tq.decode(codes_u, norms.astype(np.float64), s, c.astype(np.float64))
    err = np.linalg.norm(Yg - Yo) / np.linalg.norm(Yo)
    assert err <= 1e-6, err
    assert w4.w4a4_get_device_status() == 0


def test_zero_vector_and_empty_batch(w4, book):
    c, t, cd, td = book
    X = np.zeros((3, D_), np.float32)
    X[1] = synth.kv_vectors(1, D_, seed=3)[0]
    s = synth.random_signs(D_, seed=4)
    codes_u, norms, codes, norms_d = _encode(w4, book, X, s)
    assert norms[0] == 0.0 and norms[2] == 0.0
    assert np.all(codes_u[0] == 7) and np.all(codes_u[2] == 7)   # y = 0 lies above 7 boundaries
    Y = w4.tq_decode(codes, norms_d, torch.from_numpy(s).cuda(), cd).cpu().numpy()
    assert np.all(Y[0] == 0.0) and np.all(Y[2] == 0.0)
    e = torch.empty((0, D_), dtype=torch.float32, device="cuda")
    cz, nz = w4.tq_encode(e, torch.from_numpy(s).cuda(), td)
    assert cz.shape == (0, D_ // 2) and nz.shape == (0,)


@pytest.mark.parametrize("kind", ["isotropic", "kv"])
def test_round_trip_error_within_the_page_bound(w4, book, kind):
    """[TQ-MSE] E||x - x~||^2 / ||x||^2 <= sqrt(3) pi / 2 * 4^-b; on isotropic
    inputs the mean equals d * D(4) of the Lloyd-Max quantizer."""
    c, t, cd, td = book
    n = 4096
    rng = np.random.default_rng(5)
    X = (rng.standard_normal((n, D_)).astype(np.float32) if kind == "isotropic"
         else synth.kv_vectors(n, D_, seed=9))
    s = synth.random_signs(D_, seed=10)
    sd = torch.from_numpy(s).cuda()
    codes, norms = w4.tq_encode(torch.from_numpy(X).cuda(), sd, td)
    Y = w4.tq_decode(codes, norms, sd, cd).cpu().numpy().astype(np.float64)
    X64 = X.astype(np.float64)
    rel = np.sum((X64 - Y) ** 2, axis=1) / np.sum(X64 ** 2, axis=1)
    assert rel.mean() <= tq.mse_bound(4)
    if kind == "isotropic":
        Dd = tq.distortion(D_, c.astype(np.float64), t.astype(np.float64)) * D_
        assert abs(rel.mean() - Dd) < 4 * rel.std() / math.sqrt(n) + 1e-4 * Dd


def test_kv_cache_size_at_full_workload(w4, book):
    """The page's KV-cache case: 24576 vectors of 1024 fp32 (100.7 MB) encode to
    codes + norms of 12.68 MB (7.9x); sampled vectors checked against the oracle."""
    c, t, cd, td = book
    n = synth.KV_VECTORS
    X = synth.kv_vectors(n, D_, seed=1)
    s = synth.random_signs(D_, seed=2)
    codes, norms = w4.tq_encode(torch.from_numpy(X).cuda(), torch.from_numpy(s).cuda(), td)
    nbytes = codes.numel() + 4 * norms.numel()
    assert abs(X.nbytes / nbytes - 7.94) < 0.01
    rows = np.arange(0, n, 97)
    cg = tq.unpack4(codes.cpu().numpy()[rows], D_)
    co, gamma, Y = tq.encode(X[rows], s, t.astype(np.float64))
    np.testing.assert_allclose(norms.cpu().numpy()[rows], gamma, rtol=1e-6)
    assert _code_flips_allowed(X[rows], Y, cg, co, t) <= max(2, 1e-3 * cg.size)


# ------------------------------------------------- the page's rotation (dense Pi)
@pytest.fixture(scope="module")
def dense_pi(w4):
    """Pi from the QR of a seeded Gaussian matrix: the oracle's (numpy's QR,
    fp64) and the library's tf32 terms on the device."""
    G = synth.gaussian_matrix(D_, seed=77)
    P = tq.rotation_qr(G)
    hi, lo, thi, tlo = w4.tq_rotation_qr(G)
    dev = [torch.from_numpy(a).cuda() for a in (hi, lo, thi, tlo)]
    return P, dev


def _dense_flips_allowed(X, P, Y, codes_gpu, codes_or, t):
    """Differing codes are neighbours whose coordinate lies within the GPU's
    error bound of the boundary between them.  The GPU forms (Pi x)_j as a
    three-term tf32 product: the operands' tf32 terms carry x and Pi to 2^-22
    each, and each fp32 sum of 3 d products inside the tensor core is bounded
    as 3 d sequential additions losing up to 2u each (the MMA's summation order
    and rounding are not specified); the decision t gamma < (Pi x)_j adds a few
    u of |y|."""
    diff = codes_gpu.astype(int) - codes_or.astype(int)
    bad = np.nonzero(diff)
    if len(bad[0]) == 0:
        return 0
    assert np.all(np.abs(diff[bad]) == 1)
    X64 = X.astype(np.float64)
    gamma = np.sqrt(np.sum(X64 ** 2, axis=1))
    absdot = np.abs(X64) @ np.abs(P).T            # sum_k |x_k| |Pi_jk|
    c = 2 * 2.0 ** -22 + 3 * D_ * 2 * U
    bound = 4 * (c * absdot[bad] / gamma[bad[0]] + 8 * U * np.abs(Y[bad]))
    k = np.minimum(codes_gpu[bad], codes_or[bad]).astype(int)
    dist = np.abs(Y[bad] - t.astype(np.float64)[k])
    assert np.all(dist <= bound), (dist.max(), bound.min())
    return len(bad[0])


@pytest.mark.parametrize("n", [1, 37, 1000])
def test_dense_encode_matches_the_page_rotation(w4, book, dense_pi, n):
    """tq_encode_dense against the oracle with the page's Pi (QR of a Gaussian
    matrix): norms to 1e-6 relative, codes equal except neighbours at
    boundaries within the bound, at most 1e-3 of them."""
    c, t, cd, td = book
    P, (hi, lo, thi, tlo) = dense_pi
    X = synth.kv_vectors(n, D_, seed=300 + n)
    codes, norms = w4.tq_encode_dense(torch.from_numpy(X).cuda(), hi, lo, td)
    cg = tq.unpack4(codes.cpu().numpy(), D_)
    co, gamma, Y = tq.encode(X, P, t.astype(np.float64))
    np.testing.assert_allclose(norms.cpu().numpy(), gamma, rtol=1e-6)
    flips = _dense_flips_allowed(X, P, Y, cg, co, t)
    print(f"dense encode n={n}: {flips} code flips of {cg.size}")
    assert flips <= max(2, 1e-3 * cg.size)
    assert w4.w4a4_get_device_status() == 0


def test_dense_decode_matches_the_page_rotation(w4, book, dense_pi):
    """tq_decode_dense on given codes and norms against the oracle's fp64
    gamma Pi^T c[code], element by element within the product's error bound:
    the tf32 terms carry c and Pi to 2^-22 each and the tensor core's fp32 sum
    of 3 d products is bounded as 3 d additions losing up to 2u each, relative
    to gamma sum_k |c_k| |Pi_kj| (the sum cancels: its terms' magnitudes add up
    to about 30 times the result, so the relative error of the result is
    larger than that of its terms); then the scaling by gamma (u)."""
    c, t, cd, td = book
    P, (hi, lo, thi, tlo) = dense_pi
    n = 777
    rng = np.random.default_rng(31)
    cu = rng.integers(0, 16, size=(n, D_), dtype=np.uint8)
    gamma = rng.uniform(0.1, 10.0, size=n).astype(np.float32)
    packed = torch.from_numpy(tq.pack4(cu)).cuda()
    Yg = w4.tq_decode_dense(packed, torch.from_numpy(gamma).cuda(), thi, tlo, cd).cpu().numpy().astype(np.float64)
    Yo = tq.decode(cu, gamma.astype(np.float64), P, c.astype(np.float64))
    cv = np.abs(c.astype(np.float64))[cu.astype(np.int64)]
    bound = gamma.astype(np.float64)[:, None] * (2 * 2.0 ** -22 + 3 * D_ * 2 * U) * (cv @ np.abs(P)) + \
        2 * U * np.abs(Yo)
    assert np.all(np.abs(Yg - Yo) <= bound)
    err = np.linalg.norm(Yg - Yo) / np.linalg.norm(Yo)
    print(f"dense decode: relative Frobenius error {err:.2e}, largest error / bound "
          f"{np.max(np.abs(Yg - Yo) / bound):.3f}")
    assert w4.w4a4_get_device_status() == 0


def test_dense_zero_vectors_and_ragged_tail(w4, book, dense_pi):
    """A zero vector encodes to norm 0 and codes 7 (y = 0) and decodes to 0;
    n not a multiple of the 128-row tile."""
    c, t, cd, td = book
    P, (hi, lo, thi, tlo) = dense_pi
    n = 131
    X = synth.kv_vectors(n, D_, seed=41)
    X[[0, 130]] = 0.0
    codes, norms = w4.tq_encode_dense(torch.from_numpy(X).cuda(), hi, lo, td)
    cu = tq.unpack4(codes.cpu().numpy(), D_)
    nn = norms.cpu().numpy()
    assert nn[0] == 0.0 and nn[130] == 0.0 and np.all(nn[1:130] > 0)
    assert np.all(cu[0] == 7) and np.all(cu[130] == 7)
    Y = w4.tq_decode_dense(codes, norms, thi, tlo, cd).cpu().numpy()
    assert np.all(Y[0] == 0.0) and np.all(Y[130] == 0.0)


@pytest.mark.parametrize("kind", ["isotropic", "kv"])
def test_dense_round_trip_within_the_page_bound(w4, book, dense_pi, kind):
    """[TQ-MSE] with the page's rotation: E||x - x~||^2 / ||x||^2 under the
    bound; on isotropic inputs equal to d * D(4) within sampling error."""
    c, t, cd, td = book
    P, (hi, lo, thi, tlo) = dense_pi
    n = 4096
    rng = np.random.default_rng(6)
    X = (rng.standard_normal((n, D_)).astype(np.float32) if kind == "isotropic"
         else synth.kv_vectors(n, D_, seed=19))
    codes, norms = w4.tq_encode_dense(torch.from_numpy(X).cuda(), hi, lo, td)
    Y = w4.tq_decode_dense(codes, norms, thi, tlo, cd).cpu().numpy().astype(np.float64)
    X64 = X.astype(np.float64)
    rel = np.sum((X64 - Y) ** 2, axis=1) / np.sum(X64 ** 2, axis=1)
    assert rel.mean() <= tq.mse_bound(4)
    if kind == "isotropic":
        Dd = tq.distortion(D_, c.astype(np.float64), t.astype(np.float64)) * D_
        assert abs(rel.mean() - Dd) < 4 * rel.std() / math.sqrt(n) + 1e-4 * Dd


def test_fast_variant_against_the_page_rotation_statistics(w4, book, dense_pi):
    """The signed-Hadamard codec is not the page's rotation, so it is judged on
    the page's statistics only: on isotropic inputs its normalised error has
    the same mean as the page-rotation codec's (both d * D(4) within sampling
    error) and both stay under the bound."""
    c, t, cd, td = book
    P, (hi, lo, thi, tlo) = dense_pi
    n = 4096
    X = np.random.default_rng(7).standard_normal((n, D_)).astype(np.float32)
    Xd = torch.from_numpy(X).cuda()
    sd = torch.from_numpy(synth.random_signs(D_, seed=8)).cuda()
    X64 = X.astype(np.float64)
    rels = {}
    for name in ("hadamard", "page"):
        if name == "hadamard":
            codes, norms = w4.tq_encode(Xd, sd, td)
            Y = w4.tq_decode(codes, norms, sd, cd)
        else:
            codes, norms = w4.tq_encode_dense(Xd, hi, lo, td)
            Y = w4.tq_decode_dense(codes, norms, thi, tlo, cd)
        Y = Y.cpu().numpy().astype(np.float64)
        rels[name] = np.sum((X64 - Y) ** 2, axis=1) / np.sum(X64 ** 2, axis=1)
    a, b = rels["hadamard"], rels["page"]
    assert abs(a.mean() - b.mean()) < 4 * math.sqrt(a.var() / n + b.var() / n)
    assert a.mean() <= tq.mse_bound(4) and b.mean() <= tq.mse_bound(4)
    print(f"normalised MSE: fast variant {a.mean():.5f}, page rotation {b.mean():.5f}, "
          f"bound {tq.mse_bound(4):.5f}")
