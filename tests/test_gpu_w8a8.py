"""Parity of the W8A8 variant (W4A4_FLAG_INT8) with the CPU oracle.

The setting the QuantVGGT results report beside W4A4: the same DSFQ steps
with the symmetric 8-bit quantizer (step = absmax / 127, codes in
[-127, 127], one byte per code).  Same bars as the W4A4 path:
  * integer accumulators bit-exact against the oracle's int64 GEMM, up to the
    largest products 8-bit codes can form (|acc| = 127^2 K, beyond 2^24);
  * activation codes bit-exact except +-1 flips at rounding ties within the
    fp32 bound of tests/parity.py (qmax = 127), at most 1e-4 of the elements;
  * end to end: relative Frobenius error against the oracle's fp64 Y <= 2e-3.
"""
import numpy as np
import pytest
import torch

import oracle
from w4a4_post_quantized_b200 import synth
from parity import act_transform, compare_codes, rel_fro, tie_bound

pytestmark = pytest.mark.gpu

INT8 = 0x4


@pytest.fixture(scope="module")
def w4():
    from w4a4_post_quantized_b200 import w4a4
    assert w4a4.W4A4_FLAG_INT8 == INT8
    return w4a4


def dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


def bf16_dev(bits):
    return dev(bits.view(np.int16), torch.int16).view(torch.bfloat16)


def host(t):
    return t.cpu().numpy()


def y_to_f64(Y):
    return synth.bf16_bits_to_f32(host(Y.view(torch.int16)).view(np.uint16)).astype(np.float64)


def _raw_int8_weights(w4, B):
    """A weights struct holding raw 8-bit codes B [N, K] (no preparation)."""
    N, K = B.shape
    pw = w4.PreparedWeights(N, K, int8=True)
    pw.qw8.copy_(dev(B))
    pw.struct.flags = INT8
    return pw


# ------------------------------------------------------------------ integer GEMM
@pytest.mark.parametrize("M,N,K", [(1, 256, 1024), (300, 512, 1024), (1374, 1024, 1024),
                                   (257, 256, 4096), (640, 1024, 4096)])
def test_gemm_s32_int8_bit_exact(w4, M, N, K):
    rng = np.random.default_rng(M + N + K)
    A = rng.integers(-127, 128, (M, K)).astype(np.int8)
    B = rng.integers(-127, 128, (N, K)).astype(np.int8)
    acc = host(w4.w4a4_gemm_s32(dev(A.view(np.uint8)), _raw_int8_weights(w4, B)))
    assert np.array_equal(acc.astype(np.int64), oracle.int_gemm(A, B))


def test_gemm_s32_int8_many_tiles_per_cta(w4):
    """Byte-operand GEMM with several tiles per CTA: M = 8229 (65 row blocks,
    the last one ragged) x N = 3072 is 780 tiles of 128 x 256, 5-6 per
    persistent CTA, so every CTA cycles both accumulator buffers and the TMA
    ring several times; rows sampled from every row block, all columns,
    bit-exact against the oracle's int64 GEMM."""
    M, N, K = 8229, 3072, 1024
    rng = np.random.default_rng(77)
    A = rng.integers(-127, 128, (M, K)).astype(np.int8)
    B = rng.integers(-127, 128, (N, K)).astype(np.int8)
    acc = host(w4.w4a4_gemm_s32(dev(A.view(np.uint8)), _raw_int8_weights(w4, B)))
    rows = np.unique(np.concatenate([np.arange(0, M, 53), np.arange(M - 40, M)]))
    assert np.array_equal(acc[rows].astype(np.int64), oracle.int_gemm(A[rows], B))
    assert w4.w4a4_get_device_status() == 0


def test_gemm_int8_extreme_accumulators(w4):
    """Every product 127 * +-127 over K = 4096: |acc| = 66 064 384 > 2^24.  The
    s32 path is exact; the bf16 path converts with one rounding (relative
    error below 2^-24), so Y = bf16(acc * st * sc) exactly here."""
    K, M, N = 4096, 130, 256
    A = np.full((M, K), 127, np.int8)
    B = np.full((N, K), -127, np.int8)
    pw = _raw_int8_weights(w4, B)
    acc = host(w4.w4a4_gemm_s32(dev(A.view(np.uint8)), pw))
    assert np.all(acc == -127 * 127 * K)
    acc = host(w4.w4a4_gemm_s32(dev((-A).view(np.uint8)), pw))
    assert np.all(acc == 127 * 127 * K)
    pw.scale_ch.fill_(2.0 ** -20)
    pw.bias.zero_()
    st = torch.full((M,), 2.0 ** -4, device="cuda")
    Y = y_to_f64(w4.w4a4_linear(dev(A.view(np.uint8)), st, pw))
    want = synth.bf16_bits_to_f32(oracle.f64_to_bf16(np.full((M, N), -127.0 * 127 * K * 2.0 ** -24)))
    assert np.array_equal(Y, want.astype(np.float64))


# ------------------------------------------------------------- activation quantizer
@pytest.mark.parametrize("K", [1024, 4096])
@pytest.mark.parametrize("M,plain", [(1, False), (37, False), (1374, False), (300, True)])
def test_quantize_act_int8_parity(w4, M, K, plain):
    X = synth.activations(M, K, seed=200 + M)
    inv_s = None if plain else synth.random_scales(K, seed=K + 1, lo=0.25, hi=4.0)
    flags = INT8 | (w4.W4A4_FLAG_PLAIN if plain else 0)
    qx, st = w4.w4a4_quantize_act(bf16_dev(X), dev(inv_s) if inv_s is not None else None, flags)
    assert tuple(qx.shape) == (M, K)
    got = host(qx).view(np.int8)
    s = np.ones(K) if plain else 1.0 / inv_s.astype(np.float64)
    hat = oracle.act_hat(X, s, plain=plain)
    want_q, want_d = oracle.quantize_rows(hat, 8, "f32")
    np.testing.assert_allclose(host(st), want_d, rtol=2e-5, atol=0)
    assert got.min() >= -127 and got.max() <= 127
    amax = np.max(np.abs(hat), axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(amax[:, None] > 0, hat * 127.0 / amax[:, None], 0.0)
    xin = oracle.bf16_to_f64(X)
    mult = np.ones(K) if plain else 1.0 / s
    bound = tie_bound(xin, mult, ratio, amax, K, qmax=127.0, transform=act_transform(flags))
    compare_codes(got, want_q, ratio, bound, 1e-4 if M * K >= 10 ** 5 else None)


# -------------------------------------------------------------------- end to end
def _linear8(w4, M, N, K, seed, gelu=False, plain=False, sample=None):
    X = synth.activations(M, K, seed=seed)
    W = synth.weights(N, K, seed=seed + 1)
    b = synth.bias(N, seed=seed + 2)
    Xc = X[:synth.calibration_rows(M)]
    wflags = INT8 | (w4.W4A4_FLAG_PLAIN if plain else 0)
    pw = w4.w4a4_prepare_weights(bf16_dev(W), bf16_dev(b), bf16_dev(Xc), flags=wflags)
    assert pw.flags == wflags and pw.qw is None and pw.colsum is None
    Y = y_to_f64(w4.w4a4_linear_fused(bf16_dev(X), pw, flags=wflags | (w4.W4A4_FLAG_GELU if gelu else 0)))
    assert w4.w4a4_get_device_status() == 0
    ow = oracle.prepare_weights(W, b, Xc, plain=plain, decision="f32", bits=8)
    # the prepared 8-bit weight codes agree with the oracle's up to tie flips
    gw = host(pw.qw8).astype(np.int32) - ow.qw.astype(np.int32)
    assert np.all(np.abs(gw) <= 1) and np.count_nonzero(gw) <= max(1, 1e-4 * gw.size)
    rows = np.arange(M) if sample is None else sample
    Yo = oracle.linear(X[rows], ow, gelu=gelu, plain=plain, decision="f32", bits=8)[0]
    ref = oracle.reference_fp(X[rows], W, b, gelu=gelu)
    # at 8 bits the output's bf16 rounding is a visible part of the noise: the
    # oracle's Y is rounded the same way for the SQNR comparison
    Yo_bf = oracle.bf16_to_f64(oracle.f64_to_bf16(Yo))
    return rel_fro(Y[rows], Yo), oracle.sqnr_db(ref, Y[rows]), oracle.sqnr_db(ref, Yo_bf)


@pytest.mark.parametrize("M,N,K", [(1374, 1024, 1024), (1, 256, 1024), (200, 256, 4096),
                                   (1500, 3072, 1024)])
def test_linear_fused_int8_end_to_end(w4, M, N, K):
    err, sq_gpu, sq_or = _linear8(w4, M, N, K, seed=M + N + 5)
    assert err <= 2e-3, err
    assert abs(sq_gpu - sq_or) < 0.1


def test_linear_fused_int8_gelu_and_plain(w4):
    err, _, _ = _linear8(w4, 640, 1024, 4096, seed=177, gelu=True)
    assert err <= 2e-3, err
    err, _, _ = _linear8(w4, 640, 1024, 1024, seed=178, plain=True)
    assert err <= 2e-3, err


def test_linear_fused_int8_full_size_sampled(w4):
    """Frame-attention QKV at 8 frames (10992 x 1024 -> 3072) in the W8A8
    setting; sampled rows (special tokens included) against the oracle, and
    the 8-bit path's SQNR well above the 4-bit path's on the same layer."""
    M = 8 * synth.FRAME_TOKENS
    rows = np.unique(np.concatenate([synth.special_rows(M), np.arange(17, M, 211)]))
    err, sq8, _ = _linear8(w4, M, 3072, 1024, seed=2, sample=rows)
    assert err <= 2e-3, err
    X = synth.activations(M, 1024, seed=2)
    W, b = synth.weights(3072, 1024, seed=3), synth.bias(3072, seed=4)
    pw4 = w4.w4a4_prepare_weights(bf16_dev(W), bf16_dev(b), bf16_dev(X[:synth.calibration_rows(M)]))
    Y4 = y_to_f64(w4.w4a4_linear_fused(bf16_dev(X), pw4))
    sq4 = oracle.sqnr_db(oracle.reference_fp(X[rows], W, b), Y4[rows])
    assert sq8 > sq4 + 18.0, (sq8, sq4)


def test_host_pipeline_int8_matches_device_call(w4):
    M, N, K, chunk = 1000, 512, 1024, 384
    X = synth.activations(M, K, seed=7)
    W, b = synth.weights(N, K, seed=8), synth.bias(N, seed=9)
    pw = w4.w4a4_prepare_weights(bf16_dev(W), bf16_dev(b), bf16_dev(X[:synth.calibration_rows(M)]),
                                 flags=INT8)
    want = w4.w4a4_linear_fused(bf16_dev(X), pw, flags=INT8).cpu()
    Xh = torch.from_numpy(X.view(np.int16)).view(torch.bfloat16).pin_memory()
    Yh = torch.full((M, N), float("nan"), dtype=torch.bfloat16).pin_memory()
    pipe = w4.HostPipe()
    w4.w4a4_linear_fused_host(Xh, pw, Y_host=Yh, chunk_rows=chunk, pipe=pipe, flags=INT8)
    torch.cuda.current_stream().synchronize()
    assert torch.equal(Yh.view(torch.int16), want.view(torch.int16))
    assert w4.w4a4_get_device_status() == 0
