"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Bars (the quantized linear's numerical contract):
  * integer accumulators: bit-exact against the oracle's int64 GEMM on
    identical seeded codes;
  * activation / weight codes: bit-exact except +-1 flips at rounding ties
    within the fp32 bound of tests/parity.py, at most 1e-4 of the elements;
    per-token / per-channel steps within 1e-5 relative;
  * end to end: relative Frobenius error of Y against the oracle's fp64 Y at
    most 2e-3 (bf16 output rounding alone contributes about 1e-3); the
    epilogue on identical codes matches the oracle's dequantization rounded
    to bf16 to within one bf16 step everywhere.
Inputs are seeded synthetic VGGT-shaped tensors (w4a4_post_quantized_b200.synth).
"""
import numpy as np
import pytest
import torch

import oracle
from w4a4_post_quantized_b200 import synth
from parity import act_transform, compare_codes, rel_fro, tie_bound

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def w4():
    from w4a4_post_quantized_b200 import w4a4
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


# ------------------------------------------------------------------ integer GEMM
def _codes_weights(w4, B, K, expanded):
    """Weights struct holding raw packed codes B (and their widened copy)."""
    pw = w4.PreparedWeights(B.shape[0], K, expanded=expanded)
    pw.qw.copy_(dev(B))
    if expanded:
        w4.w4a4_expand_weights(pw)
    return pw


@pytest.mark.parametrize("expanded", [True, False])
@pytest.mark.parametrize("M,N,K", [(1, 256, 1024), (128, 256, 1024), (300, 512, 1024),
                                   (1374, 1024, 1024), (257, 256, 4096), (640, 1024, 4096)])
def test_gemm_s32_bit_exact(w4, M, N, K, expanded):
    A = synth.random_packed_codes(M, K, seed=M + 7)
    B = synth.random_packed_codes(N, K, seed=N + 11)
    acc = host(w4.w4a4_gemm_s32(dev(A), _codes_weights(w4, B, K, expanded)))
    want = oracle.int_gemm(oracle.unpack_int4(A, K), oracle.unpack_int4(B, K))
    assert np.array_equal(acc.astype(np.int64), want)


def test_expand_weights_layout_and_sums(w4):
    N, K = 256, 1024
    B = synth.random_packed_codes(N, K, seed=3)
    pw = _codes_weights(w4, B, K, True)
    codes = oracle.unpack_int4(B, K).astype(np.int64)
    assert np.array_equal(host(pw.colsum).astype(np.int64), codes.sum(axis=1))
    perm = np.array([0, 2, 4, 6, 1, 3, 5, 7])
    want = codes.reshape(N, K // 8, 8)[:, :, perm].reshape(N, K)
    assert np.array_equal(host(pw.qw8).astype(np.int64), want)


@pytest.mark.parametrize("expanded", [True, False])
def test_gemm_s32_extreme_codes(w4, expanded):
    K = 4096
    A = np.full((130, K // 2), 0x88, np.uint8)    # every code -8
    B = np.full((256, K // 2), 0x88, np.uint8)
    acc = host(w4.w4a4_gemm_s32(dev(A), _codes_weights(w4, B, K, expanded)))
    assert np.all(acc == 64 * K)
    B2 = np.full((256, K // 2), 0x77, np.uint8)   # every code 7
    acc = host(w4.w4a4_gemm_s32(dev(A), _codes_weights(w4, B2, K, expanded)))
    assert np.all(acc == -56 * K)
    A2 = np.full((130, K // 2), 0x77, np.uint8)
    acc = host(w4.w4a4_gemm_s32(dev(A2), _codes_weights(w4, B2, K, expanded)))
    assert np.all(acc == 49 * K)


# -------------------------------------------------------------- activation quantizer
def _check_quant(w4, X, K, inv_s32, flags, max_frac):
    M = X.shape[0]
    qx, st = w4.w4a4_quantize_act(bf16_dev(X), dev(inv_s32) if inv_s32 is not None else None, flags)
    qx, st = host(qx), host(st)
    plain = bool(flags & w4.W4A4_FLAG_PLAIN)
    gelu = bool(flags & w4.W4A4_FLAG_GELU)
    s = np.ones(K) if inv_s32 is None else 1.0 / inv_s32.astype(np.float64)
    hat = oracle.act_hat(X, s, gelu=gelu, plain=plain)
    xin = oracle.bf16_to_f64(oracle.gelu_bf16(X) if gelu else X)
    amax = np.max(np.abs(hat), axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(amax[:, None] > 0, hat * 7.0 / amax[:, None], 0.0)
    bound = tie_bound(xin, 1.0 / s, ratio, amax, K, transform=act_transform(flags))
    if gelu:  # GELU in fp32 may land one bf16 step away from the fp64 GELU
        bound = bound + 4.0 * 2.0 ** -8 * np.max(np.abs(xin), axis=1) * np.max(1.0 / s) / np.sqrt(K) * 7.0 / np.maximum(amax, 1e-300)
    got = oracle.unpack_int4(qx, K)
    # against the method as defined (fp64 decision) and against the binary32
    # decision; the flips of both must be ties within the bound
    # (without the rotation the ratios of bf16 inputs land exactly on ties
    # often; fp64 and binary32 round those differently, so in the plain
    # setting the fp64 comparison checks only that every flip is a tie)
    flips = {}
    for decision in ("f64", "f32"):
        want_q, want_d = oracle.quantize_rows(hat, 4, decision)
        np.testing.assert_allclose(st, want_d, rtol=2e-5, atol=0)
        cap = None if (plain and decision == "f64") else max_frac
        flips[decision] = compare_codes(got, want_q, ratio, bound, cap)
    print(f"M={M} K={K} flags={flags} ({act_transform(flags)}): flips vs fp64 {flips['f64']}, "
          f"vs binary32 {flips['f32']} of {got.size}")
    return flips["f64"]


@pytest.mark.parametrize("K", [1024, 4096])
@pytest.mark.parametrize("M", [1, 37, 1374])
def test_quantize_act_parity(w4, M, K):
    X = synth.activations(M, K, seed=100 + M)
    inv_s = synth.random_scales(K, seed=K, lo=0.25, hi=4.0)
    _check_quant(w4, X, K, inv_s, 0, None)


@pytest.mark.parametrize("K", [1024, 4096])
@pytest.mark.parametrize("M", [1, 37, 1374])
def test_quantize_act_parity_cuda_core_transform(w4, M, K):
    """W4A4_FLAG_FWHT: the same quantizer with the CUDA-core transform."""
    X = synth.activations(M, K, seed=150 + M)
    inv_s = synth.random_scales(K, seed=K + 5, lo=0.25, hi=4.0)
    _check_quant(w4, X, K, inv_s, w4.W4A4_FLAG_FWHT, None)


@pytest.mark.parametrize("fl", [0, 0x100])
def test_quantize_act_parity_frame_batch(w4, fl):
    M, K = 4 * 1374, 1024
    X = synth.activations(M, K, seed=5)
    inv_s = synth.random_scales(K, seed=6, lo=0.25, hi=4.0)
    _check_quant(w4, X, K, inv_s, fl, 1e-4)


def test_quantize_act_parity_k4096_frame_batch(w4):
    M, K = 2 * 1374 + 37, 4096
    X = synth.activations(M, K, seed=15)
    inv_s = synth.random_scales(K, seed=16, lo=0.25, hi=4.0)
    _check_quant(w4, X, K, inv_s, 0, 1e-4)


@pytest.mark.parametrize("K", [1024, 4096])
def test_quantize_act_plain(w4, K):
    X = synth.activations(300, K, seed=9)
    _check_quant(w4, X, K, None, 2, 1e-4)


def test_quantize_act_gelu(w4):
    K = 4096
    X = synth.to_bf16_bits(np.random.default_rng(3).standard_normal((700, K)).astype(np.float32) * 2)
    inv_s = synth.random_scales(K, seed=12, lo=0.5, hi=2.0)
    _check_quant(w4, X, K, inv_s, 1, 2e-4)


def test_quantize_act_zero_rows(w4):
    K = 1024
    X = synth.activations(20, K, seed=4)
    X[[0, 7, 19]] = 0
    qx, st = w4.w4a4_quantize_act(bf16_dev(X), dev(np.ones(K, np.float32)))
    qx, st = host(qx), host(st)
    assert np.all(st[[0, 7, 19]] == 0) and np.all(qx[[0, 7, 19]] == 0)
    assert np.all(st[[1, 2, 18]] > 0)


# ------------------------------------------------------------------ weight preparation
@pytest.mark.parametrize("N,K", [(256, 1024), (1024, 4096)])
def test_prepare_weights_parity(w4, N, K):
    W = synth.weights(N, K, seed=N)
    b = synth.bias(N, seed=N + 1)
    Xc = synth.activations(1374, K, seed=K + 2)
    pw = w4.w4a4_prepare_weights(bf16_dev(W), bf16_dev(b), bf16_dev(Xc))
    ow = oracle.prepare_weights(W, b, Xc)
    np.testing.assert_allclose(host(pw.smooth), ow.s, rtol=2e-5)
    np.testing.assert_allclose(host(pw.inv_smooth), 1.0 / ow.s, rtol=2e-5)
    np.testing.assert_allclose(host(pw.bias), ow.bias, rtol=0, atol=0)
    got = oracle.unpack_int4(host(pw.qw), K)
    # (1) the oracle's binary32 decision on the GPU's own (binary32) s
    s32 = host(pw.smooth).astype(np.float64)
    hat = ow.Wt * s32[None, :]
    want_q, want_d = oracle.quantize_rows(hat, 4, "f32")
    np.testing.assert_allclose(host(pw.scale_ch), want_d, rtol=2e-5)
    amax = np.max(np.abs(hat), axis=1)
    ratio = hat * 7.0 / amax[:, None]
    bound = tie_bound(oracle.bf16_to_f64(W), s32, ratio, amax, K)
    compare_codes(got, want_q, ratio, bound, 2e-4)
    # (2) the method as defined: the oracle's own fp64 s and fp64 decision.
    # The GPU's s differs from the fp64 s by the relative amount d_j (its
    # column maxima come from the fp32 transform, then s is rounded to
    # binary32); that moves a ratio by at most |ratio| (d_j + max_j d_j) (the
    # element's own factor and the absmax's), on top of the bound above.
    d = np.abs(s32 / ow.s - 1.0)
    hat64 = ow.Wt * ow.s[None, :]
    amax64 = np.max(np.abs(hat64), axis=1)
    ratio64 = hat64 * 7.0 / amax64[:, None]
    bound64 = tie_bound(oracle.bf16_to_f64(W), ow.s, ratio64, amax64, K) + \
        4.0 * 7.0 * (np.max(d) + np.max(d))
    n64 = compare_codes(got, ow.qw, ratio64, bound64, 2e-4)
    np.testing.assert_allclose(host(pw.scale_ch), ow.delta_ch, rtol=2e-5)
    print(f"N={N} K={K}: weight-code flips vs fp64 s and decision {n64} of {got.size}, "
          f"max relative s difference {np.max(d):.2e}")


# -------------------------------------------------------------------- epilogue
@pytest.mark.parametrize("expanded", [True, False])
@pytest.mark.parametrize("M,N,K", [(300, 512, 1024), (1374, 1024, 4096)])
def test_linear_epilogue_on_identical_codes(w4, M, N, K, expanded):
    A = synth.random_packed_codes(M, K, seed=1)
    B = synth.random_packed_codes(N, K, seed=2)
    st = synth.random_scales(M, seed=3, lo=1e-3, hi=1e-1)
    sc = synth.random_scales(N, seed=4, lo=1e-3, hi=1e-2)
    bias = synth.random_scales(N, seed=5, lo=-0.5, hi=0.5)
    pw = _codes_weights(w4, B, K, expanded)
    pw.scale_ch.copy_(dev(sc))
    pw.bias.copy_(dev(bias))
    Y = w4.w4a4_linear(dev(A), dev(st), pw)
    got = y_to_f64(Y)
    acc = oracle.int_gemm(oracle.unpack_int4(A, K), oracle.unpack_int4(B, K))
    want = oracle.dequant(acc, st.astype(np.float64), sc.astype(np.float64), bias.astype(np.float64))
    want_bf = oracle.bf16_to_f64(oracle.f64_to_bf16(want))
    # one bf16 step of the result, plus the fp32 epilogue's own error bound
    # (a few ulp of the largest term), which matters where y ~ -bias cancels
    terms = np.abs(acc * st.astype(np.float64)[:, None] * sc.astype(np.float64)[None, :]) + np.abs(bias)[None, :]
    tol = np.abs(want_bf) * 2.0 ** -7 + 4 * 2.0 ** -24 * terms
    assert np.all(np.abs(got - want_bf) <= tol)
    assert np.mean(got == want_bf) > 0.999


# -------------------------------------------------------------------- end to end
def _linear_case(w4, M, N, K, seed, gelu=False, plain=False, sample=None, expanded=True,
                 decision="f32"):
    X = synth.activations(M, K, seed=seed)
    W = synth.weights(N, K, seed=seed + 1)
    b = synth.bias(N, seed=seed + 2)
    Xc = X[:synth.calibration_rows(M)]
    flags = (w4.W4A4_FLAG_GELU if gelu else 0) | (w4.W4A4_FLAG_PLAIN if plain else 0)
    pw = w4.w4a4_prepare_weights(bf16_dev(W), bf16_dev(b), bf16_dev(Xc),
                                 flags=w4.W4A4_FLAG_PLAIN if plain else 0, expanded=expanded)
    Y = y_to_f64(w4.w4a4_linear_fused(bf16_dev(X), pw, flags=flags))
    assert w4.w4a4_get_device_status() == 0
    # rounding decisions in binary32 on both sides (the kernels' precision);
    # bf16 inputs without rotation hit exact rounding ties, which fp64 and fp32
    # resolve differently
    ow = oracle.prepare_weights(W, b, Xc, plain=plain, decision=decision)
    rows = np.arange(M) if sample is None else sample
    Yo = oracle.linear(X[rows], ow, gelu=gelu, plain=plain, decision=decision)[0]
    err = rel_fro(Y[rows], Yo)
    ref = oracle.reference_fp(X[rows], W, b, gelu=gelu)
    return err, oracle.sqnr_db(ref, Y[rows]), oracle.sqnr_db(ref, Yo)


@pytest.mark.parametrize("M,N,K", [(1374, 1024, 1024), (1, 256, 1024), (200, 256, 4096),
                                   (1500, 3072, 1024)])
@pytest.mark.parametrize("decision", ["f64", "f32"])
def test_linear_fused_end_to_end(w4, M, N, K, decision):
    err, sq_gpu, sq_or = _linear_case(w4, M, N, K, seed=M + N, decision=decision)
    assert err <= 2e-3, err
    assert abs(sq_gpu - sq_or) < 0.1


def test_linear_fused_packed_weights_path(w4):
    err, _, _ = _linear_case(w4, 700, 512, 1024, seed=91, expanded=False)
    assert err <= 2e-3, err


def test_linear_fused_gelu_and_plain(w4):
    err, _, _ = _linear_case(w4, 640, 1024, 4096, seed=77, gelu=True)
    assert err <= 2e-3, err
    err, _, _ = _linear_case(w4, 640, 1024, 1024, seed=78, plain=True)
    assert err <= 2e-3, err


def test_linear_fused_full_size_sampled(w4):
    """Frame-attention QKV at 8 frames (10992 x 1024 -> 3072), the benchmark's
    launch configuration; the oracle checks sampled rows, special tokens included."""
    M = 8 * synth.FRAME_TOKENS
    rows = np.unique(np.concatenate([synth.special_rows(M), np.arange(17, M, 211)]))
    for decision in ("f64", "f32"):
        err, sq_gpu, sq_or = _linear_case(w4, M, 3072, 1024, seed=2, sample=rows, decision=decision)
        print(f"frame-QKV sampled rows, oracle decision {decision}: rel_fro {err:.3e}, "
              f"SQNR gpu {sq_gpu:.2f} dB oracle {sq_or:.2f} dB")
        assert err <= 2e-3, (decision, err)
        assert abs(sq_gpu - sq_or) < 0.1


def test_empty_input_is_a_no_op(w4):
    pw = w4.PreparedWeights(256, 1024)
    X = torch.empty((0, 1024), dtype=torch.bfloat16, device="cuda")
    Y = w4.w4a4_linear_fused(X, pw)
    assert Y.shape == (0, 256)
    torch.cuda.synchronize()


def test_device_status_clear(w4):
    w4.w4a4_clear_device_status()
    assert w4.w4a4_get_device_status() == 0


# ------------------------------------------------- int4 codes one per byte (fused route)
UNPACKED = 0x8
OPERAND_ORDER = np.array([0, 2, 4, 6, 1, 3, 5, 7])


@pytest.mark.parametrize("M,K,gelu", [(1, 1024, False), (1374, 1024, False), (257, 4096, True)])
def test_unpacked_codes_equal_packed_codes(w4, M, K, gelu):
    """The quantize kernel's one-per-byte output holds exactly the packed
    codes, in the operand order of the expanded weights, with the same steps."""
    X = synth.activations(M, K, seed=600 + M)
    inv_s = synth.random_scales(K, seed=K + 3, lo=0.25, hi=4.0)
    fl = w4.W4A4_FLAG_GELU if gelu else 0
    qp, sp = w4.w4a4_quantize_act(bf16_dev(X), dev(inv_s), fl)
    qu, su = w4.w4a4_quantize_act(bf16_dev(X), dev(inv_s), fl | UNPACKED)
    assert tuple(qu.shape) == (M, K)
    codes = oracle.unpack_int4(host(qp), K)
    want = codes.reshape(M, K // 8, 8)[:, :, OPERAND_ORDER].reshape(M, K)
    assert np.array_equal(host(qu).view(np.int8), want)
    assert np.array_equal(host(sp), host(su))


@pytest.mark.parametrize("M,N,K", [(1, 256, 1024), (1374, 3072, 1024), (300, 1024, 4096)])
def test_unpacked_route_matches_packed_route(w4, M, N, K):
    """Same codes through both GEMM routes (widened per tile vs read one per
    byte): identical accumulators, so identical bf16 outputs; and the fused
    call gives the same output with the full and the minimum workspace."""
    X = synth.activations(M, K, seed=700 + M)
    W, b = synth.weights(N, K, seed=701), synth.bias(N, seed=702)
    pw = w4.w4a4_prepare_weights(bf16_dev(W), bf16_dev(b), bf16_dev(X[:synth.calibration_rows(M)]))
    qp, sp = w4.w4a4_quantize_act(bf16_dev(X), pw.inv_smooth, 0)
    qu, su = w4.w4a4_quantize_act(bf16_dev(X), pw.inv_smooth, UNPACKED)
    Yp = w4.w4a4_linear(qp, sp, pw)
    Yu = w4.w4a4_linear_ex(qu, su, pw, flags=UNPACKED)
    assert torch.equal(Yp.view(torch.int16), Yu.view(torch.int16))
    Xd = bf16_dev(X)
    small = torch.empty(w4.w4a4_workspace_bytes_min(M, K, 0), dtype=torch.uint8, device="cuda")
    Yf_small = w4.w4a4_linear_fused(Xd, pw, workspace=small)
    Yf_full = w4.w4a4_linear_fused(Xd, pw)
    assert torch.equal(Yf_small.view(torch.int16), Yp.view(torch.int16))
    assert torch.equal(Yf_full.view(torch.int16), Yp.view(torch.int16))
    assert w4.w4a4_get_device_status() == 0


# ------------------------------------------------- GELU on the output (W4A4_FLAG_GELU_OUT)
GELU_OUT = 0x10


@pytest.mark.parametrize("route", ["fused", "bytes", "expanded", "packed", "w8a8"])
def test_gelu_on_output(w4, route):
    """W4A4_FLAG_GELU_OUT gives, element by element, the oracle's GELU (exact
    erf in fp64, rounded to bf16) of the same call's output without the flag,
    on an fc1-shaped layer (K = 1024, N = 4096), through every GEMM route and
    the W8A8 setting.
    Below -5.9375 the kernel's GELU is the constant -5.9375 Phi(-5.9375)
    (-8.6e-9): the exact GELU there lies between it and 0."""
    M, N, K = 300, 4096, 1024
    X = synth.activations(M, K, seed=820)
    W, b = synth.weights(N, K, seed=821), synth.bias(N, seed=822)
    i8 = w4.W4A4_FLAG_INT8 if route == "w8a8" else 0
    pw = w4.w4a4_prepare_weights(bf16_dev(W), bf16_dev(b), bf16_dev(X[:synth.calibration_rows(M)]),
                                 flags=i8, expanded=(route != "packed"))
    Xd = bf16_dev(X)
    if route in ("fused", "w8a8"):
        Y0 = w4.w4a4_linear_fused(Xd, pw, flags=i8)
        Y1 = w4.w4a4_linear_fused(Xd, pw, flags=i8 | GELU_OUT)
    else:
        fl = UNPACKED if route == "bytes" else 0
        q, s = w4.w4a4_quantize_act(Xd, pw.inv_smooth, fl)
        Y0 = w4.w4a4_linear_ex(q, s, pw, flags=fl)
        Y1 = w4.w4a4_linear_ex(q, s, pw, flags=fl | GELU_OUT)
    y0 = host(Y0.view(torch.int16)).view(np.uint16)
    y1 = host(Y1.view(torch.int16)).view(np.uint16)
    want = oracle.gelu_bf16(y0)
    f0 = synth.bf16_bits_to_f32(y0).astype(np.float64)
    far = f0 < -5.9375
    assert far.sum() > 0 and (~far).sum() > 0.9 * f0.size   # both branches exercised
    assert np.array_equal(y1[~far], want[~far])
    f1 = synth.bf16_bits_to_f32(y1[far]).astype(np.float64)
    assert len(set(y1[far].tolist())) == 1
    assert np.all(f1 <= oracle.bf16_to_f64(want[far]))
    assert np.all(np.abs(f1) <= 1e-8 * np.abs(f0[far]))
    assert w4.w4a4_get_device_status() == 0


def test_mlp_gelu_placements_agree(w4):
    """An MLP pair (fc1 1024 -> 4096, GELU, fc2 4096 -> 1024): the GELU in
    fc1's epilogue (W4A4_FLAG_GELU_OUT) or in fc2's quantize kernel
    (W4A4_FLAG_GELU) gives the same fc2 output bits when both rotate with the
    same kernel, since both apply the same function to the same bf16 values."""
    M = 700
    X = synth.activations(M, 1024, seed=830)
    W1, b1 = synth.weights(4096, 1024, seed=831), synth.bias(4096, seed=832)
    W2, b2 = synth.weights(1024, 4096, seed=833), synth.bias(1024, seed=834)
    C = synth.calibration_rows(M)
    Xd = bf16_dev(X)
    pw1 = w4.w4a4_prepare_weights(bf16_dev(W1), bf16_dev(b1), bf16_dev(X[:C]))
    Y1 = w4.w4a4_linear_fused(Xd, pw1)
    G1 = w4.w4a4_linear_fused(Xd, pw1, flags=GELU_OUT)
    pw2 = w4.w4a4_prepare_weights(bf16_dev(W2), bf16_dev(b2), G1[:C].contiguous())
    Ya = w4.w4a4_linear_fused(Y1, pw2, flags=w4.W4A4_FLAG_GELU)
    # the GELU on fc2's input runs with the CUDA-core rotation; with the same
    # rotation on the other placement the outputs are identical bit for bit
    Yb = w4.w4a4_linear_fused(G1, pw2, flags=w4.W4A4_FLAG_FWHT)
    assert torch.equal(Ya.view(torch.int16), Yb.view(torch.int16))
    # the default (tensor-core) rotation of the same values differs only where
    # a code sits on a rounding tie
    Yc = w4.w4a4_linear_fused(G1, pw2)
    assert rel_fro(y_to_f64(Yc), y_to_f64(Ya)) < 1e-3
    assert w4.w4a4_get_device_status() == 0
