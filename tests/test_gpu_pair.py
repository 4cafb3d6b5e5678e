"""The CTA-pair GEMM (byte operands, enough tiles): two CTAs of a cluster
share a 256 x 256 tile, each loading its 128 rows of A and of B, the leader
issuing cta_group::2 MMAs.

  * accumulators bit-exact against the oracle's int64 product, with a ragged
    last pair tile (the second CTA's half partly or wholly past M), several
    tiles per pair, 4-bit and 8-bit codes;
  * bf16 outputs (with and without the GELU on the output) identical bit for
    bit to the widening route's, which takes one CTA per tile;
  * a stalled launch (no copy issued, 1 ms waits) reports the timeout and
    the next call is exact again.
"""
import numpy as np
import pytest
import torch

import oracle
from w4a4_post_quantized_b200 import synth

pytestmark = pytest.mark.gpu
K = 4096
PERM = np.array([0, 2, 4, 6, 1, 3, 5, 7])   # operand order of one-per-byte 4-bit codes


@pytest.fixture(scope="module")
def w4():
    from w4a4_post_quantized_b200 import w4a4
    return w4a4


def _bytes(codes):
    M = codes.shape[0]
    return torch.from_numpy(np.ascontiguousarray(
        codes.reshape(M, K // 8, 8)[:, :, PERM].reshape(M, K).view(np.uint8))).cuda()


def _weights4(w4, B):
    pw = w4.PreparedWeights(B.shape[0], K, expanded=True)
    pw.qw.copy_(torch.from_numpy(B).cuda())
    w4.w4a4_expand_weights(pw)
    return pw


# 2500 = 9 x 256 + 196: the last pair tile's second half is partly past M;
# 2330 = 9 x 256 + 26: wholly past M; 10992: 43 x 4 pair tiles, several per pair
@pytest.mark.parametrize("M", [2500, 2330, 10992])
def test_pair_gemm_s32_bit_exact(w4, M):
    N = 1024
    A = synth.random_packed_codes(M, K, seed=M + 901)
    B = synth.random_packed_codes(N, K, seed=902)
    pw = _weights4(w4, B)
    codes = oracle.unpack_int4(A, K)
    acc = w4.w4a4_gemm_s32_ex(_bytes(codes), pw, flags=w4.W4A4_FLAG_UNPACKED).cpu().numpy()
    want = oracle.int_gemm(codes, oracle.unpack_int4(B, K))
    assert np.array_equal(acc.astype(np.int64), want)
    assert w4.w4a4_get_device_status() == 0


def test_pair_gemm_s32_int8_bit_exact(w4):
    M, N = 2500, 1024
    rng = np.random.default_rng(903)
    A8 = rng.integers(-127, 128, size=(M, K), dtype=np.int64)
    B8 = rng.integers(-127, 128, size=(N, K), dtype=np.int64)
    A8[:3] = 127                                  # extreme rows: |acc| = 127^2 K
    B8[:2] = -127
    pw = w4.PreparedWeights(N, K, int8=True)
    pw.qw8.copy_(torch.from_numpy(B8.astype(np.int8)).cuda())
    pw.struct.flags = w4.W4A4_FLAG_INT8
    qx = torch.from_numpy(A8.astype(np.int8).view(np.uint8)).cuda()
    acc = w4.w4a4_gemm_s32_ex(qx, pw).cpu().numpy()
    assert np.array_equal(acc.astype(np.int64), A8 @ B8.T)
    assert w4.w4a4_get_device_status() == 0


@pytest.mark.parametrize("gelu", [False, True])
@pytest.mark.parametrize("k,N", [(K, 1024), (1024, 4096)])
def test_pair_outputs_equal_the_widening_route(w4, gelu, k, N):
    """fc2-shaped (K = 4096) and fc1-shaped (K = 1024, N = 4096: the stack's
    GELU layer) pair launches against the widening route, bit for bit."""
    M = 2500
    X = synth.activations(M, k, seed=904)
    W, b = synth.weights(N, k, seed=905), synth.bias(N, seed=906)
    bf = lambda a: torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    pw = w4.w4a4_prepare_weights(bf(W), bf(b), bf(X[:synth.calibration_rows(M)]))
    fl = w4.W4A4_FLAG_GELU_OUT if gelu else 0
    qp, sp = w4.w4a4_quantize_act(bf(X), pw.inv_smooth, 0)
    qu, su = w4.w4a4_quantize_act(bf(X), pw.inv_smooth, w4.W4A4_FLAG_UNPACKED)
    Yp = w4.w4a4_linear_ex(qp, sp, pw, flags=fl)                                # one CTA per tile
    Yu = w4.w4a4_linear_ex(qu, su, pw, flags=fl | w4.W4A4_FLAG_UNPACKED)        # CTA pairs
    assert torch.equal(Yp.view(torch.int16), Yu.view(torch.int16))
    assert w4.w4a4_get_device_status() == 0


def test_pair_stall_reports_timeout_then_recovers(w4):
    M, N = 2500, 1024
    A = synth.random_packed_codes(M, K, seed=907)
    B = synth.random_packed_codes(N, K, seed=908)
    pw = _weights4(w4, B)
    codes = oracle.unpack_int4(A, K)
    qx = _bytes(codes)
    w4.w4a4_clear_device_status()
    w4.w4a4_gemm_s32_ex(qx, pw, flags=w4.W4A4_FLAG_UNPACKED | w4.W4A4_DEBUG_STALL)
    torch.cuda.synchronize()
    assert w4.w4a4_get_device_status() & w4.W4A4_DEV_TIMEOUT
    w4.w4a4_clear_device_status()
    acc = w4.w4a4_gemm_s32_ex(qx, pw, flags=w4.W4A4_FLAG_UNPACKED).cpu().numpy()
    assert w4.w4a4_get_device_status() == 0
    assert np.array_equal(acc.astype(np.int64), oracle.int_gemm(codes, oracle.unpack_int4(B, K)))
