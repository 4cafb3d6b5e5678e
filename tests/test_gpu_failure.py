"""Failure detection on the GPU without a fault: a bounded wait that runs out.

Every wait inside the library's kernels is bounded; one that runs out sets
W4A4_DEV_TIMEOUT in the device status word and the kernel drains its copies,
frees its tensor memory and returns.  w4a4_gemm_s32_ex with W4A4_DEBUG_STALL
makes that happen on purpose: the GEMM's TMA producer issues no copy and the
launch's waits are limited to 1 ms, so the MMA issuer's (and the widen warps')
first wait expires.  Each case checks, through the C ABI, that the call
returns, that the host reads the status bit, that clearing it works, and that
the next normal call on the same context is bit-exact against the oracle's
int64 product again.
"""
import numpy as np
import pytest
import torch

import oracle
from w4a4_post_quantized_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def w4():
    from w4a4_post_quantized_b200 import w4a4
    return w4a4


def _weights(w4, B, K, route):
    """Weights holding packed codes B for the widening routes, or their 8-bit
    values for the W8A8 route."""
    if route == "int8":
        pw = w4.PreparedWeights(B.shape[0], K, int8=True)
        pw.qw8.copy_(torch.from_numpy(oracle.unpack_int4(B, K)).cuda())
        pw.struct.flags = w4.W4A4_FLAG_INT8
        return pw
    pw = w4.PreparedWeights(B.shape[0], K, expanded=(route != "packed"))
    pw.qw.copy_(torch.from_numpy(B).cuda())
    if route != "packed":
        w4.w4a4_expand_weights(pw)
    return pw


@pytest.mark.parametrize("route", ["expanded", "packed", "int8", "unpacked"])
def test_stalled_gemm_reports_timeout_then_recovers(w4, route):
    M, N, K = 700, 512, 1024
    A = synth.random_packed_codes(M, K, seed=71)
    B = synth.random_packed_codes(N, K, seed=72)
    pw = _weights(w4, B, K, route)
    codes = oracle.unpack_int4(A, K)
    if route == "int8":
        qx, flags = codes.view(np.uint8), 0
    elif route == "unpacked":   # one code per byte in the expanded weights' operand order
        perm = np.array([0, 2, 4, 6, 1, 3, 5, 7])
        qx = codes.reshape(M, K // 8, 8)[:, :, perm].reshape(M, K).view(np.uint8)
        flags = w4.W4A4_FLAG_UNPACKED
    else:
        qx, flags = A, 0
    qx = torch.from_numpy(np.ascontiguousarray(qx)).cuda()
    w4.w4a4_clear_device_status()
    assert w4.w4a4_get_device_status() == 0
    w4.w4a4_gemm_s32_ex(qx, pw, flags=flags | w4.W4A4_DEBUG_STALL)
    torch.cuda.synchronize()        # the stalled launch returned
    assert w4.w4a4_get_device_status() & w4.W4A4_DEV_TIMEOUT
    w4.w4a4_clear_device_status()
    assert w4.w4a4_get_device_status() == 0
    acc = w4.w4a4_gemm_s32_ex(qx, pw, flags=flags).cpu().numpy()
    assert w4.w4a4_get_device_status() == 0
    want = oracle.int_gemm(codes, oracle.unpack_int4(B, K))
    assert np.array_equal(acc.astype(np.int64), want)
