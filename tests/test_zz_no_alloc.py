"""The allocation-free fused linear, w4a4_linear_fused_noalloc.

Some callers cannot allocate device memory where they call the layer (a
serving loop or plugin host that forbids cudaMalloc / cudaFree after start-up,
cudaFree synchronizing the whole device, or a C caller holding only the buffers
another runtime gave it).  For them the library keeps its own scratch array
instead of taking a workspace.  This file checks, through the C ABI, that the
entry point gives the same output as w4a4_linear_fused with a caller-owned
workspace, on two calls in a row (the scratch keeps the previous call's
contents), and that it refuses sizes beyond its scratch.  The file name makes
pytest collect it last.
"""
import ctypes
import os

import numpy as np
import pytest
import torch

from w4a4_post_quantized_b200 import synth

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bf16(bits):
    return torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)


def test_noalloc_matches_workspace_path_twice():
    from w4a4_post_quantized_b200 import w4a4
    lib = ctypes.CDLL(os.path.join(ROOT, "w4a4_post_quantized_b200", "libw4a4.so"))
    fn = lib.w4a4_linear_fused_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.POINTER(w4a4.W4A4WeightsT),
                   ctypes.c_void_p, ctypes.c_uint32, ctypes.c_void_p]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    N, K = 1024, 1024
    W = _bf16(synth.weights(N, K, seed=41))
    b = _bf16(synth.bias(N, seed=42))
    # two different inputs of different lengths: the second call must not see
    # anything left in the scratch by the first
    for M, seed in [(3000, 43), (1374, 44)]:
        X = _bf16(synth.activations(M, K, seed=seed))
        pw = w4a4.w4a4_prepare_weights(W, b, X[:synth.calibration_rows(M)])
        want = w4a4.w4a4_linear_fused(X, pw)
        got = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        rc = fn(ctypes.c_void_p(X.data_ptr()), M, ctypes.byref(pw.struct),
                ctypes.c_void_p(got.data_ptr()), 0, stream)
        assert rc == 0
        torch.cuda.synchronize()
        # same kernels on the same inputs: the outputs agree exactly (well inside
        # the 2e-3 relative Frobenius bound the other parity tests use)
        g, w_ = got.float().cpu().numpy(), want.float().cpu().numpy()
        assert np.isfinite(g).all()
        assert np.linalg.norm(g - w_) <= 2e-3 * np.linalg.norm(w_)
        assert np.array_equal(g, w_)
    assert w4a4.w4a4_get_device_status() == 0


SCRATCH = 8 << 20   # W4A4_NOALLOC_SCRATCH_BYTES


@pytest.mark.parametrize("M,K,route", [(12000, 1024, "packed"), (16256, 1024, "packed"),
                                       (4088, 4096, "packed"), (2000, 4096, "one per byte")])
def test_noalloc_at_its_limits_matches_same_route(M, K, route):
    """Up to about half of the scratch the codes go one per byte; beyond that,
    up to the largest M the scratch holds (16256 tokens at K = 1024, 4088 at
    K = 4096, where the per-token steps end within bytes of the array's end),
    they go packed two per byte.  w4a4_linear_fused given a caller workspace of
    exactly the scratch's size takes the same route, so the two outputs are
    identical bit for bit, on two calls in a row."""
    from w4a4_post_quantized_b200 import w4a4
    lib = ctypes.CDLL(os.path.join(ROOT, "w4a4_post_quantized_b200", "libw4a4.so"))
    fn = lib.w4a4_linear_fused_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.POINTER(w4a4.W4A4WeightsT),
                   ctypes.c_void_p, ctypes.c_uint32, ctypes.c_void_p]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    one_per_byte = w4a4.w4a4_workspace_bytes(M, K) <= SCRATCH
    assert one_per_byte == (route == "one per byte")
    assert w4a4.w4a4_workspace_bytes_min(M, K, 0) <= SCRATCH
    N = 256
    W = _bf16(synth.weights(N, K, seed=51))
    b = _bf16(synth.bias(N, seed=52))
    ws = torch.empty(SCRATCH, dtype=torch.uint8, device="cuda")
    gelu = w4a4.W4A4_FLAG_GELU if K == 4096 else 0
    for seed in (53, 54):
        X = _bf16(synth.activations(M, K, seed=seed))
        pw = w4a4.w4a4_prepare_weights(W, b, X[:synth.calibration_rows(M)])
        want = w4a4.w4a4_linear_fused(X, pw, workspace=ws, flags=gelu)
        got = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        rc = fn(ctypes.c_void_p(X.data_ptr()), M, ctypes.byref(pw.struct),
                ctypes.c_void_p(got.data_ptr()), gelu, stream)
        assert rc == 0
        torch.cuda.synchronize()
        assert torch.equal(got.view(torch.int16), want.view(torch.int16))
    assert w4a4.w4a4_get_device_status() == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    from w4a4_post_quantized_b200 import w4a4
    lib = ctypes.CDLL(os.path.join(ROOT, "w4a4_post_quantized_b200", "libw4a4.so"))
    fn = lib.w4a4_linear_fused_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.POINTER(w4a4.W4A4WeightsT),
                   ctypes.c_void_p, ctypes.c_uint32, ctypes.c_void_p]
    pw = w4a4.PreparedWeights(256, 4096)
    X = torch.zeros((4089, 4096), dtype=torch.bfloat16, device="cuda")
    Y = torch.empty((4089, 256), dtype=torch.bfloat16, device="cuda")
    rc = fn(ctypes.c_void_p(X.data_ptr()), 4089, ctypes.byref(pw.struct), ctypes.c_void_p(Y.data_ptr()),
            0, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == w4a4.W4A4_ERR_SHAPE
    pw = w4a4.PreparedWeights(256, 1024)
    X = torch.zeros((16257, 1024), dtype=torch.bfloat16, device="cuda")
    Y = torch.empty((16257, 256), dtype=torch.bfloat16, device="cuda")
    rc = fn(ctypes.c_void_p(X.data_ptr()), 16257, ctypes.byref(pw.struct), ctypes.c_void_p(Y.data_ptr()),
            0, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == w4a4.W4A4_ERR_SHAPE
