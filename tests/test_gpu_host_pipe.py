"""The host-buffer entry point: w4a4_linear_fused_host on pinned host memory
must give exactly the rows w4a4_linear_fused gives on device memory (the same
kernels on independent rows), for chunkings that split M evenly, raggedly or
not at all, across repeated calls on one pipe."""
import numpy as np
import pytest
import torch

from w4a4_post_quantized_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def w4():
    from w4a4_post_quantized_b200 import w4a4
    return w4a4


def bf16(bits, device):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


@pytest.mark.parametrize("M,N,K,chunk,gelu", [(10992, 3072, 1024, 2816, False), (1000, 512, 1024, 384, False),
                                              (100, 256, 4096, 2816, True), (1374, 1024, 1024, 128, False),
                                              (1000, 4096, 1024, 384, "out")])
def test_host_pipeline_matches_device_call(w4, M, N, K, chunk, gelu):
    X = synth.activations(M, K, seed=M + K)
    W, b = synth.weights(N, K, seed=5), synth.bias(N, seed=6)
    pw = w4.w4a4_prepare_weights(bf16(W, "cuda"), bf16(b, "cuda"), bf16(X[:synth.calibration_rows(M)], "cuda"))
    # gelu: on the input (True), on the output ("out", an MLP's fc1), or none
    flags = {False: 0, True: w4.W4A4_FLAG_GELU, "out": w4.W4A4_FLAG_GELU_OUT}[gelu]
    want = w4.w4a4_linear_fused(bf16(X, "cuda"), pw, flags=flags).cpu()
    Xh = bf16(X, "cpu").pin_memory()
    pipe = w4.HostPipe()
    ws = torch.empty(w4.w4a4_host_workspace_bytes(chunk, K, N), dtype=torch.uint8, device="cuda")
    for rep in range(2):  # the pipe and workspace are reused across calls
        Yh = torch.full((M, N), float("nan"), dtype=torch.bfloat16).pin_memory()
        w4.w4a4_linear_fused_host(Xh, pw, Y_host=Yh, chunk_rows=chunk, workspace=ws, pipe=pipe, flags=flags)
        torch.cuda.current_stream().synchronize()
        assert torch.equal(Yh.view(torch.int16), want.view(torch.int16)), rep
    assert w4.w4a4_get_device_status() == 0
    pipe.close()


@pytest.mark.parametrize("side", ["x_device", "y_device"])
def test_host_pipeline_with_one_side_on_the_device(w4, side):
    """W4A4_FLAG_X_DEVICE / W4A4_FLAG_Y_DEVICE: the first layer of a stack
    reads X from host memory and leaves Y on the device, the last one reads a
    device X and writes host memory; the rows are again those of the device
    call, bit for bit."""
    M, N, K, chunk = 3000, 1024, 1024, 1408
    X = synth.activations(M, K, seed=77)
    W, b = synth.weights(N, K, seed=78), synth.bias(N, seed=79)
    pw = w4.w4a4_prepare_weights(bf16(W, "cuda"), bf16(b, "cuda"), bf16(X[:synth.calibration_rows(M)], "cuda"))
    Xd = bf16(X, "cuda")
    want = w4.w4a4_linear_fused(Xd, pw)
    Xh = bf16(X, "cpu").pin_memory()   # kept alive until the copies have run
    pipe = w4.HostPipe()
    ws = torch.empty(w4.w4a4_host_workspace_bytes(chunk, K, N), dtype=torch.uint8, device="cuda")
    for rep in range(2):
        if side == "x_device":
            Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16).pin_memory()
            w4.w4a4_linear_fused_host(Xd, pw, Y_host=Y, chunk_rows=chunk, workspace=ws, pipe=pipe,
                                      flags=w4.W4A4_FLAG_X_DEVICE)
        else:
            Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
            w4.w4a4_linear_fused_host(Xh, pw, Y_host=Y, chunk_rows=chunk,
                                      workspace=ws, pipe=pipe, flags=w4.W4A4_FLAG_Y_DEVICE)
        torch.cuda.current_stream().synchronize()
        assert torch.equal(Y.cpu().view(torch.int16), want.cpu().view(torch.int16)), rep
    assert w4.w4a4_get_device_status() == 0
    pipe.close()
