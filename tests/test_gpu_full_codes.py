"""Full-tensor checks of the quantize kernel's codes at the large workloads.

The oracle's rotation is a dense d x d product, too slow for every row of a
32-frame batch; here every row is rotated with the Kronecker-factored product
H_n R H_n (K = n^2, numpy fp64 matrix products; pinned to the oracle's dense
rotation on sampled rows), and the oracle's quantizer forms
the exact codes of
all M x K elements, in both of its decision modes (the fp64 quantizer the
pages define, and the binary32 decision), compared code by code with the
GPU's (bit-exact except
+-1 flips within the fp32 rounding-tie bound of tests/parity.py, at most 1e-4
of the codes).  Page "十亿参数的三维重建模型，能塞进手机吗？", sections
预全局旋转 / 后局部平滑 / 训练后量化（PTQ）.
"""
import numpy as np
import pytest
import scipy.linalg
import torch

import oracle
from w4a4_post_quantized_b200 import synth
from parity import act_transform, compare_codes, tie_bound

pytestmark = pytest.mark.gpu


def fwht_rows(X: np.ndarray) -> np.ndarray:
    """x H (natural-order Sylvester Hadamard, unnormalised) of every row, fp64.
    For K = n^2 the Sylvester matrix is H_n (x) H_n, so with a row folded into
    the n x n matrix R[a, b] = x[n a + b] the transform is H_n R H_n."""
    M, K = X.shape
    n = int(round(np.sqrt(K)))
    assert n * n == K
    Hn = scipy.linalg.hadamard(n).astype(np.float64)
    R = np.asarray(X, dtype=np.float64).reshape(M, n, n)
    return np.matmul(np.matmul(Hn, R), Hn).reshape(M, K)


@pytest.fixture(scope="module")
def w4():
    from w4a4_post_quantized_b200 import w4a4
    return w4a4


def test_fwht_helper_matches_the_oracle_rotation():
    X = oracle.bf16_to_f64(synth.activations(7, 1024, seed=3))
    np.testing.assert_allclose(fwht_rows(X) / 32.0, oracle.rotate(X), rtol=0, atol=1e-12)


@pytest.mark.parametrize("frames,K,gelu", [(32, 1024, False), (8, 4096, True), (8, 4096, False)])
def test_every_code_of_a_large_batch(w4, frames, K, gelu):
    M = frames * synth.FRAME_TOKENS
    X = synth.activations(M, K, seed=900 + K)
    inv_s = synth.random_scales(K, seed=901, lo=0.25, hi=4.0)
    flags = w4.W4A4_FLAG_GELU if gelu else 0
    Xd = torch.from_numpy(X.view(np.int16)).cuda().view(torch.bfloat16)
    qx, st = w4.w4a4_quantize_act(Xd, torch.from_numpy(inv_s).cuda(), flags)
    got = oracle.unpack_int4(qx.cpu().numpy(), K)
    st = st.cpu().numpy()
    del qx, Xd
    xin = oracle.bf16_to_f64(oracle.gelu_bf16(X) if gelu else X)
    hat = fwht_rows(xin) * (inv_s.astype(np.float64) / np.sqrt(K))[None, :]
    amax = np.max(np.abs(hat), axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(amax[:, None] > 0, hat * 7.0 / amax[:, None], 0.0)
    bound = tie_bound(xin, inv_s.astype(np.float64), ratio, amax, K, transform=act_transform(flags))
    if gelu:  # GELU in fp32 may land one bf16 step away from the fp64 GELU
        bound = bound + 4.0 * 2.0 ** -8 * np.max(np.abs(xin), axis=1) * np.max(inv_s) / np.sqrt(K) * 7.0 / np.maximum(amax, 1e-300)
    # the method as defined (fp64 decision), then the binary32 decision
    for decision in ("f64", "f32"):
        want_q, want_d = oracle.quantize_rows(hat, 4, decision)
        np.testing.assert_allclose(st, want_d, rtol=2e-5, atol=0)
        flips = compare_codes(got, want_q, ratio, bound, 1e-4)
        print(f"M={M} K={K} gelu={gelu} ({act_transform(flags)}): {flips} flips of {got.size} "
              f"against the {decision} decision")
        del want_q
    assert w4.w4a4_get_device_status() == 0
