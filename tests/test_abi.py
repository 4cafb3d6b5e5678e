"""C-ABI checks that need no GPU: libw4a4.so loads, exports every function
include/w4a4.h declares, and rejects bad arguments on the host (before any
CUDA call) with the documented status codes."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "w4a4.h")
LIB = os.path.join(ROOT, "w4a4_post_quantized_b200", "libw4a4.so")


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB):
        from w4a4_post_quantized_b200 import build
        build.build()
    return ctypes.CDLL(LIB)


def declared_functions():
    """Every function any include/*.h declares."""
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        names |= set(re.findall(r"\b((?:w4a4|tq)_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ["w4a4_prepare_weights", "w4a4_quantize_act", "w4a4_linear", "w4a4_linear_fused",
              "w4a4_workspace_bytes", "w4a4_gemm_s32", "w4a4_get_device_status",
              "tq_codebook", "tq_encode", "tq_decode"]:
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for n in declared_functions():
        assert hasattr(lib, n), f"{n} declared in w4a4.h but not exported by libw4a4.so"


def test_status_codes_match_binding():
    text = open(HEADER).read()
    codes = dict((k, int(v)) for k, v in re.findall(r"(W4A4_(?:OK|ERR_[A-Z]+))\s*=\s*(\d+)", text))
    assert codes == {"W4A4_OK": 0, "W4A4_ERR_ARG": 1, "W4A4_ERR_SHAPE": 2, "W4A4_ERR_ALIGN": 3,
                     "W4A4_ERR_UNSUPPORTED": 4, "W4A4_ERR_CUDA": 5, "W4A4_ERR_TIMEOUT": 6}


class WeightsT(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int32), ("K", ctypes.c_int32), ("qw", ctypes.c_void_p),
                ("scale_ch", ctypes.c_void_p), ("bias", ctypes.c_void_p),
                ("smooth", ctypes.c_void_p), ("inv_smooth", ctypes.c_void_p),
                ("qw8", ctypes.c_void_p), ("colsum", ctypes.c_void_p), ("flags", ctypes.c_uint32)]


A = 0x10000  # fake, 16-byte aligned device addresses: never dereferenced on the host


def _setup(lib):
    vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
    lib.w4a4_workspace_bytes.restype = ctypes.c_size_t
    lib.w4a4_workspace_bytes.argtypes = [i64, i32]
    lib.w4a4_workspace_bytes_min.restype = ctypes.c_size_t
    lib.w4a4_workspace_bytes_min.argtypes = [i64, i32, ctypes.c_uint32]
    lib.w4a4_linear_ex.argtypes = [vp, vp, i64, ctypes.POINTER(WeightsT), vp, ctypes.c_uint32, vp]
    lib.w4a4_quantize_act.argtypes = [vp, i64, i32, vp, vp, vp, ctypes.c_uint32, vp]
    lib.w4a4_linear.argtypes = [vp, vp, i64, ctypes.POINTER(WeightsT), vp, vp]
    lib.w4a4_linear_fused.argtypes = [vp, i64, ctypes.POINTER(WeightsT), vp, vp, ctypes.c_size_t,
                                      ctypes.c_uint32, vp]
    lib.w4a4_prepare_weights.argtypes = [vp, vp, i32, i32, vp, i64, ctypes.c_float, ctypes.c_uint32,
                                         ctypes.POINTER(WeightsT), vp]
    lib.w4a4_gemm_s32.argtypes = [vp, i64, ctypes.POINTER(WeightsT), vp, vp]
    lib.w4a4_expand_weights.argtypes = [ctypes.POINTER(WeightsT), vp]
    lib.w4a4_status_string.restype = ctypes.c_char_p
    lib.w4a4_version.restype = ctypes.c_char_p


def _weights(N=1024, K=1024, base=A, flags=0, expanded=True):
    return WeightsT(N, K, base, base + 0x1000, base + 0x2000, base + 0x3000, base + 0x4000,
                    base + 0x5000 if expanded else None, base + 0x6000 if expanded else None, flags)


def test_workspace_bytes(lib):
    _setup(lib)
    # the fast route's size: one code byte per element, then the steps
    assert lib.w4a4_workspace_bytes(10992, 1024) == 10992 * 1024 + 4 * 10992
    assert lib.w4a4_workspace_bytes(3, 4096) == 12288 + 12
    assert lib.w4a4_workspace_bytes(0, 1024) == 0
    assert lib.w4a4_workspace_bytes(10, 1000) == 0
    assert lib.w4a4_workspace_bytes(-1, 1024) == 0
    mn = lib.w4a4_workspace_bytes_min
    # packed int4 codes: two per byte, rounded up to 256, then the steps
    assert mn(10992, 1024, 0) == ((10992 * 512 + 255) // 256) * 256 + 4 * 10992
    assert mn(3, 4096, 0) == mn(3, 4096, 1) == mn(3, 4096, 2) == 6144 + 12
    for M, K in [(10992, 1024), (3, 4096), (0, 1024)]:
        assert mn(M, K, 4) == mn(M, K, 8) == mn(M, K, 4 | 2) == lib.w4a4_workspace_bytes(M, K)
    assert mn(10, 1024, 0x80) == 0 and mn(10, 1000, 4) == 0


INT8 = 0x4


def _weights8(N=1024, K=1024, base=A, flags=INT8):
    # 8-bit weights: codes in qw8, no packed qw and no colsum
    return WeightsT(N, K, None, base + 0x1000, base + 0x2000, base + 0x3000, base + 0x4000,
                    base + 0x5000, None, flags)


def test_int8_variant_argument_checks(lib):
    """W4A4_FLAG_INT8 (W8A8): weights need qw8 only; the flag must match between
    the weights and the fused call; expand_weights refuses 8-bit weights; the
    workspace check uses the 8-bit code size."""
    _setup(lib)
    w8 = _weights8()
    L, F, G, E, P = (lib.w4a4_linear, lib.w4a4_linear_fused, lib.w4a4_gemm_s32,
                     lib.w4a4_expand_weights, lib.w4a4_prepare_weights)
    assert L(A, A, 0, ctypes.byref(w8), A, None) == 0                    # accepted (empty: no-op)
    no_codes = _weights8()
    no_codes.qw8 = None
    assert L(A, A, 10, ctypes.byref(no_codes), A, None) == 1
    assert G(A, 0, ctypes.byref(w8), A, None) == 0
    assert G(A, 10, ctypes.byref(no_codes), A, None) == 1
    need4 = lib.w4a4_workspace_bytes_min(100, 1024, 0)
    need8 = lib.w4a4_workspace_bytes_min(100, 1024, INT8)
    assert F(A, 100, ctypes.byref(w8), A, A, need8, 0, None) == 1       # flag missing on the call
    assert F(A, 100, ctypes.byref(_weights()), A, A, need8, INT8, None) == 1  # 4-bit weights
    assert F(A, 100, ctypes.byref(w8), A, A, need4, INT8, None) == 2    # 4-bit-sized workspace
    assert E(ctypes.byref(_weights(flags=INT8)), None) == 1
    assert P(A, None, 1024, 1024, A, 10, 0.5, INT8, ctypes.byref(no_codes), None) == 1
    assert P(A, None, 1024, 1024, A, 10, 0.5, 0x8, ctypes.byref(w8), None) == 4   # unknown flag
    q = lib.w4a4_quantize_act
    assert q(A, 0, 1024, A, A, A, INT8, None) == 0
    assert q(A, 10, 1024, None, A, A, INT8, None) == 1                   # DSFQ needs inv_smooth


UNPACKED = 0x8


def test_unpacked_codes_argument_checks(lib):
    """W4A4_FLAG_UNPACKED: int4 codes one per byte for quantize_act and
    linear_ex; needs 4-bit weights with their expanded copy; not a flag of
    the fused call (which picks its route from the workspace size)."""
    _setup(lib)
    q, LX, F = lib.w4a4_quantize_act, lib.w4a4_linear_ex, lib.w4a4_linear_fused
    assert q(A, 0, 1024, A, A, A, UNPACKED, None) == 0
    assert q(A, 10, 1024, A, A, A, UNPACKED | INT8, None) == 4
    w = _weights()
    assert LX(A, A, 0, ctypes.byref(w), A, UNPACKED, None) == 0
    assert LX(A, A, 0, ctypes.byref(w), A, 0, None) == 0
    assert LX(A, A, 10, ctypes.byref(w), A, 0x1, None) == 4                      # GELU: not a GEMM flag
    assert LX(A, A, 10, ctypes.byref(_weights(expanded=False)), A, UNPACKED, None) == 1  # no qw8
    assert LX(A, A, 10, ctypes.byref(_weights8()), A, UNPACKED, None) == 1       # 8-bit weights
    full = lib.w4a4_workspace_bytes(100, 1024)
    assert F(A, 100, ctypes.byref(w), A, A, full, UNPACKED, None) == 4
    assert F(A, 100, ctypes.byref(w), A, A, lib.w4a4_workspace_bytes_min(100, 1024, 0) - 1, 0, None) == 2


def test_gelu_out_argument_checks(lib):
    """W4A4_FLAG_GELU_OUT (0x10): the GELU on a linear's output; a flag of
    linear_ex and linear_fused, not of the activation quantizer; the workspace
    sizes do not depend on it."""
    _setup(lib)
    q, LX, F = lib.w4a4_quantize_act, lib.w4a4_linear_ex, lib.w4a4_linear_fused
    GOUT = 0x10
    assert q(A, 10, 1024, A, A, A, GOUT, None) == 4
    w = _weights()
    assert LX(A, A, 0, ctypes.byref(w), A, GOUT, None) == 0
    assert LX(A, A, 0, ctypes.byref(w), A, GOUT | UNPACKED, None) == 0
    assert LX(A, A, 10, ctypes.byref(w), A, GOUT | 0x20, None) == 4
    assert F(A, 0, ctypes.byref(w), A, A, 0, GOUT | 0x1, None) == 0          # with the input GELU too
    assert F(A, 100, ctypes.byref(w), A, A, 16, GOUT, None) == 2              # workspace too small
    for K in (1024, 4096):
        assert lib.w4a4_workspace_bytes_min(100, K, GOUT) == lib.w4a4_workspace_bytes_min(100, K, 0)


def test_quantize_act_argument_checks(lib):
    _setup(lib)
    q = lib.w4a4_quantize_act
    assert q(A, 10, 1000, A, A, A, 0, None) == 4                 # K unsupported
    assert q(A, 10, 1024, A, A, A, 0x80, None) == 4              # unknown flag
    assert q(None, 10, 1024, A, A, A, 0, None) == 1              # null X
    assert q(A, 10, 1024, None, A, A, 0, None) == 1              # null inv_smooth (DSFQ)
    assert q(A + 8, 10, 1024, A, A, A, 0, None) == 3             # misaligned X
    assert q(A, -1, 1024, A, A, A, 0, None) == 2                 # negative M
    assert q(A, 1 << 31, 1024, A, A, A, 0, None) == 2            # M too large
    assert q(A, 0, 1024, A, A, A, 0, None) == 0                  # empty input: no-op
    assert q(A, 0, 4096, None, A, A, 2, None) == 0               # plain: inv_smooth may be null


def test_linear_argument_checks(lib):
    _setup(lib)
    w = _weights()
    L = lib.w4a4_linear
    assert L(A, A, 10, None, A, None) == 1
    assert L(A, A, 10, ctypes.byref(_weights(N=1000)), A, None) == 2
    assert L(A, A, 10, ctypes.byref(_weights(K=2048)), A, None) == 4
    assert L(A, A, 10, ctypes.byref(_weights(base=A + 4)), A, None) == 3
    assert L(A, A, 10, ctypes.byref(_weights(flags=0x10)), A, None) == 4
    assert L(None, A, 10, ctypes.byref(w), A, None) == 1
    assert L(A, A, 10, ctypes.byref(w), A + 2, None) == 3
    assert L(A, A, 0, ctypes.byref(w), A, None) == 0


def test_linear_fused_argument_checks(lib):
    _setup(lib)
    w = _weights()
    F = lib.w4a4_linear_fused
    need = lib.w4a4_workspace_bytes_min(100, 1024, 0)
    assert F(A, 100, ctypes.byref(w), A, A, need - 1, 0, None) == 2     # workspace too small
    assert F(A, 100, ctypes.byref(w), A, A, need, 2, None) == 1         # plain flag vs DSFQ weights
    assert F(A, 100, ctypes.byref(w), A, None, need, 0, None) == 1
    assert F(A, 100, ctypes.byref(w), A, A + 1, need, 0, None) == 3
    assert F(A, 0, ctypes.byref(w), A, A, 0, 0, None) == 0


def test_prepare_and_gemm_argument_checks(lib):
    _setup(lib)
    P = lib.w4a4_prepare_weights
    w = _weights()
    assert P(A, None, 1024, 1024, A, 10, 0.5, 0, ctypes.byref(_weights(N=512)), None) == 2
    assert P(A, None, 1024, 1024, None, 10, 0.5, 0, ctypes.byref(w), None) == 1
    assert P(A, None, 1024, 1024, A, 0, 0.5, 0, ctypes.byref(w), None) == 1
    assert P(A, None, 1024, 1024, A, 10, 1.5, 0, ctypes.byref(w), None) == 1
    assert P(A, None, 1024, 1024, A, 10, float("nan"), 0, ctypes.byref(w), None) == 1
    assert P(A, None, 1024, 1000, A, 10, 0.5, 0, ctypes.byref(w), None) == 4
    assert P(A, None, 100, 1024, A, 10, 0.5, 0, ctypes.byref(w), None) == 2
    assert P(A + 2, None, 1024, 1024, A, 10, 0.5, 0, ctypes.byref(w), None) == 3
    G = lib.w4a4_gemm_s32
    w = _weights()
    assert G(A, 10, ctypes.byref(w), None, None) == 1
    assert G(A, 10, None, A, None) == 1
    assert G(A, 10, ctypes.byref(_weights(N=1000)), A, None) == 2
    assert G(A, 10, ctypes.byref(_weights(K=64)), A, None) == 4
    assert G(A, 10, ctypes.byref(_weights(base=A + 8)), A, None) == 3
    assert G(A, 0, ctypes.byref(w), A, None) == 0
    half = _weights()
    half.colsum = None                                    # qw8 without colsum
    assert G(A, 10, ctypes.byref(half), A, None) == 1
    E = lib.w4a4_expand_weights
    assert E(None, None) == 1
    assert E(ctypes.byref(_weights(expanded=False)), None) == 1
    assert E(ctypes.byref(_weights(K=2048)), None) == 4
    assert E(ctypes.byref(_weights(base=A + 4)), None) == 3


def test_status_strings(lib):
    _setup(lib)
    assert lib.w4a4_status_string(0) == b"ok"
    assert lib.w4a4_status_string(6) == b"device wait timed out"
    assert b"sm_100a" in lib.w4a4_version()


def test_host_pipeline_argument_checks(lib):
    """w4a4_linear_fused_host rejects bad arguments before touching the pipe or
    the GPU; w4a4_host_workspace_bytes follows its documented layout."""
    vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
    lib.w4a4_host_workspace_bytes.restype = sz
    lib.w4a4_host_workspace_bytes.argtypes = [i64, i32, i32]
    lib.w4a4_workspace_bytes.restype = sz
    lib.w4a4_workspace_bytes.argtypes = [i64, i32]
    r256 = lambda b: (b + 255) // 256 * 256
    for rows, K, N in [(2816, 1024, 3072), (1, 4096, 1024), (300, 1024, 256)]:
        # the codes part has room for one code byte per element (every route fits)
        slot = r256(2 * rows * K) + r256(2 * rows * N) + r256(lib.w4a4_workspace_bytes(rows, K))
        assert lib.w4a4_host_workspace_bytes(rows, K, N) == 2 * slot
    assert lib.w4a4_host_workspace_bytes(0, 1024, 256) == 0
    f = lib.w4a4_linear_fused_host
    f.restype = ctypes.c_int
    f.argtypes = [vp, i64, ctypes.POINTER(WeightsT), vp, i64, vp, sz, vp, ctypes.c_uint32, vp]
    w = WeightsT(256, 1024, A, A, A, A, A, None, None, 0)
    need = lib.w4a4_host_workspace_bytes(128, 1024, 256)
    fake_pipe = vp(A)  # never dereferenced on these paths
    assert f(A, 10, ctypes.byref(w), A, 128, A, need, None, 0, None) == 1        # no pipe
    assert f(A, 10, None, A, 128, A, need, fake_pipe, 0, None) == 1              # no weights
    assert f(A, 0, ctypes.byref(w), A, 128, A, need, fake_pipe, 0, None) == 0    # empty: no-op
    assert f(A, 10, ctypes.byref(w), A, 0, A, need, fake_pipe, 0, None) == 2     # chunk_rows 0
    assert f(A, -1, ctypes.byref(w), A, 128, A, need, fake_pipe, 0, None) == 2   # negative M
    assert f(None, 10, ctypes.byref(w), A, 128, A, need, fake_pipe, 0, None) == 1
    assert f(A, 10, ctypes.byref(w), A, 128, A + 4, need, fake_pipe, 0, None) == 3  # misaligned
    assert f(A, 10, ctypes.byref(w), A, 128, A, need - 1, fake_pipe, 0, None) == 2  # too small


def test_tq_codebook_and_argument_checks(lib):
    """The codec's host codebook (no GPU needed) matches the oracle's Lloyd-Max
    to fp32 rounding; encode / decode reject bad arguments on the host."""
    import numpy as np
    from oracle import turboquant as tq
    f32 = ctypes.POINTER(ctypes.c_float)
    lib.tq_codebook.argtypes = [ctypes.c_int32, ctypes.c_int32, f32, f32]
    c = np.empty(16, np.float32)
    t = np.empty(15, np.float32)
    assert lib.tq_codebook(1024, 4, c.ctypes.data_as(f32), t.ctypes.data_as(f32)) == 0
    oc, ot = tq.lloyd_max(1024, 4)
    np.testing.assert_allclose(c, oc, rtol=2 ** -23, atol=0)
    np.testing.assert_allclose(t, ot, rtol=2 ** -23, atol=1e-30)
    assert t[7] == 0.0 and np.array_equal(c, -c[::-1])
    assert lib.tq_codebook(1024, 3, c.ctypes.data_as(f32), t.ctypes.data_as(f32)) == 4
    assert lib.tq_codebook(512, 4, c.ctypes.data_as(f32), t.ctypes.data_as(f32)) == 4
    vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
    lib.tq_encode.argtypes = [vp, i64, i32, vp, vp, vp, vp, vp]
    lib.tq_decode.argtypes = [vp, vp, i64, i32, vp, vp, vp, vp]
    E, D = lib.tq_encode, lib.tq_decode
    assert E(A, 10, 512, A, A, A, A, None) == 4
    assert E(A, -1, 1024, A, A, A, A, None) == 2
    assert E(A, 0, 1024, A, A, A, A, None) == 0
    assert E(None, 10, 1024, A, A, A, A, None) == 1
    assert E(A + 4, 10, 1024, A, A, A, A, None) == 3
    assert D(A, A, 10, 2048, A, A, A, None) == 4
    assert D(A, A, 0, 1024, A, A, A, None) == 0
    assert D(A, None, 10, 1024, A, A, A, None) == 1
    assert D(A, A, 10, 1024, A, A, A + 8, None) == 3


def test_weights_layout(lib):
    """w4a4_weights_bytes / w4a4_weights_bind: one allocation holding every
    array of a prepared layer, each at a 256-byte boundary, in the order qw,
    qw8, scale_ch, bias, smooth, inv_smooth, colsum; the arrays the layout
    leaves out are NULL.  (Sizes from the weight side of the linear: packed
    int4 codes, per-channel steps and bias, smoothing factors and their
    reciprocals.)"""
    vp, i32, u32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_uint32, ctypes.c_size_t
    lib.w4a4_weights_bytes.restype = sz
    lib.w4a4_weights_bytes.argtypes = [i32, i32, u32]
    lib.w4a4_weights_bind.restype = ctypes.c_int
    lib.w4a4_weights_bind.argtypes = [vp, sz, i32, i32, u32, ctypes.POINTER(WeightsT)]
    WB, BIND = lib.w4a4_weights_bytes, lib.w4a4_weights_bind
    r = lambda b: (b + 255) // 256 * 256
    for N, K in [(256, 1024), (3072, 1024), (1024, 4096), (4096, 1024)]:
        packed = r(N * K // 2) + 2 * r(4 * N) + 2 * r(4 * K)
        assert WB(N, K, 0) == WB(N, K, 2) == packed
        assert WB(N, K, UNPACKED) == packed + r(N * K) + r(4 * N)
        assert WB(N, K, INT8) == r(N * K) + 2 * r(4 * N) + 2 * r(4 * K)
        for flags in (0, UNPACKED, INT8, INT8 | 2):
            need = WB(N, K, flags)
            w = WeightsT()
            assert BIND(A, need, N, K, flags, ctypes.byref(w)) == 0
            assert (w.N, w.K, w.flags) == (N, K, 0)
            ptrs = {f: getattr(w, f) for f in ("qw", "qw8", "scale_ch", "bias", "smooth", "inv_smooth",
                                               "colsum")}
            size = {"qw": N * K // 2, "qw8": N * K, "scale_ch": 4 * N, "bias": 4 * N, "smooth": 4 * K,
                    "inv_smooth": 4 * K, "colsum": 4 * N}
            present = [f for f, p in ptrs.items() if p]
            want = {0: ["qw", "scale_ch", "bias", "smooth", "inv_smooth"],
                    UNPACKED: ["qw", "qw8", "scale_ch", "bias", "smooth", "inv_smooth", "colsum"]}
            want[INT8] = want[INT8 | 2] = ["qw8", "scale_ch", "bias", "smooth", "inv_smooth"]
            assert present == want[flags]
            off = A
            for f in present:                      # consecutive, 256-byte aligned, inside the buffer
                assert ptrs[f] == off and ptrs[f] % 256 == 0
                off += r(size[f])
            assert off == A + need
            # the bound struct passes the library's own weight checks (M = 0: no launch)
            w.flags = flags & (INT8 | 2)
            _setup(lib)
            assert lib.w4a4_linear(A, A, 0, ctypes.byref(w), A, None) == 0
    assert WB(1000, 1024, 0) == 0 and WB(256, 2048, 0) == 0 and WB(256, 1024, 0x10) == 0
    w = WeightsT()
    assert BIND(A, WB(256, 1024, 0) - 1, 256, 1024, 0, ctypes.byref(w)) == 2   # too small
    assert BIND(A + 8, 1 << 30, 256, 1024, 0, ctypes.byref(w)) == 3            # misaligned
    assert BIND(None, 1 << 30, 256, 1024, 0, ctypes.byref(w)) == 1
    assert BIND(A, 1 << 30, 256, 1024, 0, None) == 1
    assert BIND(A, 1 << 30, 100, 1024, 0, ctypes.byref(w)) == 2                 # N
    assert BIND(A, 1 << 30, 256, 1000, 0, ctypes.byref(w)) == 4                 # K
    assert BIND(A, 1 << 30, 256, 1024, 0x1, ctypes.byref(w)) == 4               # flag


STALL = 0x80000000


def test_gemm_s32_ex_argument_checks(lib):
    """w4a4_gemm_s32_ex: flags 0, W4A4_FLAG_UNPACKED (one-per-byte codes, with
    the expanded weights) and the failure-path test bit W4A4_DEBUG_STALL."""
    vp, i64 = ctypes.c_void_p, ctypes.c_int64
    G = lib.w4a4_gemm_s32_ex
    G.restype = ctypes.c_int
    G.argtypes = [vp, i64, ctypes.POINTER(WeightsT), vp, ctypes.c_uint32, vp]
    w = _weights()
    assert G(A, 0, ctypes.byref(w), A, 0, None) == 0
    assert G(A, 0, ctypes.byref(w), A, UNPACKED | STALL, None) == 0
    assert G(A, 10, ctypes.byref(w), A, 0x1, None) == 4                         # GELU: no
    assert G(A, 10, ctypes.byref(w), A, INT8, None) == 4                        # a weight flag
    assert G(A, 10, ctypes.byref(_weights(expanded=False)), A, UNPACKED, None) == 1
    assert G(A, 10, ctypes.byref(_weights8()), A, UNPACKED, None) == 1
    assert G(A, 10, ctypes.byref(w), None, STALL, None) == 1


def test_noalloc_argument_order(lib):
    """w4a4_linear_fused_noalloc refuses the flags w4a4_linear_fused refuses
    (W4A4_FLAG_UNPACKED among them) with the same status whatever M is, and
    sizes beyond its scratch with W4A4_ERR_SHAPE, before any CUDA call."""
    vp, i64 = ctypes.c_void_p, ctypes.c_int64
    f = lib.w4a4_linear_fused_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [vp, i64, ctypes.POINTER(WeightsT), vp, ctypes.c_uint32, vp]
    w = _weights()
    for M in (10, 1 << 20):
        assert f(A, M, ctypes.byref(w), A, UNPACKED, None) == 4
        assert f(A, M, ctypes.byref(w), A, 0x40, None) == 4
    assert f(A, 16257, ctypes.byref(w), A, 0, None) == 2         # one token past the scratch
    assert f(A, 4089, ctypes.byref(_weights(K=4096)), A, 0, None) == 2
    assert f(A, -1, ctypes.byref(w), A, 0, None) == 2
    assert f(A, 10, None, A, 0, None) == 1


def test_tq_rotation_qr_on_the_host(lib):
    """tq_rotation_qr (host code, no GPU): the library's Householder QR gives
    the oracle's sign-fixed Q factor (numpy's QR) of the same Gaussian matrix;
    its tf32 terms carry Pi to 2^-21 relative, the hi terms have the 13 low
    mantissa bits clear, and the Pi^T terms are the transposes."""
    import numpy as np
    from oracle import turboquant as tq
    from w4a4_post_quantized_b200 import synth
    vp = ctypes.c_void_p
    lib.tq_rotation_qr.argtypes = [vp, ctypes.c_int32, vp, vp, vp, vp]
    lib.tq_rotation_qr.restype = ctypes.c_int
    d = 1024
    G = synth.gaussian_matrix(d, seed=5)
    out = [np.empty((d, d), np.float32) for _ in range(4)]
    assert lib.tq_rotation_qr(G.ctypes.data_as(vp), d, *[o.ctypes.data_as(vp) for o in out]) == 0
    P = tq.rotation_qr(G)
    hi, lo = out[0].astype(np.float64), out[1].astype(np.float64)
    assert np.max(np.abs(hi + lo - P) / np.abs(P)) < 2.0 ** -21
    assert np.all((out[0].view(np.uint32) & 0x1FFF) == 0) and np.all((out[1].view(np.uint32) & 0x1FFF) == 0)
    assert np.array_equal(out[2], out[0].T) and np.array_equal(out[3], out[1].T)
    assert lib.tq_rotation_qr(G.ctypes.data_as(vp), 512, *[o.ctypes.data_as(vp) for o in out]) == 4
    assert lib.tq_rotation_qr(None, d, *[o.ctypes.data_as(vp) for o in out]) == 1
