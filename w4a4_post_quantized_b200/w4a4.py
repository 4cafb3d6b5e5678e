"""ctypes binding of libw4a4 (include/w4a4.h) for torch tensors.

Argument marshalling only: every step of the computation runs in the CUDA
library.  Importing this module raises ImportError when libw4a4.so has not
been built (``python -m w4a4_post_quantized_b200.build``); there is no
fallback.

The functions carry the C names.  Tensors must be contiguous CUDA tensors;
bf16 data is passed as torch.bfloat16, packed int4 codes as torch.uint8.
Calls are asynchronous on the given stream (default: torch's current stream).
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libw4a4.so")
if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m w4a4_post_quantized_b200.build`")
_lib = ctypes.CDLL(LIB_PATH)

W4A4_OK, W4A4_ERR_ARG, W4A4_ERR_SHAPE, W4A4_ERR_ALIGN, W4A4_ERR_UNSUPPORTED, W4A4_ERR_CUDA, \
    W4A4_ERR_TIMEOUT = range(7)
W4A4_DEV_TIMEOUT = 0x1
W4A4_FLAG_GELU = 0x1
W4A4_FLAG_PLAIN = 0x2
W4A4_FLAG_INT8 = 0x4
W4A4_FLAG_UNPACKED = 0x8
W4A4_FLAG_GELU_OUT = 0x10
W4A4_FLAG_X_DEVICE = 0x20
W4A4_FLAG_FWHT = 0x100
W4A4_FLAG_Y_DEVICE = 0x40
W4A4_DEBUG_STALL = 0x80000000

_vp, _i32, _i64, _u32, _f32, _sz = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32,
                                    ctypes.c_float, ctypes.c_size_t)


class W4A4WeightsT(ctypes.Structure):
    _fields_ = [("N", _i32), ("K", _i32), ("qw", _vp), ("scale_ch", _vp), ("bias", _vp),
                ("smooth", _vp), ("inv_smooth", _vp), ("qw8", _vp), ("colsum", _vp), ("flags", _u32)]


def _sig(name, res, args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = args
    return f


_workspace_bytes = _sig("w4a4_workspace_bytes", _sz, [_i64, _i32])
_workspace_bytes_min = _sig("w4a4_workspace_bytes_min", _sz, [_i64, _i32, _u32])
_prepare = _sig("w4a4_prepare_weights", ctypes.c_int,
                [_vp, _vp, _i32, _i32, _vp, _i64, _f32, _u32, ctypes.POINTER(W4A4WeightsT), _vp])
_quantize = _sig("w4a4_quantize_act", ctypes.c_int, [_vp, _i64, _i32, _vp, _vp, _vp, _u32, _vp])
_linear = _sig("w4a4_linear", ctypes.c_int, [_vp, _vp, _i64, ctypes.POINTER(W4A4WeightsT), _vp, _vp])
_linear_ex = _sig("w4a4_linear_ex", ctypes.c_int,
                  [_vp, _vp, _i64, ctypes.POINTER(W4A4WeightsT), _vp, _u32, _vp])
_fused = _sig("w4a4_linear_fused", ctypes.c_int,
              [_vp, _i64, ctypes.POINTER(W4A4WeightsT), _vp, _vp, _sz, _u32, _vp])
_fused_noalloc = _sig("w4a4_linear_fused_noalloc", ctypes.c_int,
                      [_vp, _i64, ctypes.POINTER(W4A4WeightsT), _vp, _u32, _vp])
_gemm_s32 = _sig("w4a4_gemm_s32", ctypes.c_int, [_vp, _i64, ctypes.POINTER(W4A4WeightsT), _vp, _vp])
_gemm_s32_ex = _sig("w4a4_gemm_s32_ex", ctypes.c_int,
                    [_vp, _i64, ctypes.POINTER(W4A4WeightsT), _vp, _u32, _vp])
_weights_bytes = _sig("w4a4_weights_bytes", _sz, [_i32, _i32, _u32])
_weights_bind = _sig("w4a4_weights_bind", ctypes.c_int,
                     [_vp, _sz, _i32, _i32, _u32, ctypes.POINTER(W4A4WeightsT)])
_pipe_create = _sig("w4a4_host_pipe_create", ctypes.c_int, [ctypes.POINTER(_vp)])
_pipe_destroy = _sig("w4a4_host_pipe_destroy", ctypes.c_int, [_vp])
_host_ws_bytes = _sig("w4a4_host_workspace_bytes", _sz, [_i64, _i32, _i32])
_fused_host = _sig("w4a4_linear_fused_host", ctypes.c_int,
                   [_vp, _i64, ctypes.POINTER(W4A4WeightsT), _vp, _i64, _vp, _sz, _vp, _u32, _vp])
_expand = _sig("w4a4_expand_weights", ctypes.c_int, [ctypes.POINTER(W4A4WeightsT), _vp])
_get_status = _sig("w4a4_get_device_status", ctypes.c_int, [_vp, ctypes.POINTER(_u32)])
_clear_status = _sig("w4a4_clear_device_status", ctypes.c_int, [_vp])
_tq_codebook = _sig("tq_codebook", ctypes.c_int, [_i32, _i32, _vp, _vp])
_tq_encode = _sig("tq_encode", ctypes.c_int, [_vp, _i64, _i32, _vp, _vp, _vp, _vp, _vp])
_tq_decode = _sig("tq_decode", ctypes.c_int, [_vp, _vp, _i64, _i32, _vp, _vp, _vp, _vp])
_tq_rotation_qr = _sig("tq_rotation_qr", ctypes.c_int, [_vp, _i32, _vp, _vp, _vp, _vp])
_tq_encode_dense = _sig("tq_encode_dense", ctypes.c_int, [_vp, _i64, _i32, _vp, _vp, _vp, _vp, _vp, _vp])
_tq_decode_dense = _sig("tq_decode_dense", ctypes.c_int, [_vp, _vp, _i64, _i32, _vp, _vp, _vp, _vp, _vp])
_status_string = _sig("w4a4_status_string", ctypes.c_char_p, [ctypes.c_int])
_version = _sig("w4a4_version", ctypes.c_char_p, [])


class W4A4Error(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {_status_string(code).decode()} (status {code})")


def _check(rc: int, where: str) -> None:
    if rc != W4A4_OK:
        raise W4A4Error(rc, where)


def _stream(stream) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t) -> ctypes.c_void_p:
    if t is None:
        return ctypes.c_void_p(0)
    if not t.is_contiguous():
        raise ValueError("tensors passed to libw4a4 must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def version() -> str:
    return _version().decode()


def w4a4_workspace_bytes(M: int, K: int) -> int:
    return int(_workspace_bytes(M, K))


def w4a4_workspace_bytes_min(M: int, K: int, flags: int) -> int:
    return int(_workspace_bytes_min(M, K, flags))


def w4a4_weights_bytes(N: int, K: int, flags: int = 0) -> int:
    return int(_weights_bytes(N, K, flags))


class PreparedWeights:
    """Device arrays of one prepared layer and the C struct that points at
    them: one torch-owned allocation of w4a4_weights_bytes(N, K, layout) bytes,
    laid out by w4a4_weights_bind; the attributes (qw, scale_ch, ...) are typed
    views into it.  expanded=True also holds the widened int8 copy of the codes
    (qw8, N*K bytes) and the per-row code sums the fast GEMM path uses;
    expanded=False keeps only the packed int4 codes.  int8=True (the W8A8
    setting) holds qw8 with the 8-bit codes and no packed codes."""

    def __init__(self, N: int, K: int, device="cuda", expanded: bool = True, int8: bool = False):
        self.N, self.K = N, K
        self.device = torch.device(device)
        layout = W4A4_FLAG_INT8 if int8 else (W4A4_FLAG_UNPACKED if expanded else 0)
        nbytes = w4a4_weights_bytes(N, K, layout)
        if nbytes == 0:
            raise W4A4Error(W4A4_ERR_SHAPE, "w4a4_weights_bytes")
        self.storage = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.struct = W4A4WeightsT()
        _check(_weights_bind(_ptr(self.storage), nbytes, N, K, layout, ctypes.byref(self.struct)),
               "w4a4_weights_bind")
        base = self.storage.data_ptr()

        def view(addr, count, dtype, shape):
            if not addr:
                return None
            off = addr - base
            nb = count * torch.empty((), dtype=dtype).element_size()
            return self.storage[off:off + nb].view(dtype).view(shape)
        st = self.struct
        self.qw = view(st.qw, N * K // 2, torch.uint8, (N, K // 2))
        self.scale_ch = view(st.scale_ch, N, torch.float32, (N,))
        self.bias = view(st.bias, N, torch.float32, (N,))
        self.smooth = view(st.smooth, K, torch.float32, (K,))
        self.inv_smooth = view(st.inv_smooth, K, torch.float32, (K,))
        self.qw8 = view(st.qw8, N * K, torch.int8, (N, K))
        self.colsum = view(st.colsum, N, torch.int32, (N,))

    @property
    def flags(self) -> int:
        return int(self.struct.flags)


def w4a4_prepare_weights(W: torch.Tensor, bias, X_calib, alpha: float = 0.5, flags: int = 0,
                         out: PreparedWeights | None = None, expanded: bool = True,
                         stream=None) -> PreparedWeights:
    N, K = W.shape
    out = out or PreparedWeights(N, K, W.device, expanded=expanded, int8=bool(flags & W4A4_FLAG_INT8))
    mc = 0 if X_calib is None else X_calib.shape[0]
    _check(_prepare(_ptr(W), _ptr(bias), N, K, _ptr(X_calib), mc, alpha, flags,
                    ctypes.byref(out.struct), _stream(stream)), "w4a4_prepare_weights")
    return out


def w4a4_quantize_act(X: torch.Tensor, inv_smooth, flags: int = 0, qx=None, scale_tok=None,
                      stream=None):
    M, K = X.shape
    width = K if flags & (W4A4_FLAG_INT8 | W4A4_FLAG_UNPACKED) else K // 2
    qx = qx if qx is not None else torch.empty((M, width), dtype=torch.uint8, device=X.device)
    scale_tok = scale_tok if scale_tok is not None else torch.empty(M, dtype=torch.float32, device=X.device)
    _check(_quantize(_ptr(X), M, K, _ptr(inv_smooth), _ptr(qx), _ptr(scale_tok), flags,
                     _stream(stream)), "w4a4_quantize_act")
    return qx, scale_tok


def w4a4_linear(qx: torch.Tensor, scale_tok: torch.Tensor, w: PreparedWeights, Y=None, stream=None):
    M = qx.shape[0]
    Y = Y if Y is not None else torch.empty((M, w.N), dtype=torch.bfloat16, device=qx.device)
    _check(_linear(_ptr(qx), _ptr(scale_tok), M, ctypes.byref(w.struct), _ptr(Y), _stream(stream)),
           "w4a4_linear")
    return Y


def w4a4_linear_ex(qx: torch.Tensor, scale_tok: torch.Tensor, w: PreparedWeights, flags: int = 0, Y=None,
                   stream=None):
    M = qx.shape[0]
    Y = Y if Y is not None else torch.empty((M, w.N), dtype=torch.bfloat16, device=qx.device)
    _check(_linear_ex(_ptr(qx), _ptr(scale_tok), M, ctypes.byref(w.struct), _ptr(Y), flags,
                      _stream(stream)), "w4a4_linear_ex")
    return Y


def w4a4_linear_fused(X: torch.Tensor, w: PreparedWeights, Y=None, workspace=None, flags: int = 0,
                      stream=None):
    M = X.shape[0]
    Y = Y if Y is not None else torch.empty((M, w.N), dtype=torch.bfloat16, device=X.device)
    need = w4a4_workspace_bytes(M, w.K)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=X.device)
    _check(_fused(_ptr(X), M, ctypes.byref(w.struct), _ptr(Y), _ptr(workspace),
                  workspace.numel() * workspace.element_size(), flags, _stream(stream)),
           "w4a4_linear_fused")
    return Y


W4A4_NOALLOC_SCRATCH_BYTES = 8 << 20


def w4a4_linear_fused_noalloc(X: torch.Tensor, w: PreparedWeights, Y=None, flags: int = 0,
                              stream=None):
    """w4a4_linear_fused without a workspace argument, for callers that may
    not allocate device memory where they run: the library's built-in scratch
    array (W4A4_NOALLOC_SCRATCH_BYTES per GPU) holds the intermediate codes.
    Calls that overlap on the GPU share that array and must not be issued."""
    M = X.shape[0]
    if Y is None:  # allocating the output here is a convenience of this binding only
        Y = torch.empty((M, w.N), dtype=torch.bfloat16, device=X.device)
    _check(_fused_noalloc(_ptr(X), M, ctypes.byref(w.struct), _ptr(Y), flags, _stream(stream)),
           "w4a4_linear_fused_noalloc")
    return Y


class HostPipe:
    """The copy streams and events of w4a4_linear_fused_host (created on the
    current device by the library; freed with the object)."""

    def __init__(self):
        h = _vp()
        _check(_pipe_create(ctypes.byref(h)), "w4a4_host_pipe_create")
        self.handle = h

    def close(self):
        if self.handle:
            _check(_pipe_destroy(self.handle), "w4a4_host_pipe_destroy")
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def w4a4_host_workspace_bytes(chunk_rows: int, K: int, N: int) -> int:
    return _host_ws_bytes(chunk_rows, K, N)


def w4a4_linear_fused_host(X_host: torch.Tensor, w: PreparedWeights, Y_host=None, chunk_rows: int = 2816,
                           workspace=None, pipe: HostPipe | None = None, flags: int = 0, stream=None):
    """Y_host = w4a4_linear_fused(X_host) with X_host / Y_host in (pinned) host
    memory; row chunks of chunk_rows are copied in, computed and copied out
    concurrently.  Returns Y_host (enqueued: synchronize `stream` before reading)."""
    M = X_host.shape[0]
    if Y_host is None:  # a convenience of this binding only
        Y_host = (torch.empty((M, w.N), dtype=torch.bfloat16, device=w.device)
                  if flags & W4A4_FLAG_Y_DEVICE else
                  torch.empty((M, w.N), dtype=torch.bfloat16, pin_memory=True))
    if workspace is None:
        workspace = torch.empty(w4a4_host_workspace_bytes(chunk_rows, w.K, w.N), dtype=torch.uint8,
                                device=w.device)
    if pipe is None:
        raise ValueError("w4a4_linear_fused_host needs a HostPipe")
    _check(_fused_host(_ptr(X_host), M, ctypes.byref(w.struct), _ptr(Y_host), chunk_rows, _ptr(workspace),
                       workspace.numel(), pipe.handle, flags, _stream(stream)), "w4a4_linear_fused_host")
    return Y_host


def w4a4_expand_weights(w: PreparedWeights, stream=None) -> PreparedWeights:
    _check(_expand(ctypes.byref(w.struct), _stream(stream)), "w4a4_expand_weights")
    return w


def w4a4_gemm_s32(qx: torch.Tensor, w: PreparedWeights, acc=None, stream=None):
    M = qx.shape[0]
    acc = acc if acc is not None else torch.empty((M, w.N), dtype=torch.int32, device=qx.device)
    _check(_gemm_s32(_ptr(qx), M, ctypes.byref(w.struct), _ptr(acc), _stream(stream)), "w4a4_gemm_s32")
    return acc


def w4a4_gemm_s32_ex(qx: torch.Tensor, w: PreparedWeights, flags: int = 0, acc=None, stream=None):
    M = qx.shape[0]
    acc = acc if acc is not None else torch.empty((M, w.N), dtype=torch.int32, device=qx.device)
    _check(_gemm_s32_ex(_ptr(qx), M, ctypes.byref(w.struct), _ptr(acc), flags, _stream(stream)),
           "w4a4_gemm_s32_ex")
    return acc


def w4a4_get_device_status(stream=None) -> int:
    v = _u32(0)
    rc = _get_status(_stream(stream), ctypes.byref(v))
    if rc not in (W4A4_OK, W4A4_ERR_TIMEOUT):
        _check(rc, "w4a4_get_device_status")
    return int(v.value)


def w4a4_clear_device_status(stream=None) -> None:
    _check(_clear_status(_stream(stream)), "w4a4_clear_device_status")


# ------------------------------------------------- 3DTurboQuant codec (include/tq.h)
def tq_codebook(d: int = 1024, b: int = 4):
    """Host Lloyd-Max codebook: (centroids [2^b], boundaries [2^b - 1]) as fp32 numpy arrays."""
    import numpy as np
    c = np.empty(1 << b, np.float32)
    t = np.empty((1 << b) - 1, np.float32)
    _check(_tq_codebook(d, b, c.ctypes.data_as(_vp), t.ctypes.data_as(_vp)), "tq_codebook")
    return c, t


def tq_encode(X: torch.Tensor, signs: torch.Tensor, boundaries: torch.Tensor, codes=None, norms=None,
              stream=None):
    """X [n, d] fp32 -> (codes uint8 [n, d/2], norms fp32 [n])."""
    n, d = X.shape
    codes = codes if codes is not None else torch.empty((n, d // 2), dtype=torch.uint8, device=X.device)
    norms = norms if norms is not None else torch.empty(n, dtype=torch.float32, device=X.device)
    _check(_tq_encode(_ptr(X), n, d, _ptr(signs), _ptr(boundaries), _ptr(codes), _ptr(norms),
                      _stream(stream)), "tq_encode")
    return codes, norms


def tq_decode(codes: torch.Tensor, norms: torch.Tensor, signs: torch.Tensor, centroids: torch.Tensor,
              Y=None, stream=None):
    """(codes [n, d/2], norms [n]) -> Y [n, d] fp32."""
    n, d = codes.shape[0], codes.shape[1] * 2
    Y = Y if Y is not None else torch.empty((n, d), dtype=torch.float32, device=codes.device)
    _check(_tq_decode(_ptr(codes), _ptr(norms), n, d, _ptr(signs), _ptr(centroids), _ptr(Y),
                      _stream(stream)), "tq_decode")
    return Y


# ---------------------------------- the page's dense rotation (QR of a Gaussian)
def tq_rotation_qr(G):
    """Host: Pi = the sign-fixed Q factor of the d x d Gaussian matrix G (numpy
    float64), as tf32 hi / lo terms of Pi and of Pi^T: returns
    (pi_hi, pi_lo, pit_hi, pit_lo), numpy float32 [d, d] each."""
    import numpy as np
    G = np.ascontiguousarray(G, dtype=np.float64)
    d = G.shape[0]
    out = [np.empty((d, d), np.float32) for _ in range(4)]
    _check(_tq_rotation_qr(G.ctypes.data_as(_vp), d, *[o.ctypes.data_as(_vp) for o in out]),
           "tq_rotation_qr")
    return tuple(out)


def tq_encode_dense(X: torch.Tensor, pi_hi: torch.Tensor, pi_lo: torch.Tensor, boundaries: torch.Tensor,
                    codes=None, norms=None, stream=None):
    """X [n, d] fp32 -> (codes uint8 [n, d/2], norms fp32 [n]) with the dense Pi."""
    n, d = X.shape
    codes = codes if codes is not None else torch.empty((n, d // 2), dtype=torch.uint8, device=X.device)
    norms = norms if norms is not None else torch.empty(n, dtype=torch.float32, device=X.device)
    _check(_tq_encode_dense(_ptr(X), n, d, _ptr(pi_hi), _ptr(pi_lo), _ptr(boundaries), _ptr(codes),
                            _ptr(norms), _stream(stream)), "tq_encode_dense")
    return codes, norms


def tq_decode_dense(codes: torch.Tensor, norms: torch.Tensor, pit_hi: torch.Tensor, pit_lo: torch.Tensor,
                    centroids: torch.Tensor, Y=None, stream=None):
    """(codes [n, d/2], norms [n]) -> Y [n, d] fp32 with the dense Pi."""
    n, d = codes.shape[0], codes.shape[1] * 2
    Y = Y if Y is not None else torch.empty((n, d), dtype=torch.float32, device=codes.device)
    _check(_tq_decode_dense(_ptr(codes), _ptr(norms), n, d, _ptr(pit_hi), _ptr(pit_lo), _ptr(centroids),
                            _ptr(Y), _stream(stream)), "tq_decode_dense")
    return Y
