"""Python binding of the qlin C ABI (include/qlin.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of ``libqlin.so``.  The binding takes torch CUDA tensors, passes their
device pointers and the current CUDA stream through ctypes, and raises
``QlinError`` on any non-OK status.  There is no CPU path: when the library or
a CUDA device is missing the calls raise.
"""
import ctypes as C
import os

import torch

__all__ = [
    "QlinError", "Q4_G64", "Q5_G64", "Q8_G32", "FP8_ROW", "BF16", "Q3_G64", "Q6_G64",
    "SRC_F32", "SRC_BF16", "SRC_MXFP8", "SRC_MLX_AFFINE8", "SRC_FP8_BLOCK128", "OUT_BF16", "OUT_F32",
    "ALLOW_A8", "DEBUG_GROUP_SUMS", "PackedWeights", "Workspace", "lib",
    "qlin_packed_bytes", "qlin_pack_weights", "qlin_decode_mxfp8", "qlin_quantize_act",
    "qlin_gemv", "qlin_gemv_workspace_bytes", "qlin_gemm_a8", "qlin_gemm_a8_workspace_bytes",
    "qlin_status_string", "qlin_gemv_noalloc", "qlin_quantize_act_fp8",
    "qlin_gemm_fp8_workspace_bytes", "qlin_gemm_fp8",
]

Q4_G64, Q5_G64, Q8_G32, FP8_ROW, BF16, Q3_G64, Q6_G64 = 0, 1, 2, 3, 4, 5, 6
SRC_F32, SRC_BF16, SRC_MXFP8, SRC_MLX_AFFINE8, SRC_FP8_BLOCK128 = 0, 1, 2, 3, 4
OUT_BF16, OUT_F32 = 0, 1
ALLOW_A8 = 0x1
DEBUG_GROUP_SUMS = 0x1
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_NOT_PERMITTED, ERR_CUDA, ERR_TIMEOUT, ERR_WORKSPACE = range(7)

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libqlin.so")

EXPORTED = (
    "qlin_status_string", "qlin_packed_bytes", "qlin_pack_weights", "qlin_decode_mxfp8",
    "qlin_quantize_act", "qlin_gemv_workspace_bytes", "qlin_gemv",
    "qlin_gemm_a8_workspace_bytes", "qlin_gemm_a8", "qlin_gemv_noalloc",
    "qlin_quantize_act_fp8", "qlin_gemm_fp8_workspace_bytes", "qlin_gemm_fp8",
)


class QlinError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__(f"{what}: {qlin_status_string(status)} (status {status})")


class _Exec(C.Structure):
    _fields_ = [("stream", C.c_void_p), ("dev_status", C.c_void_p), ("workspace", C.c_void_p),
                ("workspace_bytes", C.c_size_t)]


class _Weights(C.Structure):
    _fields_ = [("fmt", C.c_int32), ("flags", C.c_uint32), ("n", C.c_int64), ("k", C.c_int64),
                ("codes", C.c_void_p), ("hibits", C.c_void_p), ("scales", C.c_void_p)]


_lib = None


def lib():
    """Load libqlin.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libqlin.so is missing at {LIB_PATH}: build it first "
                               "(python -m quantized_weight_linear_qlin_b200._build)")
        L = C.CDLL(LIB_PATH)
        vp, i64, i32, u32 = C.c_void_p, C.c_int64, C.c_int, C.c_uint32
        L.qlin_status_string.argtypes = [i32]
        L.qlin_status_string.restype = C.c_char_p
        L.qlin_packed_bytes.argtypes = [i32, i64, i64, vp, vp, vp]
        L.qlin_pack_weights.argtypes = [i32, vp, vp, vp, C.POINTER(_Weights), C.POINTER(_Exec)]
        L.qlin_decode_mxfp8.argtypes = [vp, vp, i64, i64, vp, C.POINTER(_Exec)]
        L.qlin_quantize_act.argtypes = [vp, i64, i64, vp, vp, C.POINTER(_Exec)]
        L.qlin_gemv_workspace_bytes.argtypes = [C.POINTER(_Weights), i64, vp]
        L.qlin_gemv.argtypes = [C.POINTER(_Weights), vp, i64, vp, i32, C.POINTER(_Exec)]
        L.qlin_gemv_noalloc.argtypes = [C.POINTER(_Weights), vp, i64, vp, i32, vp, vp]
        L.qlin_gemm_a8_workspace_bytes.argtypes = [i64, i64, i64, vp]
        L.qlin_gemm_a8.argtypes = [C.POINTER(_Weights), vp, vp, vp, i64, vp, i32, u32, vp,
                                   C.POINTER(_Exec)]
        L.qlin_quantize_act_fp8.argtypes = [vp, i64, i64, vp, vp, C.POINTER(_Exec)]
        L.qlin_gemm_fp8_workspace_bytes.argtypes = [i64, i64, vp]
        L.qlin_gemm_fp8.argtypes = [C.POINTER(_Weights), vp, vp, vp, i64, vp, i32, C.POINTER(_Exec)]
        for name in EXPORTED[1:]:
            getattr(L, name).restype = i32
        _lib = L
    return _lib


def qlin_status_string(status: int) -> str:
    try:
        return lib().qlin_status_string(int(status)).decode()
    except Exception:  # library missing: still produce a message
        return f"status {status}"


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch tensor")
    if not t.is_cuda:
        raise ValueError("qlin works on CUDA tensors only (no CPU path)")
    if not t.is_contiguous():
        raise ValueError("qlin needs contiguous tensors")
    return t.data_ptr()


_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)
_get_device = getattr(torch._C, "_cuda_getDevice", None)


def _current_stream_handle():
    """cudaStream_t of torch's current stream on the current device."""
    if _raw_stream is not None and _get_device is not None:
        return _raw_stream(_get_device())
    return torch.cuda.current_stream().cuda_stream


def _exec(stream=None, workspace=None, dev_status=None):
    e = _Exec()
    e.stream = C.c_void_p(_current_stream_handle() if stream is None else stream.cuda_stream)
    e.dev_status = None if dev_status is None else _ptr(dev_status)
    if workspace is not None:
        buf = workspace.buffer if isinstance(workspace, Workspace) else workspace
        e.workspace = _ptr(buf)
        e.workspace_bytes = buf.numel() * buf.element_size()
    return e


def _check(rc, what):
    if rc != OK:
        raise QlinError(rc, what)


def qlin_packed_bytes(fmt, n, k):
    c, h, s = C.c_size_t(), C.c_size_t(), C.c_size_t()
    _check(lib().qlin_packed_bytes(fmt, n, k, C.byref(c), C.byref(h), C.byref(s)), "qlin_packed_bytes")
    return c.value, h.value, s.value


class PackedWeights:
    """Device buffers of one packed matrix plus its qlin_weights descriptor."""

    def __init__(self, fmt, n, k, device="cuda", allow_a8=False, codes=None, hibits=None,
                 scales=None):
        cb, hb, sb = qlin_packed_bytes(fmt, n, k)
        self.fmt, self.n, self.k = fmt, n, k
        self.flags = ALLOW_A8 if allow_a8 else 0
        self.codes = codes if codes is not None else torch.empty(cb, dtype=torch.uint8, device=device)
        self.hibits = hibits if hibits is not None else (
            torch.empty(hb, dtype=torch.uint8, device=device) if hb else None)
        self.scales = scales if scales is not None else (
            torch.empty(sb, dtype=torch.uint8, device=device) if sb else None)

    def desc(self):
        """The qlin_weights descriptor (built once; rebuilt if a buffer is replaced)."""
        key = (self.codes.data_ptr(), None if self.hibits is None else self.hibits.data_ptr(),
               None if self.scales is None else self.scales.data_ptr(), self.flags)
        if getattr(self, "_desc_key", None) != key:
            d = _Weights()
            d.fmt, d.flags, d.n, d.k = self.fmt, self.flags, self.n, self.k
            d.codes = _ptr(self.codes)
            d.hibits = None if self.hibits is None else _ptr(self.hibits)
            d.scales = None if self.scales is None else _ptr(self.scales)
            self._desc, self._desc_key = d, key
        return self._desc

    def bytes(self):
        return sum(t.numel() * t.element_size() for t in (self.codes, self.hibits, self.scales)
                   if t is not None)


class Workspace:
    """Caller-owned device scratch (zero-filled once when allocated or grown)."""

    def __init__(self, device="cuda"):
        self.device = device
        self.buffer = torch.zeros(256, dtype=torch.uint8, device=device)

    def ensure(self, nbytes):
        if nbytes > self.buffer.numel():
            self.buffer = torch.zeros((nbytes + 255) // 256 * 256, dtype=torch.uint8, device=self.device)
        return self


def qlin_pack_weights(src_kind, src, dst: PackedWeights, aux0=None, aux1=None, stream=None):
    d = dst.desc()
    e = _exec(stream)
    _check(lib().qlin_pack_weights(src_kind, _ptr(src), _ptr(aux0), _ptr(aux1), C.byref(d),
                                   C.byref(e)), "qlin_pack_weights")
    return dst


def qlin_decode_mxfp8(words, scales, rows, cols, out, stream=None):
    e = _exec(stream)
    _check(lib().qlin_decode_mxfp8(_ptr(words), _ptr(scales), rows, cols, _ptr(out), C.byref(e)),
           "qlin_decode_mxfp8")
    return out


def qlin_quantize_act(x, xq, xs, stream=None):
    t, k = x.shape
    e = _exec(stream)
    _check(lib().qlin_quantize_act(_ptr(x), t, k, _ptr(xq), _ptr(xs), C.byref(e)), "qlin_quantize_act")
    return xq, xs


def qlin_gemv_workspace_bytes(w: PackedWeights, t):
    b = C.c_size_t()
    d = w.desc()
    _check(lib().qlin_gemv_workspace_bytes(C.byref(d), t, C.byref(b)), "qlin_gemv_workspace_bytes")
    return b.value


def qlin_gemv(w: PackedWeights, x, y, y_dtype=OUT_BF16, workspace=None, stream=None,
              dev_status=None):
    t = x.shape[0]
    d = w.desc()
    e = _exec(stream, workspace, dev_status)
    _check(lib().qlin_gemv(C.byref(d), _ptr(x), t, _ptr(y), y_dtype, C.byref(e)), "qlin_gemv")
    return y


def qlin_gemv_noalloc(w: PackedWeights, x, y, y_dtype=OUT_BF16, stream=None, dev_status=None):
    """qlin_gemv with the library's fixed device scratch instead of a workspace."""
    t = x.shape[0]
    d = w.desc()
    sh = _current_stream_handle() if stream is None else stream.cuda_stream
    _check(lib().qlin_gemv_noalloc(C.byref(d), _ptr(x), t, _ptr(y), y_dtype, C.c_void_p(sh),
                                   None if dev_status is None else _ptr(dev_status)), "qlin_gemv_noalloc")
    return y


def qlin_gemm_a8_workspace_bytes(t, n, k):
    b = C.c_size_t()
    _check(lib().qlin_gemm_a8_workspace_bytes(t, n, k, C.byref(b)), "qlin_gemm_a8_workspace_bytes")
    return b.value


def qlin_gemm_a8(w: PackedWeights, y, x=None, xq=None, xs=None, y_dtype=OUT_BF16, flags=0,
                 sums_dbg=None, workspace=None, stream=None, dev_status=None):
    t = (x if x is not None else xq).shape[0]
    d = w.desc()
    e = _exec(stream, workspace, dev_status)
    _check(lib().qlin_gemm_a8(C.byref(d), _ptr(x), _ptr(xq), _ptr(xs), t, _ptr(y), y_dtype, flags,
                              _ptr(sums_dbg), C.byref(e)), "qlin_gemm_a8")
    return y


def qlin_quantize_act_fp8(x, xq, xs, stream=None):
    t, k = x.shape
    e = _exec(stream)
    _check(lib().qlin_quantize_act_fp8(_ptr(x), t, k, _ptr(xq), _ptr(xs), C.byref(e)),
           "qlin_quantize_act_fp8")
    return xq, xs


def qlin_gemm_fp8_workspace_bytes(t, k):
    b = C.c_size_t()
    _check(lib().qlin_gemm_fp8_workspace_bytes(t, k, C.byref(b)), "qlin_gemm_fp8_workspace_bytes")
    return b.value


def qlin_gemm_fp8(w: PackedWeights, y, x=None, xq=None, xs=None, y_dtype=OUT_BF16, workspace=None,
                  stream=None, dev_status=None):
    t = (x if x is not None else xq).shape[0]
    d = w.desc()
    e = _exec(stream, workspace, dev_status)
    _check(lib().qlin_gemm_fp8(C.byref(d), _ptr(x), _ptr(xq), _ptr(xs), t, _ptr(y), y_dtype,
                               C.byref(e)), "qlin_gemm_fp8")
    return y
