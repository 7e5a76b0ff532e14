"""CPU oracle for the quantized linear path -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never calls it and
shares no code with it.  The arithmetic lives in ``qlin_oracle.cpp`` (plain
scalar C++); this module only marshals numpy arrays through ctypes.

Parity status: every function is pinned by the ``-m "not gpu"`` tests in
``tests/test_oracle_*.py`` (closed forms, library routines, invariants, brute
force).  No function is "parity unpinned".
"""
import ctypes as C
import os

import numpy as np

from . import build as _build

Q4_G64, Q5_G64, Q8_G32, FP8_ROW, BF16, Q3_G64, Q6_G64 = 0, 1, 2, 3, 4, 5, 6

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        i64, vp, i32 = C.c_int64, C.c_void_p, C.c_int
        L.oracle_f16_value.argtypes = [C.c_uint16]
        L.oracle_f16_value.restype = C.c_double
        L.oracle_f16_rne.argtypes = [C.c_double]
        L.oracle_f16_rne.restype = C.c_uint16
        L.oracle_bf16_value.argtypes = [C.c_uint16]
        L.oracle_bf16_value.restype = C.c_double
        L.oracle_bf16_rne.argtypes = [C.c_double]
        L.oracle_bf16_rne.restype = C.c_uint16
        L.oracle_e4m3_value.argtypes = [C.c_uint8]
        L.oracle_e4m3_value.restype = C.c_double
        L.oracle_e4m3_rne_satfinite.argtypes = [C.c_double]
        L.oracle_e4m3_rne_satfinite.restype = C.c_uint8
        L.oracle_to_bf16.argtypes = [vp, i64, vp]
        L.oracle_pack_groupwise.argtypes = [i32, vp, i64, i64, vp, vp, vp]
        L.oracle_pack_fp8_row.argtypes = [vp, i64, i64, vp, vp]
        L.oracle_decode_mxfp8.argtypes = [vp, vp, i64, i64, vp]
        L.oracle_decode_mlx_affine.argtypes = [vp, vp, vp, i64, i64, vp]
        L.oracle_decode_fp8_block128.argtypes = [vp, vp, i64, i64, vp]
        L.oracle_dequant.argtypes = [i32, vp, vp, vp, i64, i64, vp]
        L.oracle_gemv.argtypes = [i32, vp, vp, vp, i64, i64, vp, i64, vp, vp, i32]
        L.oracle_quantize_act.argtypes = [vp, i64, i64, vp, vp]
        L.oracle_group_sums.argtypes = [i32, vp, vp, vp, i64, i64, i64, vp]
        L.oracle_gemm_a8.argtypes = [i32, vp, vp, vp, vp, vp, i64, i64, i64, vp, vp, i32]
        L.oracle_quantize_act_fp8.argtypes = [vp, i64, i64, vp, vp]
        L.oracle_gemm_fp8.argtypes = [vp, vp, vp, vp, i64, i64, i64, vp, vp, i32]
        for name in ("oracle_to_bf16", "oracle_pack_groupwise", "oracle_pack_fp8_row", "oracle_decode_mxfp8",
                     "oracle_decode_mlx_affine", "oracle_decode_fp8_block128", "oracle_dequant", "oracle_gemv",
                     "oracle_quantize_act", "oracle_group_sums", "oracle_gemm_a8",
                     "oracle_quantize_act_fp8", "oracle_gemm_fp8"):
            getattr(L, name).restype = C.c_int
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments (rc={rc})")


# ---- codecs -----------------------------------------------------------------
def f16_value(bits: int) -> float:
    return lib().oracle_f16_value(int(bits))


def f16_rne(v: float) -> int:
    return lib().oracle_f16_rne(float(v))


def bf16_value(bits: int) -> float:
    return lib().oracle_bf16_value(int(bits))


def bf16_rne(v: float) -> int:
    return lib().oracle_bf16_rne(float(v))


def e4m3_value(code: int) -> float:
    return lib().oracle_e4m3_value(int(code))


def e4m3_rne_satfinite(v: float) -> int:
    return lib().oracle_e4m3_rne_satfinite(float(v))


# ---- packed sizes of this library's layouts ---------------------------------
def packed_shapes(fmt, n, k):
    """(codes dtype, codes shape, hibits shape or None, scales dtype, scales shape)."""
    if fmt == Q4_G64:
        return np.uint8, (n, k // 2), None, np.uint16, (n, k // 64)
    if fmt == Q5_G64:
        return np.uint8, (n, k // 2), (n, k // 8), np.uint16, (n, k // 64)
    if fmt == Q3_G64:
        return np.uint8, (n, k // 4), (n, k // 8), np.uint16, (n, k // 64)
    if fmt == Q6_G64:
        return np.uint8, (n, k // 2), (n, k // 4), np.uint16, (n, k // 64)
    if fmt == Q8_G32:
        return np.int8, (n, k), None, np.uint16, (n, k // 32)
    if fmt == FP8_ROW:
        return np.uint8, (n, k), None, np.uint16, (n,)
    if fmt == BF16:
        return np.uint16, (n, k), None, None, None
    raise ValueError(fmt)


# ---- method -----------------------------------------------------------------
def pack(fmt, w):
    """Quantize float32 values w[n][k] -> dict(codes, hibits, scales)."""
    w = _c(w, np.float32)
    n, k = w.shape
    cdt, cshape, hshape, sdt, sshape = packed_shapes(fmt, n, k)
    codes = np.zeros(cshape, cdt)
    hib = np.zeros(hshape, np.uint8) if hshape else None
    if fmt == FP8_ROW:
        scales = np.zeros(sshape, sdt)
        _check(lib().oracle_pack_fp8_row(_p(w), n, k, _p(codes), _p(scales)), "pack_fp8_row")
    elif fmt in (Q4_G64, Q5_G64, Q8_G32, Q3_G64, Q6_G64):
        scales = np.zeros(sshape, sdt)
        _check(lib().oracle_pack_groupwise(fmt, _p(w), n, k, _p(codes), _p(hib), _p(scales)),
               "pack_groupwise")
    elif fmt == BF16:
        codes = np.zeros((n, k), np.uint16)
        _check(lib().oracle_to_bf16(_p(w), n * k, _p(codes)), "to_bf16")
        scales = None
    else:
        raise ValueError(fmt)
    return {"fmt": fmt, "n": n, "k": k, "codes": codes, "hibits": hib, "scales": scales}


def dequant(pw):
    out = np.zeros((pw["n"], pw["k"]), np.float64)
    _check(lib().oracle_dequant(pw["fmt"], _p(pw["codes"]), _p(pw["hibits"]), _p(pw["scales"]),
                                pw["n"], pw["k"], _p(out)), "dequant")
    return out


def decode_mxfp8(words, scales, rows, cols):
    words = _c(words, np.uint32)
    scales = _c(scales, np.uint8)
    out = np.zeros((rows, cols), np.uint16)
    _check(lib().oracle_decode_mxfp8(_p(words), _p(scales), rows, cols, _p(out)), "decode_mxfp8")
    return out


def decode_mlx_affine(q, scales, biases, rows, cols):
    q = _c(q, np.uint8)
    scales = _c(scales, np.uint16)
    biases = _c(biases, np.uint16)
    out = np.zeros((rows, cols), np.uint16)
    _check(lib().oracle_decode_mlx_affine(_p(q), _p(scales), _p(biases), rows, cols, _p(out)),
           "decode_mlx_affine")
    return out


def decode_fp8_block128(codes, scale_inv, rows, cols):
    """E4M3 codes uint8[rows][cols] + float32 scale_inv[ceil(rows/128)][ceil(cols/128)]
    -> bfloat16 bits [rows][cols]."""
    codes = _c(codes, np.uint8)
    scale_inv = _c(scale_inv, np.float32)
    out = np.zeros((rows, cols), np.uint16)
    _check(lib().oracle_decode_fp8_block128(_p(codes), _p(scale_inv), rows, cols, _p(out)),
           "decode_fp8_block128")
    return out


def gemv(pw, x_bf16, nthreads=1, with_bound=True):
    """x_bf16: uint16 [t][k] (bfloat16 bits) -> (y[t][n] float64, bound[t][n])."""
    x = _c(x_bf16, np.uint16)
    t = x.shape[0]
    n = pw["n"]
    y = np.zeros((t, n), np.float64)
    b = np.zeros((t, n), np.float64) if with_bound else None
    _check(lib().oracle_gemv(pw["fmt"], _p(pw["codes"]), _p(pw["hibits"]), _p(pw["scales"]), n,
                             pw["k"], _p(x), t, _p(y), _p(b), int(nthreads)), "gemv")
    return y, b


def quantize_act(x_bf16):
    x = _c(x_bf16, np.uint16)
    t, k = x.shape
    qa = np.zeros((t, k), np.int8)
    as_ = np.zeros((t, k // 64), np.float32)
    _check(lib().oracle_quantize_act(_p(x), t, k, _p(qa), _p(as_)), "quantize_act")
    return qa, as_


def group_sums(pw, qa):
    qa = _c(qa, np.int8)
    t = qa.shape[0]
    n, k = pw["n"], pw["k"]
    S = np.zeros((t, n, k // 64), np.int32)
    _check(lib().oracle_group_sums(pw["fmt"], _p(pw["codes"]), _p(pw["hibits"]), _p(qa), t, n, k,
                                   _p(S)), "group_sums")
    return S


def gemm_a8(pw, qa, as_, nthreads=1, with_bound=True):
    qa = _c(qa, np.int8)
    as_ = _c(as_, np.float32)
    t = qa.shape[0]
    n, k = pw["n"], pw["k"]
    y = np.zeros((t, n), np.float64)
    b = np.zeros((t, n), np.float64) if with_bound else None
    _check(lib().oracle_gemm_a8(pw["fmt"], _p(pw["codes"]), _p(pw["hibits"]), _p(pw["scales"]),
                                _p(qa), _p(as_), t, n, k, _p(y), _p(b), int(nthreads)), "gemm_a8")
    return y, b


def quantize_act_fp8(x_bf16):
    """Per-token E4M3 activations: (xq uint8[t][k], xs float32[t])."""
    x = _c(x_bf16, np.uint16)
    t, k = x.shape
    xq = np.zeros((t, k), np.uint8)
    xs = np.zeros((t,), np.float32)
    _check(lib().oracle_quantize_act_fp8(_p(x), t, k, _p(xq), _p(xs)), "quantize_act_fp8")
    return xq, xs


def gemm_fp8(pw, xq, xs, nthreads=1, with_bound=True):
    """Row-FP8 weights (oracle.pack(FP8_ROW, ...)) x per-token FP8 activations."""
    assert pw["fmt"] == FP8_ROW
    xq = _c(xq, np.uint8)
    xs = _c(xs, np.float32)
    t = xq.shape[0]
    n, k = pw["n"], pw["k"]
    y = np.zeros((t, n), np.float64)
    b = np.zeros((t, n), np.float64) if with_bound else None
    _check(lib().oracle_gemm_fp8(_p(pw["codes"]), _p(pw["scales"]), _p(xq), _p(xs), t, n, k, _p(y), _p(b),
                                 int(nthreads)), "gemm_fp8")
    return y, b


def cores_available() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:  # pragma: no cover
        return os.cpu_count() or 1
