"""CPU checks of the C ABI: the library loads, exports every entry point the
header declares, and rejects bad arguments on the host before touching the
GPU (these calls return before any CUDA call, so they run without a device)."""
import ctypes as C
import os
import re

import pytest

import quantized_weight_linear_qlin_b200 as q

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            with open(os.path.join(ROOT, "include", fn)) as f:
                txt = f.read()
            names |= set(re.findall(r"QLIN_API\s+[\w\s\*]+?\b(qlin_\w+)\s*\(", txt))
    return names


@pytest.fixture(scope="module")
def L():
    from quantized_weight_linear_qlin_b200 import _build
    _build.build()
    return q.lib()


def test_exports_every_declared_symbol(L):
    names = _declared()
    assert len(names) >= 9
    for n in names:
        assert hasattr(L, n), n
    assert names == set(q.EXPORTED)


def test_status_strings(L):
    for s in range(7):
        assert q.qlin_status_string(s)
    assert "unknown" in q.qlin_status_string(99)


def test_packed_bytes(L):
    assert q.qlin_packed_bytes(q.Q4_G64, 34816, 5120) == (34816 * 2560, 0, 34816 * 80 * 2)
    assert q.qlin_packed_bytes(q.Q5_G64, 5120, 17408) == (5120 * 8704, 5120 * 2176, 5120 * 272 * 2)
    assert q.qlin_packed_bytes(q.Q8_G32, 5120, 5120) == (5120 * 5120, 0, 5120 * 160 * 2)
    assert q.qlin_packed_bytes(q.FP8_ROW, 152064, 5120) == (152064 * 5120, 0, 152064 * 2)
    assert q.qlin_packed_bytes(q.BF16, 96, 5120) == (96 * 5120 * 2, 0, 0)
    assert q.qlin_packed_bytes(q.Q3_G64, 34816, 5120) == (34816 * 1280, 34816 * 640, 34816 * 80 * 2)
    assert q.qlin_packed_bytes(q.Q6_G64, 5120, 17408) == (5120 * 8704, 5120 * 4352, 5120 * 272 * 2)
    # the configs' algorithmic weight bytes
    c, h, s = q.qlin_packed_bytes(q.Q4_G64, 34816, 5120)
    assert c + h + s == 94_699_520
    c, h, s = q.qlin_packed_bytes(q.Q5_G64, 5120, 17408)
    assert c + h + s == 58_490_880
    for fmt, k in ((q.Q4_G64, 96), (q.Q8_G32, 48), (q.Q3_G64, 96), (q.Q6_G64, 32), (9, 64)):
        with pytest.raises(q.QlinError) as e:
            q.qlin_packed_bytes(fmt, 4, k)
        assert e.value.status == q.ERR_INVALID_ARG


def _weights(fmt, n, k, flags=0, addr=0x10000):
    d = q._Weights()
    d.fmt, d.flags, d.n, d.k = fmt, flags, n, k
    d.codes, d.hibits, d.scales = addr, addr + 0x1000 if fmt in (q.Q5_G64, q.Q3_G64, q.Q6_G64) else None, \
        None if fmt == q.BF16 else addr + 0x2000
    return d


def test_host_validation_rejects_before_cuda(L):
    ex = q._Exec()
    fake = C.c_void_p(0x20000)
    odd = C.c_void_p(0x20008)
    w = _weights(q.Q4_G64, 256, 512, flags=q.ALLOW_A8)
    # gemv: T above 64 is unsupported for quantized weights
    assert L.qlin_gemv(C.byref(w), fake, 65, fake, q.OUT_BF16, C.byref(ex)) == q.ERR_UNSUPPORTED
    # the no-alloc variant runs the same checks first (before any CUDA call)
    assert L.qlin_gemv_noalloc(C.byref(w), fake, 65, fake, q.OUT_BF16, None, None) == q.ERR_UNSUPPORTED
    assert L.qlin_gemv_noalloc(C.byref(w), odd, 1, fake, q.OUT_BF16, None, None) == q.ERR_INVALID_ARG
    assert L.qlin_gemv_noalloc(None, fake, 1, fake, q.OUT_BF16, None, None) == q.ERR_INVALID_ARG
    # misaligned activation / output pointers
    assert L.qlin_gemv(C.byref(w), odd, 1, fake, q.OUT_BF16, C.byref(ex)) == q.ERR_INVALID_ARG
    assert L.qlin_gemv(C.byref(w), fake, 1, odd, q.OUT_BF16, C.byref(ex)) == q.ERR_INVALID_ARG
    assert L.qlin_gemv(C.byref(w), fake, 1, fake, 7, C.byref(ex)) == q.ERR_INVALID_ARG
    assert L.qlin_gemv(C.byref(w), None, 1, fake, q.OUT_BF16, C.byref(ex)) == q.ERR_INVALID_ARG
    # K not a multiple of the group
    bad = _weights(q.Q4_G64, 256, 96)
    assert L.qlin_gemv(C.byref(bad), fake, 1, fake, q.OUT_BF16, C.byref(ex)) == q.ERR_INVALID_ARG
    # Q5, Q3 and Q6 need their second plane
    for fmt in (q.Q5_G64, q.Q3_G64, q.Q6_G64):
        w5 = _weights(fmt, 256, 512)
        w5.hibits = None
        assert L.qlin_gemv(C.byref(w5), fake, 1, fake, q.OUT_BF16, C.byref(ex)) == q.ERR_INVALID_ARG
    # int8 route: permission, formats, activation arguments
    a16 = _weights(q.Q4_G64, 256, 512, flags=0)
    assert L.qlin_gemm_a8(C.byref(a16), fake, None, None, 256, fake, q.OUT_BF16, 0, None,
                          C.byref(ex)) == q.ERR_NOT_PERMITTED
    for fmt in (q.Q8_G32, q.FP8_ROW, q.BF16):
        wf = _weights(fmt, 256, 512, flags=q.ALLOW_A8)
        assert L.qlin_gemm_a8(C.byref(wf), fake, None, None, 256, fake, q.OUT_BF16, 0, None,
                              C.byref(ex)) == q.ERR_UNSUPPORTED
    # both or neither activation form
    assert L.qlin_gemm_a8(C.byref(w), fake, fake, fake, 256, fake, q.OUT_BF16, 0, None,
                          C.byref(ex)) == q.ERR_INVALID_ARG
    assert L.qlin_gemm_a8(C.byref(w), None, None, None, 256, fake, q.OUT_BF16, 0, None,
                          C.byref(ex)) == q.ERR_INVALID_ARG
    # debug dump requested without a buffer
    assert L.qlin_gemm_a8(C.byref(w), fake, None, None, 256, fake, q.OUT_BF16,
                          q.DEBUG_GROUP_SUMS, None, C.byref(ex)) == q.ERR_INVALID_ARG
    # decode / quantize argument checks
    assert L.qlin_decode_mxfp8(fake, fake, 4, 48, fake, C.byref(ex)) == q.ERR_INVALID_ARG
    assert L.qlin_quantize_act(fake, 4, 96, fake, fake, C.byref(ex)) == q.ERR_INVALID_ARG
    assert L.qlin_quantize_act(odd, 4, 128, fake, fake, C.byref(ex)) == q.ERR_INVALID_ARG
    # pack: unknown source kind, MLX source needs K % 128
    assert L.qlin_pack_weights(9, fake, None, None, C.byref(w), C.byref(ex)) == q.ERR_INVALID_ARG
    w64 = _weights(q.Q4_G64, 4, 64)
    assert L.qlin_pack_weights(q.SRC_MLX_AFFINE8, fake, fake, fake, C.byref(w64),
                               C.byref(ex)) == q.ERR_INVALID_ARG
    # block-128 FP8 source needs its scale grid, 16-byte aligned
    assert L.qlin_pack_weights(q.SRC_FP8_BLOCK128, fake, None, None, C.byref(w64),
                               C.byref(ex)) == q.ERR_INVALID_ARG
    assert L.qlin_pack_weights(q.SRC_FP8_BLOCK128, fake, odd, None, C.byref(w64),
                               C.byref(ex)) == q.ERR_INVALID_ARG

    # FP8-activation route: FP8_ROW weights only, one activation form, K % 16
    w8 = _weights(q.FP8_ROW, 256, 512)
    assert L.qlin_gemm_fp8(C.byref(w), fake, None, None, 4, fake, q.OUT_BF16,
                           C.byref(ex)) == q.ERR_UNSUPPORTED
    assert L.qlin_gemm_fp8(C.byref(w8), fake, fake, fake, 4, fake, q.OUT_BF16,
                           C.byref(ex)) == q.ERR_INVALID_ARG
    assert L.qlin_gemm_fp8(C.byref(w8), None, fake, None, 4, fake, q.OUT_BF16,
                           C.byref(ex)) == q.ERR_INVALID_ARG
    assert L.qlin_gemm_fp8(C.byref(w8), None, fake, odd, 4, fake, q.OUT_BF16,
                           C.byref(ex)) == q.ERR_INVALID_ARG
    assert L.qlin_gemm_fp8(C.byref(w8), fake, None, None, 0, fake, q.OUT_BF16,
                           C.byref(ex)) == q.ERR_INVALID_ARG
    assert L.qlin_gemm_fp8(C.byref(w8), fake, None, None, 4, fake, 5,
                           C.byref(ex)) == q.ERR_INVALID_ARG
    assert L.qlin_quantize_act_fp8(fake, 4, 40, fake, fake, C.byref(ex)) == q.ERR_INVALID_ARG
    assert L.qlin_quantize_act_fp8(fake, 4, 48, fake, odd, C.byref(ex)) == q.ERR_INVALID_ARG
    b = C.c_size_t()
    assert L.qlin_gemm_fp8_workspace_bytes(3, 40, C.byref(b)) == q.ERR_INVALID_ARG
    assert L.qlin_gemm_fp8_workspace_bytes(3, 4096, C.byref(b)) == q.OK
    assert b.value == (3 * 4096 + 255) // 256 * 256 + 3 * 4


def test_product_path_has_no_cpu_fallback():
    """The binding refuses CPU tensors instead of computing on the host."""
    import torch
    pw = q.PackedWeights.__new__(q.PackedWeights)
    with pytest.raises((ValueError, RuntimeError, AssertionError)):
        q._ptr(torch.zeros(4))
    src = open(os.path.join(ROOT, "quantized_weight_linear_qlin_b200", "__init__.py")).read()
    assert "import oracle" not in src and "from oracle" not in src
