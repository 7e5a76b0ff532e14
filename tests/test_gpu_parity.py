"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.  Bit-exact for codes, scales, decodes, activation codes
and int32 group sums; within the stated tolerances for FP32/BF16 outputs:
|y - y_ref| <= 1e-3 * sum|w||x| (BF16 route) and <= 5e-6 * sum|q ws||qa as|
(int8 route, FP32 output before rounding); a BF16 output may differ by one
more half BF16 ulp of |y_ref| (its own rounding: half an ulp is at most 2^-8 of the value)."""
import numpy as np
import pytest
import torch

import oracle
import quantized_weight_linear_qlin_b200 as q
import synth

pytestmark = pytest.mark.gpu

FMTS = {"q4": q.Q4_G64, "q5": q.Q5_G64, "q8": q.Q8_G32, "fp8": q.FP8_ROW, "bf16": q.BF16,
        "q3": q.Q3_G64, "q6": q.Q6_G64}
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from quantized_weight_linear_qlin_b200 import _build
    _build.build()
    q.lib()


def bits16(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_value(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def gpu_packed_to_numpy(pw):
    n, k = pw.n, pw.k
    cdt, cshape, hshape, sdt, sshape = oracle.packed_shapes(pw.fmt, n, k)
    codes = pw.codes.cpu().numpy().view(cdt).reshape(cshape)
    hib = pw.hibits.cpu().numpy().reshape(hshape) if hshape else None
    sc = pw.scales.cpu().numpy().view(sdt).reshape(sshape) if sshape else None
    return {"fmt": pw.fmt, "n": n, "k": k, "codes": codes, "hibits": hib, "scales": sc}


def pack_gpu(fmt, w_dev, allow_a8=False, src_kind=q.SRC_F32, aux0=None, aux1=None):
    n, k = w_dev.shape[0], (w_dev.shape[1] * (4 if src_kind == q.SRC_MXFP8 else 1))
    pw = q.PackedWeights(fmt, n, k, device=DEV, allow_a8=allow_a8)
    q.qlin_pack_weights(src_kind, w_dev, pw, aux0=aux0, aux1=aux1)
    return pw


def assert_packed_equal(pw, ref):
    got = gpu_packed_to_numpy(pw)
    for key in ("codes", "hibits", "scales"):
        if ref[key] is None:
            continue
        assert np.array_equal(got[key], ref[key]), key


# ---------------------------------------------------------------------------
# packing and decoding: bit-exact
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("fmt", list(FMTS))
@pytest.mark.parametrize("shape", [(200, 320), (129, 1024)])
def test_pack_from_f32_bit_exact(fmt, shape):
    n, k = shape
    w = synth.weights_f32(n, k, seed=100 + n)
    w[3, :64] = 0.0          # an all-zero group
    w[5] = 0.0               # an all-zero row (FP8 row scale 0)
    w[7, 10] = 1e-30         # a tiny value next to a large one
    w[8, :] *= 1e3
    ref = oracle.pack(FMTS[fmt], w.numpy())
    pw = pack_gpu(FMTS[fmt], w.to(DEV))
    torch.cuda.synchronize()
    assert_packed_equal(pw, ref)


@pytest.mark.parametrize("fmt", ["q4", "q5", "q8", "fp8", "q3", "q6"])
def test_pack_from_bf16_bit_exact(fmt):
    w = synth.weights_f32(96, 512, seed=7).to(torch.bfloat16)
    ref = oracle.pack(FMTS[fmt], w.float().numpy())
    pw = pack_gpu(FMTS[fmt], w.to(DEV).view(torch.int16), src_kind=q.SRC_BF16)
    torch.cuda.synchronize()
    assert_packed_equal(pw, ref)


@pytest.mark.parametrize("fmt", ["q4", "q5", "q8", "fp8", "bf16", "q3", "q6"])
def test_pack_from_mxfp8_bit_exact(fmt):
    rows, cols = 64, 512
    words, scales = synth.mxfp8_source(rows, cols, seed=11)
    dec = oracle.decode_mxfp8(words.numpy().view(np.uint32), scales.numpy(), rows, cols)
    ref = oracle.pack(FMTS[fmt], bf16_value(dec).astype(np.float32))
    pw = pack_gpu(FMTS[fmt], words.to(DEV), src_kind=q.SRC_MXFP8, aux0=scales.to(DEV))
    torch.cuda.synchronize()
    assert_packed_equal(pw, ref)


@pytest.mark.parametrize("fmt", ["q4", "q8", "bf16"])
def test_pack_from_mlx_affine_bit_exact(fmt):
    rows, cols = 48, 384
    qq, s16, b16 = synth.mlx_affine_source(rows, cols, seed=13)
    dec = oracle.decode_mlx_affine(qq.numpy(), s16.numpy().view(np.uint16), b16.numpy().view(np.uint16),
                                   rows, cols)
    ref = oracle.pack(FMTS[fmt], bf16_value(dec).astype(np.float32))
    pw = q.PackedWeights(FMTS[fmt], rows, cols, device=DEV)
    q.qlin_pack_weights(q.SRC_MLX_AFFINE8, qq.to(DEV), pw, aux0=s16.to(DEV), aux1=b16.to(DEV))
    torch.cuda.synchronize()
    assert_packed_equal(pw, ref)


def test_decode_mxfp8_exhaustive_bit_exact():
    # every code at every block exponent, NaNs included
    codes = np.tile(np.arange(256, dtype=np.uint8), 256).reshape(256, 256)
    words = codes.view(np.uint32).reshape(256, 64)
    scales = np.repeat(np.arange(256, dtype=np.uint8)[:, None], 8, axis=1)
    ref = oracle.decode_mxfp8(words, scales, 256, 256)
    out = torch.empty(256, 256, dtype=torch.int16, device=DEV)
    q.qlin_decode_mxfp8(torch.from_numpy(words.view(np.int32)).to(DEV),
                        torch.from_numpy(scales).to(DEV), 256, 256, out)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy().view(np.uint16), ref)


def test_decode_mxfp8_full_size_bit_exact():
    rows, cols = 5120, 17408
    words, scales = synth.mxfp8_source(rows, cols, seed=synth.seed_for(2, 1), device=DEV)
    out = torch.empty(rows, cols, dtype=torch.int16, device=DEV)
    q.qlin_decode_mxfp8(words, scales, rows, cols, out)
    sel = torch.arange(0, rows, 97)
    ref = oracle.decode_mxfp8(words[sel].cpu().numpy().view(np.uint32), scales[sel].cpu().numpy(),
                              len(sel), cols)
    torch.cuda.synchronize()
    assert np.array_equal(out[sel.to(DEV)].cpu().numpy().view(np.uint16), ref)


# ---------------------------------------------------------------------------
# activation quantizer: bit-exact
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("shape", [(1, 64), (37, 320), (130, 5120), (5, 17408)])
def test_quantize_act_bit_exact(shape):
    t, k = shape
    x = synth.activations_bf16(t, k, seed=t + k)
    xf = x.float()
    xf[0, :64] = 0.0                     # zero group
    if t > 2:
        xf[2, 64:128] = 3.0e38           # huge values
        xf[1, :64] = 1e-38               # tiny values
    x = xf.to(torch.bfloat16)
    qa_ref, as_ref = oracle.quantize_act(bits16(x))
    xq = torch.empty(t, k, dtype=torch.int8, device=DEV)
    xs = torch.empty(t, k // 64, dtype=torch.float32, device=DEV)
    q.qlin_quantize_act(x.to(DEV), xq, xs)
    torch.cuda.synchronize()
    assert np.array_equal(xq.cpu().numpy(), qa_ref)
    assert np.array_equal(xs.cpu().numpy().view(np.uint32), as_ref.view(np.uint32))


def test_quantize_act_bit_exact_wide_ranges():
    """33 M values whose 64-groups span the whole BF16 exponent range (each
    group scaled by its own power of two, some groups subnormal), against the
    oracle's IEEE quotient and round-to-nearest-even."""
    t, k = 4096, 8192
    g = torch.Generator().manual_seed(1234)
    x = torch.randn(t, k, generator=g)
    e = torch.randint(-140, 120, (t, k // 64), generator=g).float()
    x = (x.view(t, k // 64, 64) * torch.exp2(e)[..., None]).view(t, k)
    x = x.to(torch.bfloat16)
    qa_ref, as_ref = oracle.quantize_act(bits16(x))
    xq = torch.empty(t, k, dtype=torch.int8, device=DEV)
    xs = torch.empty(t, k // 64, dtype=torch.float32, device=DEV)
    q.qlin_quantize_act(x.to(DEV), xq, xs)
    torch.cuda.synchronize()
    assert np.array_equal(xs.cpu().numpy().view(np.uint32), as_ref.view(np.uint32))
    got = xq.cpu().numpy()
    bad = np.argwhere(got != qa_ref)
    assert bad.size == 0, (bad[:5], got[tuple(bad[0])], qa_ref[tuple(bad[0])])


# ---------------------------------------------------------------------------
# BF16-route GEMV
# ---------------------------------------------------------------------------
def check_gemv(pw, ref, x, y_dtype=q.OUT_F32, ws=None):
    t = x.shape[0]
    y = torch.empty(t, pw.n, dtype=torch.float32 if y_dtype == q.OUT_F32 else torch.bfloat16,
                    device=DEV)
    if ws is None:
        ws = q.Workspace(DEV)
    ws.ensure(q.qlin_gemv_workspace_bytes(pw, t))
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    q.qlin_gemv(pw, x.to(DEV), y, y_dtype, workspace=ws, dev_status=status)
    yr, br = oracle.gemv(ref, bits16(x), nthreads=8)
    torch.cuda.synchronize()
    assert status.item() == 0
    got = y.float().cpu().numpy().astype(np.float64)
    tol = 1e-3 * br
    if y_dtype == q.OUT_BF16:
        tol = tol + np.abs(yr) * 2.0 ** -8
    bad = np.abs(got - yr) > tol
    assert not bad.any(), (np.argwhere(bad)[:5], got[bad][:5], yr[bad][:5])
    return got, yr


@pytest.mark.parametrize("fmt", list(FMTS))
@pytest.mark.parametrize("t", [1, 3, 4, 5, 17, 33, 64])
def test_gemv_small_shapes(fmt, t):
    n, k = 200, 1216  # ragged rows; K not a multiple of the K-split
    w = synth.weights_f32(n, k, seed=200 + t)
    x = synth.activations_bf16(t, k, seed=300 + t)
    ref = oracle.pack(FMTS[fmt], w.numpy())
    pw = pack_gpu(FMTS[fmt], w.to(DEV))
    check_gemv(pw, ref, x, q.OUT_F32)


@pytest.mark.parametrize("fmt", list(FMTS))
@pytest.mark.parametrize("t", [1, 3, 16, 17, 33, 48, 64])
def test_gemv_tensor_core_path_split_tiles(fmt, t):
    """K = 1536 is whole units for every format, so the tensor-core kernel runs;
    200 rows x 3 units per tile over 6 CTAs splits every tile three ways."""
    n, k = 200, 1536
    w = synth.weights_f32(n, k, seed=600 + t)
    x = synth.activations_bf16(t, k, seed=700 + t)
    ref = oracle.pack(FMTS[fmt], w.numpy())
    pw = pack_gpu(FMTS[fmt], w.to(DEV))
    ws = q.Workspace(DEV)
    check_gemv(pw, ref, x, q.OUT_F32, ws=ws)
    # a second call on the same workspace: the split-tile counters were left at zero
    check_gemv(pw, ref, x, q.OUT_BF16, ws=ws)
    counters = ws.buffer[: ((n + 127) // 128) * 4]
    assert not counters.any()


@pytest.mark.parametrize("fmt", ["q4", "q5", "fp8", "q3", "q6"])
def test_gemv_bf16_output_and_long_k(fmt):
    n, k, t = 96, 17408, 2
    w = synth.weights_f32(n, k, seed=5)
    x = synth.activations_bf16(t, k, seed=6)
    ref = oracle.pack(FMTS[fmt], w.numpy())
    pw = pack_gpu(FMTS[fmt], w.to(DEV))
    check_gemv(pw, ref, x, q.OUT_BF16)


@pytest.mark.parametrize("t", [65, 130, 512, 1792])
def test_gemv_bf16_weights_prefill_sizes(t):
    # GDN a/b projection kept in BF16: 96 x 5120 at a prefill chunk (tokens on
    # the MMA's M side, K split over CTAs; 65 and 130 leave ragged token tiles)
    n, k = 96, 5120
    w = synth.weights_f32(n, k, seed=9)
    x = synth.activations_bf16(t, k, seed=10)
    ref = oracle.pack(q.BF16, w.numpy())
    pw = pack_gpu(q.BF16, w.to(DEV))
    check_gemv(pw, ref, x, q.OUT_F32)


@pytest.mark.parametrize("n,k,t,y_dtype", [(80, 1024, 300, q.OUT_BF16), (256, 640, 129, q.OUT_F32),
                                           (16, 4096, 2000, q.OUT_F32), (200, 192, 777, q.OUT_BF16),
                                           (96, 5120, 1100, q.OUT_BF16), (64, 2048, 1025, q.OUT_F32),
                                           (90, 512, 333, q.OUT_BF16), (250, 1024, 1500, q.OUT_F32)])
def test_gemv_bf16_weights_prefill_ragged_n(n, k, t, y_dtype):
    """Small BF16 projections at prefill sizes: N padded inside the kernel
    (80 -> 96, 200 and 250 -> 256), few K stages (K = 192: one part), BF16 and
    FP32 out; 1100 and 1025 tokens leave the last CTA's second 128-token
    sub-tile wholly or all but one token out of range; N = 90 and 250 are not
    multiples of 4 (element-wise stores of the cluster reduction)."""
    w = synth.weights_f32(n, k, seed=11 + n)
    x = synth.activations_bf16(t, k, seed=12 + t)
    ref = oracle.pack(q.BF16, w.numpy())
    pw = pack_gpu(q.BF16, w.to(DEV))
    check_gemv(pw, ref, x, y_dtype)


@pytest.mark.parametrize("t", [8192, 40000])
def test_gemv_bf16_gdn_ab_full_size_sampled(t):
    """The GDN a/b projection 96 x 5120 at an 8192-token prefill chunk (K split
    over a cluster of CTAs, reduced through distributed shared memory) and at
    40000 tokens (one part per tile): sampled tokens, always the first and the
    last (ragged) tile."""
    n, k = 96, 5120
    w = synth.weights_f32(n, k, seed=synth.seed_for(5, 0), device=DEV)
    x = synth.activations_bf16(t, k, seed=synth.seed_for(5, 1), device=DEV)
    pw = pack_gpu(q.BF16, w)
    y = torch.empty(t, n, dtype=torch.float32, device=DEV)
    ws = q.Workspace(DEV).ensure(q.qlin_gemv_workspace_bytes(pw, t))
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    q.qlin_gemv(pw, x, y, q.OUT_F32, workspace=ws, dev_status=status)
    g = torch.Generator().manual_seed(t)
    toks = torch.cat([torch.randperm(t, generator=g)[:40], torch.tensor([0, 127, 128, t - 1])]).unique()
    ref = oracle.pack(q.BF16, w.cpu().numpy())
    yr, br = oracle.gemv(ref, bits16(x[toks.to(DEV)]), nthreads=8)
    torch.cuda.synchronize()
    assert status.item() == 0
    got = y[toks.to(DEV)].cpu().numpy().astype(np.float64)
    bad = np.abs(got - yr) > 1e-3 * br
    assert not bad.any(), (np.argwhere(bad)[:5], got[bad][:5], yr[bad][:5])


@pytest.mark.parametrize("name,fmt,n,k,t", [
    ("gate_up_q4", q.Q4_G64, 34816, 5120, 4),
    ("down_q5", q.Q5_G64, 5120, 17408, 33),
    ("q8_5120", q.Q8_G32, 5120, 5120, 17),
    ("head_fp8", q.FP8_ROW, 152064, 5120, 1),
    # the head in both formats at the top of the verify range (FP8-vs-Q8 crossover)
    ("head_q8_T64", q.Q8_G32, 152064, 5120, 64),
    ("head_fp8_T64", q.FP8_ROW, 152064, 5120, 64),
    # the other group-64 widths at the MLP shapes
    ("gate_up_q3", q.Q3_G64, 34816, 5120, 1),
    ("gate_up_q3_T17", q.Q3_G64, 34816, 5120, 17),
    ("down_q6", q.Q6_G64, 5120, 17408, 33),
    ("down_q6_T1", q.Q6_G64, 5120, 17408, 1),
])
def test_gemv_full_size_sampled_rows(name, fmt, n, k, t):
    """Full-size weights in the bench's launch configuration; the oracle
    checks a sample of rows (packing is row-independent)."""
    w = synth.weights_f32(n, k, seed=synth.seed_for(1, 0), device=DEV)
    x = synth.activations_bf16(t, k, seed=synth.seed_for(1, 1), device=DEV)
    pw = pack_gpu(fmt, w)
    y = torch.empty(t, n, dtype=torch.float32, device=DEV)
    ws = q.Workspace(DEV).ensure(q.qlin_gemv_workspace_bytes(pw, t))
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    q.qlin_gemv(pw, x, y, q.OUT_F32, workspace=ws, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0  # no on-chip wait ran out
    g = torch.Generator().manual_seed(1)
    rows = torch.cat([torch.randperm(n, generator=g)[:61], torch.tensor([0, n - 1])])
    ref = oracle.pack(fmt, w[rows.to(DEV)].cpu().numpy())
    got_packed = {"codes": None}
    yr, br = oracle.gemv(ref, bits16(x), nthreads=8)
    torch.cuda.synchronize()
    got = y[:, rows.to(DEV)].cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - yr) <= 1e-3 * br)
    # packed rows bit-exact as well
    sub = gpu_packed_to_numpy(pw)
    for key in ("codes", "hibits", "scales"):
        if ref[key] is not None:
            assert np.array_equal(sub[key][rows.numpy()], ref[key]), key
    del got_packed


@pytest.mark.parametrize("fmt", list(FMTS))
@pytest.mark.parametrize("t", [1, 17, 33, 64])
def test_gemv_several_units_per_cta(fmt, t):
    """4096 x 4096: every CTA walks several units, so each ring and barrier of
    the pipeline goes through several phases; sampled rows against the oracle
    and no on-chip wait may run out."""
    n, k = 4096, 4096
    w = synth.weights_f32(n, k, seed=800 + t, device=DEV)
    x = synth.activations_bf16(t, k, seed=900 + t)
    pw = pack_gpu(FMTS[fmt], w)
    y = torch.empty(t, n, dtype=torch.float32, device=DEV)
    ws = q.Workspace(DEV).ensure(q.qlin_gemv_workspace_bytes(pw, t))
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    for _ in range(2):
        q.qlin_gemv(pw, x.to(DEV), y, q.OUT_F32, workspace=ws, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    g = torch.Generator().manual_seed(t)
    rows = torch.cat([torch.randperm(n, generator=g)[:45], torch.tensor([0, 127, 128, n - 1])])
    ref = oracle.pack(FMTS[fmt], w[rows.to(DEV)].cpu().numpy())
    yr, br = oracle.gemv(ref, bits16(x), nthreads=8)
    got = y[:, rows.to(DEV)].cpu().numpy().astype(np.float64)
    bad = np.abs(got - yr) > 1e-3 * br
    assert not bad.any(), (np.argwhere(bad)[:5], got[bad][:5], yr[bad][:5])


# ---------------------------------------------------------------------------
# int8 route
# ---------------------------------------------------------------------------
def act_ws_bytes(t, k):
    """The activation part of the int8 route's workspace (codes + scales)."""
    return (t * k + 255) // 256 * 256 + t * (k // 64) * 4


def run_gemm_a8(pw, x, fused=True, debug=True, y_dtype=q.OUT_F32, full_ws=True):
    """full_ws: the recommended workspace (weights expanded to int8 once, TMA-fed
    GEMM); else only the activation part (codes expanded on chip)."""
    t, k = x.shape
    n = pw.n
    xd = x.to(DEV)
    y = torch.empty(t, n, dtype=torch.float32 if y_dtype == q.OUT_F32 else torch.bfloat16, device=DEV)
    dbg = torch.zeros(t, n, k // 64, dtype=torch.int32, device=DEV) if debug else None
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    flags = q.DEBUG_GROUP_SUMS if debug else 0
    if fused:
        ws = q.Workspace(DEV).ensure(q.qlin_gemm_a8_workspace_bytes(t, n, k) if full_ws else act_ws_bytes(t, k))
        q.qlin_gemm_a8(pw, y, x=xd, y_dtype=y_dtype, flags=flags, sums_dbg=dbg, workspace=ws,
                       dev_status=status)
    else:
        xq = torch.empty(t, k, dtype=torch.int8, device=DEV)
        xs = torch.empty(t, k // 64, dtype=torch.float32, device=DEV)
        q.qlin_quantize_act(xd, xq, xs)
        q.qlin_gemm_a8(pw, y, xq=xq, xs=xs, y_dtype=y_dtype, flags=flags, sums_dbg=dbg,
                       dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    return y, dbg


@pytest.mark.parametrize("full_ws", [True, False])
@pytest.mark.parametrize("fmt", ["q4", "q5", "q3", "q6"])
@pytest.mark.parametrize("n,k,t", [(128, 256, 128), (256, 512, 130), (200, 640, 257), (384, 1152, 1),
                                   (128, 5120, 64)])
def test_gemm_a8_group_sums_bit_exact_and_output(fmt, n, k, t, full_ws):
    w = synth.weights_f32(n, k, seed=400 + n + k)
    x = synth.activations_bf16(t, k, seed=500 + t)
    ref = oracle.pack(FMTS[fmt], w.numpy())
    pw = pack_gpu(FMTS[fmt], w.to(DEV), allow_a8=True)
    y, dbg = run_gemm_a8(pw, x, fused=True, debug=True, full_ws=full_ws)
    qa, as_ = oracle.quantize_act(bits16(x))
    S = oracle.group_sums(ref, qa)
    assert np.array_equal(dbg.cpu().numpy(), S)
    yr, br = oracle.gemm_a8(ref, qa, as_, nthreads=8)
    got = y.cpu().numpy().astype(np.float64)
    bad = np.abs(got - yr) > 5e-6 * br
    assert not bad.any(), (np.argwhere(bad)[:5], got[bad][:5], yr[bad][:5])


@pytest.mark.parametrize("fmt", ["q4", "q5", "q3", "q6"])
def test_gemm_a8_prequantized_and_bf16_out(fmt):
    n, k, t = 256, 1024, 300
    w = synth.weights_f32(n, k, seed=41)
    x = synth.activations_bf16(t, k, seed=42)
    ref = oracle.pack(FMTS[fmt], w.numpy())
    pw = pack_gpu(FMTS[fmt], w.to(DEV), allow_a8=True)
    y, _ = run_gemm_a8(pw, x, fused=False, debug=False, y_dtype=q.OUT_BF16)
    qa, as_ = oracle.quantize_act(bits16(x))
    yr, br = oracle.gemm_a8(ref, qa, as_, nthreads=8)
    got = y.float().cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - yr) <= 5e-6 * br + np.abs(yr) * 2.0 ** -8)


@pytest.mark.parametrize("fmt,qmax", [(q.Q3_G64, 3), (q.Q6_G64, 31)])
def test_gemm_a8_extreme_codes_q3_q6(fmt, qmax):
    """Every code at +-Qmax against activation codes +-127: |S| = 64 * Qmax * 127, exact."""
    n, k, t = 128, 512, 128
    w = torch.full((n, k), 0.5, dtype=torch.float32)
    w[::2] *= -1
    x = torch.full((t, k), 2.0, dtype=torch.float32).to(torch.bfloat16)
    pw = pack_gpu(fmt, w.to(DEV), allow_a8=True)
    y, dbg = run_gemm_a8(pw, x, fused=True, debug=True)
    S = dbg.cpu().numpy()
    assert np.all(np.abs(S) == 64 * qmax * 127)
    ref = oracle.pack(fmt, w.numpy())
    qa, as_ = oracle.quantize_act(bits16(x))
    assert np.array_equal(S, oracle.group_sums(ref, qa))


def test_gemm_a8_extreme_codes():
    """All codes at their extremes: |S| = 64 * 15 * 127 per group, exact."""
    n, k, t = 128, 512, 128
    w = torch.full((n, k), 0.5, dtype=torch.float32)
    w[::2] *= -1
    x = torch.full((t, k), 2.0, dtype=torch.float32).to(torch.bfloat16)
    pw = pack_gpu(q.Q5_G64, w.to(DEV), allow_a8=True)
    y, dbg = run_gemm_a8(pw, x, fused=True, debug=True)
    S = dbg.cpu().numpy()
    assert np.all(np.abs(S) == 64 * 15 * 127)
    ref = oracle.pack(q.Q5_G64, w.numpy())
    qa, as_ = oracle.quantize_act(bits16(x))
    assert np.array_equal(S, oracle.group_sums(ref, qa))


@pytest.mark.parametrize("name,fmt,n,k", [("gate_up_q4", q.Q4_G64, 34816, 5120),
                                          ("down_q5", q.Q5_G64, 5120, 17408),
                                          ("gate_up_q3", q.Q3_G64, 34816, 5120),
                                          ("down_q6", q.Q6_G64, 5120, 17408)])
def test_gemm_a8_full_size_sampled(name, fmt, n, k):
    t = 2048
    w = synth.weights_f32(n, k, seed=synth.seed_for(3, 0), device=DEV)
    x = synth.activations_bf16(t, k, seed=synth.seed_for(3, 1), device=DEV)
    pw = pack_gpu(fmt, w, allow_a8=True)
    y = torch.empty(t, n, dtype=torch.float32, device=DEV)
    ws = q.Workspace(DEV).ensure(q.qlin_gemm_a8_workspace_bytes(t, n, k))
    q.qlin_gemm_a8(pw, y, x=x, y_dtype=q.OUT_F32, workspace=ws)
    g = torch.Generator().manual_seed(3)
    rows = torch.randperm(n, generator=g)[:24]
    toks = torch.cat([torch.randperm(t, generator=g)[:14], torch.tensor([0, t - 1])])
    ref = oracle.pack(fmt, w[rows.to(DEV)].cpu().numpy())
    qa, as_ = oracle.quantize_act(bits16(x[toks.to(DEV)]))
    yr, br = oracle.gemm_a8(ref, qa, as_, nthreads=8)
    torch.cuda.synchronize()
    got = y[toks.to(DEV)][:, rows.to(DEV)].cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - yr) <= 5e-6 * br)


# ---------------------------------------------------------------------------
# ties: quotients exactly on k + 1/2 (hand-worked groups, tests/golden)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("name,fmt", [("q4_group", "q4"), ("q5_group", "q5"), ("q8_group", "q8"),
                                      ("q3_group", "q3"), ("q6_group", "q6")])
def test_pack_ties_bit_exact(golden, name, fmt):
    ex = golden["ties"][name]
    gs = 32 if fmt == "q8" else 64
    w = torch.full((3, 4 * gs), float(ex["rest"]), dtype=torch.float32)
    for r in range(3):
        w[r, r * gs:r * gs + len(ex["w_head"])] = torch.tensor(ex["w_head"]) * (-1) ** r
    ref = oracle.pack(FMTS[fmt], w.numpy())
    pw = pack_gpu(FMTS[fmt], w.to(DEV))
    torch.cuda.synchronize()
    assert_packed_equal(pw, ref)


@pytest.mark.parametrize("name", ["act_group_unit_scale", "act_group_half_scale"])
def test_quantize_act_ties_bit_exact(golden, name):
    ex = golden["ties"][name]
    x = torch.full((2, 128), float(ex["rest"]), dtype=torch.float32)
    x[0, :len(ex["x_head"])] = torch.tensor(ex["x_head"])
    x[1, 64:64 + len(ex["x_head"])] = -torch.tensor(ex["x_head"])
    x = x.to(torch.bfloat16)
    qa_ref, as_ref = oracle.quantize_act(bits16(x))
    assert list(qa_ref[0, :len(ex["codes_head"])]) == ex["codes_head"]
    xq = torch.empty(2, 128, dtype=torch.int8, device=DEV)
    xs = torch.empty(2, 2, dtype=torch.float32, device=DEV)
    q.qlin_quantize_act(x.to(DEV), xq, xs)
    torch.cuda.synchronize()
    assert np.array_equal(xq.cpu().numpy(), qa_ref)
    assert np.array_equal(xs.cpu().numpy().view(np.uint32), as_ref.view(np.uint32))


# ---------------------------------------------------------------------------
# one 27B-class layer's projections on the int8 route at the long-chunk
# prefill sizes, and the decode MLP with the formats swapped
# ---------------------------------------------------------------------------
LAYER = [("q", 6144, 5120), ("k", 1024, 5120), ("v", 1024, 5120), ("o", 5120, 6144),
         ("gate", 17408, 5120), ("up", 17408, 5120), ("down", 5120, 17408)]


@pytest.mark.parametrize("t", [512, 1792, 8192])
@pytest.mark.parametrize("variant", ["mixed", "all_q5"])
@pytest.mark.parametrize("proj", [p[0] for p in LAYER])
def test_gemm_a8_layer_sweep_sampled(proj, variant, t):
    """Sampled rows and tokens, always including the last row tile and the
    last token tile, at the int8 route's 5e-6 bound; the full output is
    written (no on-chip wait may run out)."""
    _, n, k = next(p for p in LAYER if p[0] == proj)
    fmt = q.Q5_G64 if (variant == "all_q5" or proj == "down") else q.Q4_G64
    w = synth.weights_f32(n, k, seed=synth.seed_for(4, 10 + LAYER.index((proj, n, k))), device=DEV)
    x = synth.activations_bf16(t, k, seed=synth.seed_for(4, 30 + k % 97), device=DEV)
    pw = pack_gpu(fmt, w, allow_a8=True)
    y = torch.empty(t, n, dtype=torch.bfloat16, device=DEV)
    ws = q.Workspace(DEV).ensure(q.qlin_gemm_a8_workspace_bytes(t, n, k))
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    q.qlin_gemm_a8(pw, y, x=x, y_dtype=q.OUT_BF16, workspace=ws, dev_status=status)
    g = torch.Generator().manual_seed(n + t)
    rows = torch.cat([torch.randperm(n, generator=g)[:10], torch.tensor([n - 128, n - 1])]).unique()
    toks = torch.cat([torch.randperm(t, generator=g)[:8], torch.tensor([0, t - 128, t - 1])]).unique()
    ref = oracle.pack(fmt, w[rows.to(DEV)].cpu().numpy())
    qa, as_ = oracle.quantize_act(bits16(x[toks.to(DEV)]))
    yr, br = oracle.gemm_a8(ref, qa, as_, nthreads=8)
    torch.cuda.synchronize()
    assert status.item() == 0
    got = y[toks.to(DEV)][:, rows.to(DEV)].float().cpu().numpy().astype(np.float64)
    bad = np.abs(got - yr) > 5e-6 * br + np.abs(yr) * 2.0 ** -8
    assert not bad.any(), (np.argwhere(bad)[:5], got[bad][:5], yr[bad][:5])
    assert torch.isfinite(y.float()).all()


@pytest.mark.parametrize("t", [1, 4, 17, 33])
@pytest.mark.parametrize("name,fmt,n,k", [("gate_up_q5", q.Q5_G64, 34816, 5120),
                                          ("down_q4", q.Q4_G64, 5120, 17408)])
def test_gemv_decode_mlp_swapped_formats(name, fmt, n, k, t):
    w = synth.weights_f32(n, k, seed=synth.seed_for(1, 40), device=DEV)
    x = synth.activations_bf16(t, k, seed=synth.seed_for(1, 41), device=DEV)
    pw = pack_gpu(fmt, w)
    y = torch.empty(t, n, dtype=torch.bfloat16, device=DEV)
    ws = q.Workspace(DEV).ensure(q.qlin_gemv_workspace_bytes(pw, t))
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    q.qlin_gemv(pw, x, y, q.OUT_BF16, workspace=ws, dev_status=status)
    g = torch.Generator().manual_seed(t)
    rows = torch.cat([torch.randperm(n, generator=g)[:40], torch.tensor([0, n - 1])]).unique()
    ref = oracle.pack(fmt, w[rows.to(DEV)].cpu().numpy())
    yr, br = oracle.gemv(ref, bits16(x), nthreads=8)
    torch.cuda.synchronize()
    assert status.item() == 0
    got = y[:, rows.to(DEV)].float().cpu().numpy().astype(np.float64)
    bad = np.abs(got - yr) > 1e-3 * br + np.abs(yr) * 2.0 ** -8
    assert not bad.any(), (np.argwhere(bad)[:5], got[bad][:5], yr[bad][:5])


def test_gemv_q8_head_overflowing_scales_exact_path():
    """A Q8 group-32 matrix of 2^27 weights takes the kernel that folds the
    FP16 group scale into an FP16 operand; rows whose scale is above 511.75
    (q * s could overflow FP16) are recomputed exactly on the CUDA cores."""
    n, k, t = 32768, 4096, 3
    w = synth.weights_f32(n, k, seed=77, device=DEV)
    huge = torch.tensor([5, 1000, 4097, n - 1], device=DEV)
    w[huge] = w[huge] * 5e6  # |w| up to ~5e5: group scales ~4e3
    x = synth.activations_bf16(t, k, seed=78, device=DEV)
    pw = pack_gpu(q.Q8_G32, w)
    y = torch.empty(t, n, dtype=torch.float32, device=DEV)
    ws = q.Workspace(DEV).ensure(q.qlin_gemv_workspace_bytes(pw, t))
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    q.qlin_gemv(pw, x, y, q.OUT_F32, workspace=ws, dev_status=status)
    rows = torch.cat([huge.cpu(), torch.tensor([0, 6, 999, 1001, 4096, n - 2])])
    ref = oracle.pack(q.Q8_G32, w[rows.to(DEV)].cpu().numpy())
    assert (oracle.dequant(ref)[:4] != 0).any()
    yr, br = oracle.gemv(ref, bits16(x), nthreads=8)
    torch.cuda.synchronize()
    assert status.item() == 0
    got = y[:, rows.to(DEV)].cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all()
    bad = np.abs(got - yr) > 1e-3 * br
    assert not bad.any(), (np.argwhere(bad)[:5], got[bad][:5], yr[bad][:5])


# ---------------------------------------------------------------------------
# FP8 block-128 source (E4M3 + weight_scale_inv per 128 x 128 block) -> any
# target; FP8_ROW is the block -> row re-encode
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("fmt", list(FMTS))
@pytest.mark.parametrize("shape", [(200, 320), (384, 1024)])
def test_pack_from_fp8_block128_bit_exact(fmt, shape):
    rows, cols = shape
    codes, sc = synth.fp8_block128_source(rows, cols, seed=31 + rows)
    sc = sc.clone()
    sc[0, 0] = 0.0  # an all-zero block
    dec = oracle.decode_fp8_block128(codes.numpy(), sc.numpy(), rows, cols)
    ref = oracle.pack(FMTS[fmt], bf16_value(dec).astype(np.float32))
    pw = q.PackedWeights(FMTS[fmt], rows, cols, device=DEV)
    q.qlin_pack_weights(q.SRC_FP8_BLOCK128, codes.to(DEV), pw, aux0=sc.to(DEV))
    torch.cuda.synchronize()
    assert_packed_equal(pw, ref)


def test_pack_from_fp8_block128_full_size_rows_bit_exact():
    """A 17408 x 5120 text projection re-encoded from block-128 to row FP8;
    sampled rows (every row band of 128, first and last) against the oracle."""
    rows, cols = 17408, 5120
    codes, sc = synth.fp8_block128_source(rows, cols, seed=synth.seed_for(2, 5), device=DEV)
    pw = q.PackedWeights(q.FP8_ROW, rows, cols, device=DEV)
    q.qlin_pack_weights(q.SRC_FP8_BLOCK128, codes, pw, aux0=sc)
    sel = torch.cat([torch.arange(0, rows, 131), torch.tensor([rows - 1])])
    bands = (sel // 128).unique()
    sc_sub = sc.cpu().numpy()
    dec = np.concatenate([oracle.decode_fp8_block128(codes[int(r)].cpu().numpy()[None, :],
                                                     sc_sub[int(r) // 128][None, :], 1, cols) for r in sel])
    ref = oracle.pack(q.FP8_ROW, bf16_value(dec).astype(np.float32))
    torch.cuda.synchronize()
    got = gpu_packed_to_numpy(pw)
    assert np.array_equal(got["codes"][sel.numpy()], ref["codes"])
    assert np.array_equal(got["scales"][sel.numpy()], ref["scales"])
    assert len(bands) > 100
