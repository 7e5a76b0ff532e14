"""GPU parity of the FP8-activation route (row-FP8 weights x per-token E4M3
activations on the tensor cores) against the CPU oracle.

The quantizer is bit-exact (codes and FP32 scales).  The product of E4M3
values is exact, so the GEMM differs from the oracle's exact sum only by FP32
accumulation: about K/32 additions on the tensor core, each rounding at most
2^-24 of a partial sum bounded by sum|w||xq|, plus the rounding of the final
scale product -- K = 17408 gives 545 * 2^-24 < 3.3e-5; the stated bound is
|y - y_ref| <= 4e-5 * |ws xs| sum_k |w||xq| for any K up to 20480 (FP32
output), plus half a BF16 ulp of |y_ref| for a BF16 output."""
import numpy as np
import pytest
import torch

import oracle
import quantized_weight_linear_qlin_b200 as q
import synth

pytestmark = pytest.mark.gpu

DEV = "cuda"
TOL = 4e-5


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from quantized_weight_linear_qlin_b200 import _build
    _build.build()
    q.lib()


def bits16(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def quantize_gpu(x):
    t, k = x.shape
    xq = torch.empty(t, k, dtype=torch.uint8, device=DEV)
    xs = torch.empty(t, dtype=torch.float32, device=DEV)
    q.qlin_quantize_act_fp8(x.to(DEV), xq, xs)
    torch.cuda.synchronize()
    return xq, xs


def assert_quant_equal(x, xq, xs):
    qr, sr = oracle.quantize_act_fp8(bits16(x))
    assert np.array_equal(xs.cpu().numpy().view(np.uint32), sr.view(np.uint32))
    got = xq.cpu().numpy()
    bad = np.argwhere(got != qr)
    assert bad.size == 0, (bad[:5], got[tuple(bad[0])], qr[tuple(bad[0])])
    return qr, sr


# ---------------------------------------------------------------------------
# quantizer: bit-exact
# ---------------------------------------------------------------------------
def test_quantize_act_fp8_golden_token(golden):
    g = golden["fp8_act_token"]
    k = 64
    x = torch.zeros(2, k, dtype=torch.float32)
    x[0, :len(g["x_head"])] = torch.tensor(g["x_head"], dtype=torch.float32)
    x = x.to(torch.bfloat16)
    xq, xs = quantize_gpu(x)
    assert xs[0].item() == g["scale_f32"] and xs[1].item() == 0.0
    codes = [int(c, 16) for c in g["codes_head"]]
    assert xq[0, :len(codes)].cpu().tolist() == codes
    assert not xq[0, len(codes):].any() and not xq[1].any()


@pytest.mark.parametrize("shape", [(1, 16), (37, 320), (130, 5120), (5, 17408)])
def test_quantize_act_fp8_bit_exact(shape):
    t, k = shape
    x = synth.activations_bf16(t, k, seed=700 + t + k).float()
    x[0] = 0.0                              # zero token: scale 0, all codes 0
    if t > 2:
        x[1, :5] = 3.0e38                   # huge values
        x[2] = 1e-38                        # subnormal scale
    x = x.to(torch.bfloat16)
    xq, xs = quantize_gpu(x)
    assert_quant_equal(x, xq, xs)


def test_quantize_act_fp8_bit_exact_wide_ranges():
    """8 M values, each token scaled by its own power of two over the whole
    BF16 exponent range (some tokens subnormal)."""
    t, k = 2048, 4096
    g = torch.Generator().manual_seed(4321)
    x = torch.randn(t, k, generator=g)
    e = torch.randint(-140, 120, (t, 1), generator=g).float()
    x = (x * torch.exp2(e)).to(torch.bfloat16)
    xq, xs = quantize_gpu(x)
    assert_quant_equal(x, xq, xs)


# ---------------------------------------------------------------------------
# GEMM: within TOL of the oracle's exact sum over the same codes
# ---------------------------------------------------------------------------
def pack_fp8(w):
    pw = q.PackedWeights(q.FP8_ROW, w.shape[0], w.shape[1], device=DEV)
    q.qlin_pack_weights(q.SRC_F32, w.to(DEV), pw)
    return pw


def run_gemm_fp8(pw, x, fused=True, y_dtype=q.OUT_F32, ws=None):
    t, k = x.shape
    xd = x.to(DEV)
    y = torch.full((t, pw.n), float("nan"), device=DEV,
                   dtype=torch.float32 if y_dtype == q.OUT_F32 else torch.bfloat16)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    if fused:
        if ws is None:
            ws = q.Workspace(DEV)
        ws.ensure(q.qlin_gemm_fp8_workspace_bytes(t, k))
        q.qlin_gemm_fp8(pw, y, x=xd, y_dtype=y_dtype, workspace=ws, dev_status=status)
    else:
        xq = torch.empty(t, k, dtype=torch.uint8, device=DEV)
        xs = torch.empty(t, dtype=torch.float32, device=DEV)
        q.qlin_quantize_act_fp8(xd, xq, xs)
        q.qlin_gemm_fp8(pw, y, xq=xq, xs=xs, y_dtype=y_dtype, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    return y


def assert_close(got, yr, br, bf16_out):
    got = got.float().cpu().numpy().astype(np.float64) if isinstance(got, torch.Tensor) else got
    tol = TOL * br
    if bf16_out:
        tol = tol + np.abs(yr) * 2.0 ** -8
    bad = ~(np.abs(got - yr) <= tol)     # NaN (an unwritten element) fails too
    assert not bad.any(), (np.argwhere(bad)[:5], got[bad][:5], yr[bad][:5])


@pytest.mark.parametrize("n,k,t", [(128, 256, 1), (200, 640, 17), (256, 512, 130), (384, 1152, 257),
                                   (129, 1024, 300), (1000, 5120, 33), (300, 17408, 5)])
@pytest.mark.parametrize("fused", [True, False])
def test_gemm_fp8_parity(n, k, t, fused):
    w = synth.weights_f32(n, k, seed=800 + n + k)
    x = synth.activations_bf16(t, k, seed=900 + t)
    ref = oracle.pack(q.FP8_ROW, w.numpy())
    pw = pack_fp8(w)
    y = run_gemm_fp8(pw, x, fused=fused)
    xq, xs = oracle.quantize_act_fp8(bits16(x))
    yr, br = oracle.gemm_fp8(ref, xq, xs, nthreads=8)
    assert_close(y, yr, br, False)


@pytest.mark.parametrize("t", [1, 16, 64, 200])
def test_gemm_fp8_bf16_output_every_tile_width(t):
    n, k = 640, 2048
    w = synth.weights_f32(n, k, seed=31 + t)
    x = synth.activations_bf16(t, k, seed=32 + t)
    ref = oracle.pack(q.FP8_ROW, w.numpy())
    y = run_gemm_fp8(pack_fp8(w), x, fused=True, y_dtype=q.OUT_BF16)
    xq, xs = oracle.quantize_act_fp8(bits16(x))
    yr, br = oracle.gemm_fp8(ref, xq, xs, nthreads=8)
    assert_close(y, yr, br, True)


def test_gemm_fp8_fused_quantizer_matches_oracle():
    """The fused call's activation codes and scales (left in the workspace) are
    the oracle's, bit for bit."""
    n, k, t = 256, 1536, 77
    w = synth.weights_f32(n, k, seed=5)
    x = synth.activations_bf16(t, k, seed=6)
    ws = q.Workspace(DEV)
    run_gemm_fp8(pack_fp8(w), x, fused=True, ws=ws)
    buf = ws.buffer.cpu()
    off = (t * k + 255) // 256 * 256
    xq = buf[:t * k].view(t, k)
    xs = buf[off:off + 4 * t].view(torch.float32)
    assert_quant_equal(x, xq, xs)


def test_gemm_fp8_zero_tokens_and_saturation():
    """A zero token gives zero outputs; a token whose values saturate the
    E4M3 range and extreme weight rows stay within the bound."""
    n, k, t = 256, 1024, 40
    w = synth.weights_f32(n, k, seed=7)
    w[3] *= 1e4
    x = synth.activations_bf16(t, k, seed=8).float()
    x[0] = 0.0
    x[5] *= 1e30
    x = x.to(torch.bfloat16)
    ref = oracle.pack(q.FP8_ROW, w.numpy())
    y = run_gemm_fp8(pack_fp8(w), x, fused=True)
    assert not y[0].any()
    xq, xs = oracle.quantize_act_fp8(bits16(x))
    yr, br = oracle.gemm_fp8(ref, xq, xs, nthreads=8)
    assert_close(y, yr, br, False)


@pytest.mark.parametrize("name,n,k,t", [("head_decode", 152064, 5120, 1),
                                        ("head_verify", 152064, 5120, 33),
                                        ("q_prefill", 6144, 5120, 8192),
                                        ("down_prefill", 5120, 17408, 2048)])
def test_gemm_fp8_full_size_sampled(name, n, k, t):
    w = synth.weights_f32(n, k, seed=synth.seed_for(6, 0), device=DEV)
    x = synth.activations_bf16(t, k, seed=synth.seed_for(6, 1), device=DEV)
    pw = pack_fp8(w)
    y = run_gemm_fp8(pw, x, fused=True)
    g = torch.Generator().manual_seed(6)
    rows = torch.cat([torch.randperm(n, generator=g)[:30], torch.tensor([0, n - 1])])
    toks = torch.cat([torch.randperm(t, generator=g)[:min(t, 14)], torch.tensor([0, t - 1])]).unique()
    ref = oracle.pack(q.FP8_ROW, w[rows.to(DEV)].cpu().numpy())
    xq, xs = oracle.quantize_act_fp8(bits16(x[toks.to(DEV)]))
    yr, br = oracle.gemm_fp8(ref, xq, xs, nthreads=8)
    got = y[toks.to(DEV)][:, rows.to(DEV)]
    assert_close(got, yr, br, False)
