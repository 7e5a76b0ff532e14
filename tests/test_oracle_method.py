"""Pins for the oracle's method functions: hand-worked examples, closed forms,
library routines (numpy integer / float64 matmul, numpy FP32 arithmetic),
invariants the pages state, and brute force on tiny shapes."""
import numpy as np
import pytest
import torch

import synth

Q4, Q5, Q8, FP8, BF16, Q3, Q6 = 0, 1, 2, 3, 4, 5, 6
QMAX = {Q4: 7, Q5: 15, Q8: 127, Q3: 3, Q6: 31}
GS = {Q4: 64, Q5: 64, Q8: 32, Q3: 64, Q6: 64}


def _bf16(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _bf16_val(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32)


def _f16_val(bits):
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


# ---- hand-worked examples (tests/golden/hand_examples.json) ------------------
def test_golden_mxfp8(orc, golden):
    for ex in golden["mxfp8"]:
        byte, b = int(ex["byte"], 16), ex["b"]
        words = np.array([[byte]], np.uint32).repeat(8, 1)  # 32 columns, element 0 = byte
        words[0, 0] = byte
        scales = np.full((1, 1), b, np.uint8)
        out = orc.decode_mxfp8(words, scales, 1, 32)
        assert out[0, 0] == int(ex["bf16"], 16), ex


def test_golden_fp8_row(orc, golden):
    ex = golden["fp8_row"]
    pw = orc.pack(FP8, np.array([ex["w"]], np.float32))
    assert pw["scales"][0] == int(ex["scale_bf16"], 16)
    assert [int(c) for c in pw["codes"][0]] == [int(c, 16) for c in ex["codes"]]


def test_golden_q4_group(orc, golden):
    ex = golden["q4_group"]
    w = np.array([[np.float32((i - 32) * 0.01) for i in range(64)]], np.float32)
    pw = orc.pack(Q4, w)
    assert pw["scales"][0, 0] == int(ex["scale_f16"], 16)
    s = _f16_val(pw["scales"][0, 0])
    wdq = orc.dequant(pw)[0]
    for i, q in ex["codes_at"].items():
        assert wdq[int(i)] == q * s


def test_golden_act_group(orc, golden):
    ex = golden["act_group"]
    x = np.zeros((1, 64), np.float32)
    x[0, :3] = ex["x_head"]
    qa, as_ = orc.quantize_act(_bf16(x))
    assert as_[0, 0] == np.float32(ex["scale_f32"])
    assert list(qa[0, :3]) == ex["codes_head"]
    assert not qa[0, 3:].any()


def _tie_row(ex, width):
    v = np.full((1, width), ex["rest"], np.float32)
    v[0, :len(ex["w_head"] if "w_head" in ex else ex["x_head"])] = ex["w_head"] if "w_head" in ex else ex["x_head"]
    return v


@pytest.mark.parametrize("name,fmt", [("q4_group", Q4), ("q5_group", Q5), ("q8_group", Q8),
                                      ("q3_group", Q3), ("q6_group", Q6)])
def test_golden_pack_ties_round_half_even(orc, golden, name, fmt):
    """w/s exactly on k + 1/2: the codes are the even neighbours (a
    round-half-away-from-zero oracle fails here)."""
    ex = golden["ties"][name]
    pw = orc.pack(fmt, _tie_row(ex, GS[fmt]))
    assert pw["scales"][0, 0] == int(ex["scale_f16"], 16)
    s = _f16_val(pw["scales"][0, 0])
    wdq = orc.dequant(pw)[0]
    for i, q in enumerate(ex["codes_head"]):
        assert wdq[i] == q * s, (i, wdq[i] / s, q)
    assert not wdq[len(ex["codes_head"]):].any()


@pytest.mark.parametrize("name", ["act_group_unit_scale", "act_group_half_scale"])
def test_golden_act_ties_round_half_even(orc, golden, name):
    ex = golden["ties"][name]
    qa, as_ = orc.quantize_act(_bf16(_tie_row(ex, 64)))
    assert as_[0, 0] == np.float32(ex["scale_f32"])
    assert list(qa[0, :len(ex["codes_head"])]) == ex["codes_head"]
    assert not qa[0, len(ex["codes_head"]):].any()


def test_page_constants_used(orc, golden):
    c = golden["constants"]
    x = np.zeros((1, c["act_group"]["value"] * 2), np.float32)
    x[0, 5] = 3.0
    x[0, 64 + 7] = -0.5
    qa, as_ = orc.quantize_act(_bf16(x))
    assert as_.shape == (1, 2)
    assert as_[0, 0] == np.float32(3.0) / np.float32(c["act_divisor"]["value"])
    assert qa[0, 5] == c["act_divisor"]["value"] and qa[0, 64 + 7] == -c["act_divisor"]["value"]


# ---- layouts: the documented bit positions ----------------------------------
def _word(plane, r, i):
    return int.from_bytes(plane[r, 4 * i:4 * i + 4].tobytes(), "little")


def _layout_code(fmt, codes, hib, r, e):
    """Read element e of row r straight from the documented layout."""
    if fmt == Q3:
        i = e % 16
        u = (_word(codes, r, e // 16) >> (16 * (i % 2) + 2 * (i // 2))) & 0x3
    else:
        i = e % 8
        u = (_word(codes, r, e // 8) >> (16 * (i % 2) + 4 * (i // 2))) & 0xF
    ee = e % 32
    hbit = 16 * (ee % 2) + 4 * (ee // 8) + (ee % 8) // 2
    if fmt == Q5:
        return (u | (((_word(hib, r, e // 32) >> hbit) & 1) << 4)) - 16
    if fmt == Q3:
        return (u | (((_word(hib, r, e // 32) >> hbit) & 1) << 2)) - 4
    if fmt == Q6:
        i = e % 16
        return (u | (((_word(hib, r, e // 16) >> (16 * (i % 2) + 2 * (i // 2))) & 0x3) << 4)) - 32
    return u - 8


@pytest.mark.parametrize("name,fmt", [("q3_group", Q3), ("q6_group", Q6)])
def test_golden_packed_words(orc, golden, name, fmt):
    """The packed planes of the hand-derived tie groups, word for word."""
    pw = orc.pack(fmt, _tie_row(golden["ties"][name], 64))
    lay = golden["layouts"][name]
    for key in ("codes", "hibits"):
        plane = pw[key]
        want = [int(h, 16) for h in lay[key + "_words"]]
        assert plane.shape[1] == 4 * len(want), key
        assert [_word(plane, 0, i) for i in range(len(want))] == want, key


def _exact_codes_matrix(fmt, n, k, rng, scale_pow2=True):
    """W whose quantization is known exactly: every group holds +-Qmax*s once,
    s a power of two -> codes equal the chosen integers."""
    qmax, gs = QMAX[fmt], GS[fmt]
    q = rng.integers(-qmax, qmax + 1, (n, k))
    q[:, ::gs] = qmax * rng.choice([-1, 1], (n, k // gs))
    sexp = rng.integers(-12, -2, (n, k // gs))
    s = np.ldexp(1.0, sexp)
    w = (q * np.repeat(s, gs, axis=1)).astype(np.float32)
    return q, s, w


@pytest.mark.parametrize("fmt", [Q4, Q5, Q8, Q3, Q6])
def test_pack_exact_codes_and_layout(orc, fmt):
    rng = np.random.default_rng(10 + fmt)
    n, k = 5, 192
    q, s, w = _exact_codes_matrix(fmt, n, k, rng)
    pw = orc.pack(fmt, w)
    assert np.array_equal(_f16_val(pw["scales"]), s)
    if fmt == Q8:
        assert np.array_equal(pw["codes"].astype(np.int64), q)
    else:
        for r in range(n):
            for e in range(k):
                assert _layout_code(fmt, pw["codes"], pw["hibits"], r, e) == q[r, e]
    assert np.array_equal(orc.dequant(pw), w.astype(np.float64))


@pytest.mark.parametrize("fmt", [Q4, Q5, Q8, Q3, Q6])
def test_pack_half_step_bound_and_idempotence(orc, fmt):
    w = synth.weights_f32(24, 512, seed=77 + fmt).numpy()
    pw = orc.pack(fmt, w)
    qmax, gs = QMAX[fmt], GS[fmt]
    s = np.repeat(_f16_val(pw["scales"]), gs, axis=1)
    wdq = orc.dequant(pw)
    q = np.where(s > 0, wdq / np.where(s > 0, s, 1), 0)
    assert np.all(np.abs(q) <= qmax) and np.array_equal(q, np.round(q))
    # quantize -> dequantize stays within half a scale step, plus the rounding of
    # the FP32 quotient w/s (half an ulp at magnitude <= 128: s * 2^-17)
    assert np.all(np.abs(wdq - w) <= s * (0.5 + 2.0 ** -17))
    # the group's amax element lands on +-Qmax
    wa = np.abs(w).reshape(24, -1, gs)
    idx = wa.argmax(axis=2)
    qg = np.abs(q.reshape(24, -1, gs))
    assert np.all(np.take_along_axis(qg, idx[..., None], 2) == qmax)
    pw2 = orc.pack(fmt, wdq.astype(np.float32))
    for key in ("codes", "hibits", "scales"):
        if pw[key] is not None:
            assert np.array_equal(pw[key], pw2[key]), key


def test_pack_zero_group(orc):
    w = np.zeros((2, 128), np.float32)
    w[1, 64:] = 0.25
    for fmt in (Q4, Q5, Q8, Q3, Q6):
        pw = orc.pack(fmt, w)
        assert np.all(orc.dequant(pw)[0] == 0)
        assert pw["scales"][0, 0] == 0
    pw = orc.pack(FP8, w)
    assert pw["scales"][0] == 0 and not pw["codes"][0].any()


def _e4m3_half_ulp(m):
    e = np.floor(np.log2(np.maximum(m, 2.0 ** -6)))
    return 2.0 ** (e - 3) / 2


def test_fp8_row_bound_idempotence_noise(orc):
    """The page: every element within the E4M3 half-ulp at its own magnitude;
    a re-encode is bit-exact; relative L2 at the E4M3 noise floor (~2-3%)."""
    w = synth.weights_f32(64, 1024, seed=91).numpy()
    pw = orc.pack(FP8, w)
    sc = _bf16_val(pw["scales"]).astype(np.float64)[:, None]
    wdq = orc.dequant(pw)
    ratio = np.abs(w.astype(np.float64)) / sc
    bound = _e4m3_half_ulp(ratio) * sc * (1 + 2.0 ** -20)
    assert np.all(np.abs(wdq - w) <= bound)
    assert np.all(np.abs(torch.from_numpy(pw["codes"]).view(torch.float8_e4m3fn).float().numpy()) <= 448)
    pw2 = orc.pack(FP8, wdq.astype(np.float32))
    assert np.array_equal(pw["codes"], pw2["codes"]) and np.array_equal(pw["scales"], pw2["scales"])
    rel = np.linalg.norm(wdq - w, axis=1) / np.linalg.norm(w, axis=1)
    assert 0.015 < rel.mean() < 0.035


def test_mlx_affine_hand_and_exact(orc):
    rows, cols = 2, 256
    q = np.zeros((rows, cols), np.uint8)
    sc = np.ones((rows, 2), np.float16)
    bi = np.zeros((rows, 2), np.float16)
    q[0, :4] = [0, 1, 255, 128]
    bi[0, 0] = np.float16(-0.5)
    out = orc.decode_mlx_affine(q, sc.view(np.uint16), bi.view(np.uint16), rows, cols)
    assert list(out[0, :4]) == list(_bf16([-0.5, 0.5, 254.5, 127.5]))
    # random: fma(q, s, b) equals the exact double product-sum rounded once to FP32
    src = synth.mlx_affine_source(8, 512, seed=5)
    qq, s16, b16 = (t.numpy() for t in src)
    out = orc.decode_mlx_affine(qq, s16.view(np.uint16), b16.view(np.uint16), 8, 512)
    exact = qq.astype(np.float64) * np.repeat(s16.astype(np.float64), 128, 1) + np.repeat(b16.astype(np.float64), 128, 1)
    ref = _bf16(exact.astype(np.float32))
    assert np.array_equal(out, ref)


def test_mxfp8_synthetic_matches_closed_form(orc):
    words, scales = synth.mxfp8_source(16, 256, seed=6)
    words, scales = words.numpy(), scales.numpy()
    out = orc.decode_mxfp8(words, scales, 16, 256)
    codes = torch.from_numpy(words.view(np.uint8).reshape(16, 256).copy()).view(torch.float8_e4m3fn)
    v = codes.to(torch.float64) * torch.from_numpy(2.0 ** (np.repeat(scales, 32, 1).astype(np.float64) - 127))
    ref = v.to(torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(out, ref)


# ---- GEMV ---------------------------------------------------------------------
@pytest.mark.parametrize("fmt", [Q4, Q5, Q8, Q3, Q6])
def test_gemv_unit_scales_is_integer_matmul(orc, fmt):
    rng = np.random.default_rng(20 + fmt)
    n, k, t = 7, 256, 3
    qmax, gs = QMAX[fmt], GS[fmt]
    q = rng.integers(-qmax, qmax + 1, (n, k))
    q[:, ::gs] = qmax
    w = q.astype(np.float32)  # unit scales
    pw = orc.pack(fmt, w)
    assert np.all(_f16_val(pw["scales"]) == 1.0)
    xi = rng.integers(-9, 10, (t, k))
    y, b = orc.gemv(pw, _bf16(xi.astype(np.float32)))
    ref = xi.astype(np.int64) @ q.astype(np.int64).T
    assert np.array_equal(y, ref.astype(np.float64))
    assert np.array_equal(b, (np.abs(xi) @ np.abs(q).T).astype(np.float64))


def test_gemv_fp8_and_bf16_against_float64_matmul(orc):
    w = synth.weights_f32(33, 320, seed=8).numpy()
    x = synth.activations_bf16(5, 320, seed=9).view(torch.int16).numpy().view(np.uint16)
    xv = _bf16_val(x).astype(np.float64)
    for fmt in (FP8, BF16, Q4, Q8):
        pw = orc.pack(fmt, w)
        y, b = orc.gemv(pw, x)
        wdq = orc.dequant(pw)
        ref = xv @ wdq.T
        assert np.all(np.abs(y - ref) <= 1e-12 * (np.abs(xv) @ np.abs(wdq).T))
        assert np.allclose(b, np.abs(xv) @ np.abs(wdq).T, rtol=1e-12)
    # FP8 row scale factors out of the row: codes on the grid with unit scale
    pw = orc.pack(FP8, w)
    c = torch.from_numpy(pw["codes"]).view(torch.float8_e4m3fn).double().numpy()
    sc = _bf16_val(pw["scales"]).astype(np.float64)
    y, _ = orc.gemv(pw, x)
    assert np.allclose(y, (xv @ c.T) * sc[None, :], rtol=1e-12, atol=0)


def test_gemv_threads_identical(orc):
    w = synth.weights_f32(50, 256, seed=3).numpy()
    x = synth.activations_bf16(2, 256, seed=4).view(torch.int16).numpy().view(np.uint16)
    pw = orc.pack(Q5, w)
    y1, _ = orc.gemv(pw, x, nthreads=1)
    y4, _ = orc.gemv(pw, x, nthreads=4)
    assert np.array_equal(y1, y4)


# ---- activation quantization and the int8 route -------------------------------
def test_quantize_act_invariants(orc):
    x = synth.activations_bf16(9, 640, seed=12)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    xv = x.float().numpy()
    xv[3, 64:128] = 0.0
    xb = _bf16(xv)
    qa, as_ = orc.quantize_act(xb)
    a = np.abs(xv).reshape(9, 10, 64).max(axis=2)
    assert np.array_equal(as_, a / np.float32(127))  # numpy FP32 division
    assert as_[3, 1] == 0 and not qa[3, 64:128].any()
    s = np.repeat(as_, 64, 1).astype(np.float64)
    assert np.all(np.abs(qa) <= 127)
    # half a step, plus the rounding of the FP32 quotient x/as (ties can land
    # on the far side by up to half an ulp of a magnitude <= 127)
    assert np.all(np.abs(qa * s - xv) <= s * (0.5 + 2.0 ** -17))
    idx = np.abs(xv).reshape(9, 10, 64).argmax(axis=2)
    qg = np.abs(qa.reshape(9, 10, 64))
    top = np.take_along_axis(qg, idx[..., None], 2)[..., 0]
    assert np.all(top[as_ > 0] == 127)


@pytest.mark.parametrize("fmt", [Q4, Q5, Q3, Q6])
def test_group_sums_bruteforce(orc, fmt):
    rng = np.random.default_rng(30 + fmt)
    for k in (64, 128, 192):
        n, t = 7, 5
        q, s, w = _exact_codes_matrix(fmt, n, k, rng)
        pw = orc.pack(fmt, w)
        qa = rng.integers(-127, 128, (t, k)).astype(np.int8)
        S = orc.group_sums(pw, qa)
        for g in range(k // 64):
            ref = qa[:, g * 64:(g + 1) * 64].astype(np.int64) @ q[:, g * 64:(g + 1) * 64].T
            assert np.array_equal(S[:, :, g], ref)


@pytest.mark.parametrize("fmt", [Q4, Q5, Q3, Q6])
def test_group_sums_extremes(orc, fmt):
    qmax = QMAX[fmt]
    for sign_w, sign_a in ((1, 1), (-1, 1), (1, -1)):
        w = np.full((2, 64), sign_w * qmax * 0.125, np.float32)
        pw = orc.pack(fmt, w)
        qa = np.full((1, 64), sign_a * 127, np.int8)
        S = orc.group_sums(pw, qa)
        assert np.all(S == sign_w * sign_a * 64 * qmax * 127)


@pytest.mark.parametrize("fmt", [Q4, Q5, Q3, Q6])
def test_gemm_a8_unit_scales_is_integer_matmul(orc, fmt):
    rng = np.random.default_rng(40 + fmt)
    n, k, t = 6, 192, 4
    qmax = QMAX[fmt]
    q = rng.integers(-qmax, qmax + 1, (n, k))
    q[:, ::64] = qmax
    pw = orc.pack(fmt, q.astype(np.float32))
    qa = rng.integers(-127, 128, (t, k)).astype(np.int8)
    as_ = np.ones((t, k // 64), np.float32)
    y, b = orc.gemm_a8(pw, qa, as_)
    assert np.array_equal(y, (qa.astype(np.int64) @ q.T).astype(np.float64))
    assert np.array_equal(b, (np.abs(qa.astype(np.int64)) @ np.abs(q).T).astype(np.float64))


def test_gemm_a8_scaled_matches_group_sums(orc):
    """With real scales: y = sum_g FP32(ws*as) * S_g (numpy FP32 product)."""
    w = synth.weights_f32(12, 320, seed=50).numpy()
    x = synth.activations_bf16(6, 320, seed=51).view(torch.int16).numpy().view(np.uint16)
    for fmt in (Q4, Q5, Q3, Q6):
        pw = orc.pack(fmt, w)
        qa, as_ = orc.quantize_act(x)
        S = orc.group_sums(pw, qa).astype(np.float64)
        ws = pw["scales"].view(np.float16).astype(np.float32)
        c = (ws[None, :, :] * as_[:, None, :]).astype(np.float64)  # FP32 products
        ref = (c * S).sum(axis=2)
        y, _ = orc.gemm_a8(pw, qa, as_)
        assert np.allclose(y, ref, rtol=1e-13, atol=1e-30)
        # and the int8 route approximates the BF16 route within the quantization noise
        yb, bb = orc.gemv(pw, x)
        assert np.all(np.abs(y - yb) <= 0.05 * bb)


# ---- FP8 block-128 source (E4M3 codes + weight_scale_inv per 128x128 block) ----
def _e4m3_vals(codes):
    """E4M3 code -> float64 through torch's own float8_e4m3fn conversion."""
    return torch.from_numpy(np.asarray(codes, np.uint8)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def _bf16_bits_of_f32(v32):
    return torch.from_numpy(np.asarray(v32, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_golden_fp8_block128(orc, golden):
    ex = golden["fp8_block128"]
    codes = np.full((2, 128), int(ex["rest_code"], 16), np.uint8)
    codes[0, :4] = [int(c, 16) for c in ex["codes_head"]]
    out = orc.decode_fp8_block128(codes, np.array([[ex["block_scale"]]], np.float32), 2, 128)
    assert [int(v) for v in out[0, :4]] == [int(b, 16) for b in ex["bf16_head"]]
    assert not out[0, 4:].any() and not out[1].any()
    pw = orc.pack(FP8, _bf16_val(out[:1]))
    assert pw["scales"][0] == int(ex["row_scale_bf16"], 16)
    assert [int(c) for c in pw["codes"][0, :4]] == [int(c, 16) for c in ex["codes_head"]]


def _block_source(rng, rows, cols, bf16_scales):
    codes = rng.integers(0, 256, (rows, cols)).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x3C  # no NaN codes
    gr, gc = (rows + 127) // 128, (cols + 127) // 128
    sc = np.exp2(rng.uniform(-14, -4, (gr, gc))).astype(np.float32) * rng.uniform(1, 2, (gr, gc)).astype(np.float32)
    if bf16_scales:
        sc = _bf16_val(_bf16_bits_of_f32(sc)).astype(np.float32)
    return codes, sc


def test_fp8_block128_exact_for_bf16_scales(orc):
    """A BF16 block scale times an E4M3 value has at most 12 significant bits:
    the FP32 product is exact (the page's "fits exactly") and the decode is
    that exact value rounded once to BF16.  Ragged grid: 200 x 300."""
    rng = np.random.default_rng(21)
    rows, cols = 200, 300
    codes, sc = _block_source(rng, rows, cols, True)
    full = np.repeat(np.repeat(sc.astype(np.float64), 128, 0), 128, 1)[:rows, :cols]
    exact = _e4m3_vals(codes) * full
    assert np.array_equal(exact.astype(np.float32).astype(np.float64), exact)  # exact in FP32
    out = orc.decode_fp8_block128(codes, sc, rows, cols)
    assert np.array_equal(out, _bf16_bits_of_f32(exact.astype(np.float32)))


def test_fp8_block128_general_fp32_scales(orc):
    """Scales with a full FP32 mantissa: one IEEE single product (numpy float32)
    then BF16 rounding (torch)."""
    rng = np.random.default_rng(22)
    rows, cols = 131, 256
    codes, sc = _block_source(rng, rows, cols, False)
    full = np.repeat(np.repeat(sc, 128, 0), 128, 1)[:rows, :cols]
    prod = _e4m3_vals(codes).astype(np.float32) * full  # IEEE single multiply
    out = orc.decode_fp8_block128(codes, sc, rows, cols)
    assert np.array_equal(out, _bf16_bits_of_f32(prod))


def test_fp8_block128_to_row_within_page_bound(orc):
    """The page's verification bound for the block -> row re-encode: every
    element stays within the E4M3 half-ulp of its own magnitude at the stored
    row scale plus the source value's own BF16 rounding."""
    rng = np.random.default_rng(23)
    rows, cols = 256, 384
    codes, sc = _block_source(rng, rows, cols, False)
    full = np.repeat(np.repeat(sc.astype(np.float64), 128, 0), 128, 1)[:rows, :cols]
    src = (_e4m3_vals(codes).astype(np.float32) * full.astype(np.float32)).astype(np.float64)
    dec = orc.decode_fp8_block128(codes, sc, rows, cols)
    pw = orc.pack(FP8, _bf16_val(dec))
    rs = _bf16_val(pw["scales"]).astype(np.float64)[:, None]
    got = orc.dequant(pw)
    mag = np.abs(src) / rs
    e = np.floor(np.log2(np.maximum(mag, 2.0 ** -6)))
    half_ulp = np.exp2(np.maximum(e, -6) - 3) / 2 * rs  # E4M3: 3 mantissa bits, min normal 2^-6
    bf16_err = np.abs(_bf16_val(dec).astype(np.float64) - src)
    assert np.all(np.abs(got - src) <= half_ulp + bf16_err + 1e-300)


def test_fp8_block128_row_reencode_is_identity_when_scales_agree(orc):
    """A row whose codes all share one BF16 block scale and which holds a
    +-448 code re-encodes to the very same codes, with the block scale as its
    row scale (the page's bit-exact re-encode of the converter's arithmetic)."""
    rng = np.random.default_rng(24)
    rows, cols = 64, 128
    codes, _ = _block_source(rng, rows, cols, True)
    codes[:, 5] = np.where(rng.integers(0, 2, rows) > 0, 0x7E, 0xFE)
    sc = np.array([[2.0 ** -7 * 1.5]], np.float32)
    dec = orc.decode_fp8_block128(codes, sc, rows, cols)
    pw = orc.pack(FP8, _bf16_val(dec))
    assert np.all(_bf16_val(pw["scales"]) == sc[0, 0])
    ref = codes.copy()
    ref[(ref & 0x7F) == 0] = 0x00  # -0 and +0 both encode +0 after the round trip
    got = pw["codes"].copy()
    got[(got & 0x7F) == 0] = 0x00
    assert np.array_equal(got, ref)


# ---- FP8-activation route ------------------------------------------------------
def test_golden_fp8_act_token(orc, golden):
    ex = golden["fp8_act_token"]
    x = np.zeros((1, 64), np.float32)
    x[0, :len(ex["x_head"])] = ex["x_head"]
    xq, xs = orc.quantize_act_fp8(_bf16(x))
    assert xs[0] == np.float32(ex["scale_f32"])
    assert [int(c) for c in xq[0, :len(ex["codes_head"])]] == [int(c, 16) for c in ex["codes_head"]]
    assert not xq[0, len(ex["codes_head"]):].any()


def test_fp8_act_invariants(orc):
    """amax element -> +-448 code; zero token -> scale 0, codes 0; every element
    within half an E4M3 step of its own magnitude (scaled back by xs)."""
    rng = np.random.default_rng(31)
    t, k = 9, 1536
    x = rng.standard_normal((t, k)).astype(np.float32) * np.exp2(rng.integers(-20, 20, (t, 1)))
    x[3] = 0.0
    xb = _bf16(x)
    xf = _bf16_val(xb).astype(np.float64)
    xq, xs = orc.quantize_act_fp8(xb)
    assert xs[3] == 0 and not xq[3].any()
    vals = _e4m3_vals(xq)
    for tt in range(t):
        if tt == 3:
            continue
        assert xs[tt] == np.float32(np.float32(np.abs(xf[tt]).max()) / np.float32(448.0))
        i = int(np.argmax(np.abs(xf[tt])))
        assert abs(vals[tt, i]) == 448.0
        mag = np.abs(xf[tt]) / xs[tt]
        e = np.floor(np.log2(np.maximum(mag, 2.0 ** -6)))
        half = np.exp2(np.maximum(e, -6) - 3) / 2
        assert np.all(np.abs(vals[tt] - xf[tt] / xs[tt]) <= half * (1 + 2.0 ** -20) + 2.0 ** -30)


def test_gemm_fp8_reduces_to_integer_matmul(orc):
    """Integer-valued E4M3 codes (|v| <= 16 are all exact) with unit scales:
    the route is an exact integer matrix product."""
    rng = np.random.default_rng(32)
    n, k, t = 19, 320, 7
    wi = rng.integers(-16, 17, (n, k))
    xi = rng.integers(-16, 17, (t, k))
    wi[:, 0] = 448 // 28 * 0  # keep the row max well inside
    enc = lambda a: torch.from_numpy(a.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    pw = {"fmt": FP8, "n": n, "k": k, "codes": enc(wi), "hibits": None,
          "scales": np.full((n,), 0x3F80, np.uint16)}
    y, b = orc.gemm_fp8(pw, enc(xi), np.ones((t,), np.float32))
    exact = (xi.astype(np.int64) @ wi.T.astype(np.int64)).astype(np.float64)
    assert np.array_equal(y, exact)
    assert np.array_equal(b, (np.abs(xi) @ np.abs(wi).T).astype(np.float64))
