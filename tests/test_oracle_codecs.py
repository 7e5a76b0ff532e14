"""Pins for the oracle's number-format codecs: exhaustive decodes and RNE
encodes checked against numpy / torch conversions and closed forms."""
import math

import numpy as np
import pytest
import torch


def test_f16_decode_exhaustive(orc):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([orc.f16_value(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_f16_encode_rne_against_numpy(orc):
    rng = np.random.default_rng(1)
    vals = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.integers(-9, 6, 20000),
        # exact ties between neighbouring binary16 values, normal and subnormal
        (np.arange(1, 2048, dtype=np.float64) + 0.5) * 2.0 ** -24,
        (np.arange(1024, 2047, dtype=np.float64) + 0.5) * 2.0 ** -10,
        np.array([65504.0, 65519.99, 65520.0, 1e6, 2.0 ** -25, 2.0 ** -25 * 1.0000001, 0.0, -0.0]),
    ])
    vals = np.concatenate([vals, -vals])
    with np.errstate(over="ignore"):
        ref = vals.astype(np.float16).view(np.uint16)
    got = np.array([orc.f16_rne(float(v)) for v in vals], np.uint16)
    assert np.array_equal(got, ref)


def test_bf16_decode_exhaustive(orc):
    bits = np.arange(65536, dtype=np.uint32)
    ref = (bits << 16).astype(np.uint32).view(np.float32).astype(np.float64)
    got = np.array([orc.bf16_value(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_bf16_encode_rne_against_torch(orc):
    rng = np.random.default_rng(2)
    f = np.concatenate([
        (rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000)).astype(np.float32),
        # ties: 8 significant bits + exactly one half
        ((np.arange(128, 256, dtype=np.float64) + 0.5) * 2.0 ** -3).astype(np.float32),
        np.array([3.3895313e38, 3.4e38, 1e-40, 0.0], np.float32),
    ])
    f = np.concatenate([f, -f])
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([orc.bf16_rne(float(v)) for v in f], np.uint16)
    assert np.array_equal(got, ref)


def _e4m3_closed_form(c):
    s = -1.0 if c & 0x80 else 1.0
    e = (c >> 3) & 0xF
    m = c & 7
    if e == 15 and m == 7:
        return math.nan
    if e == 0:
        return s * 2.0 ** -6 * (m / 8.0)
    return s * 2.0 ** (e - 7) * (1.0 + m / 8.0)


def test_e4m3_decode_exhaustive(orc):
    codes = np.arange(256, dtype=np.uint8)
    lib_ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        got = orc.e4m3_value(c)
        cf = _e4m3_closed_form(c)
        if math.isnan(cf):
            assert math.isnan(got) and math.isnan(lib_ref[c])
        else:
            assert got == cf == lib_ref[c], c
    assert orc.e4m3_value(0x7E) == 448.0


def test_e4m3_encode_rne_satfinite(orc):
    rng = np.random.default_rng(3)
    f = np.concatenate([
        (rng.standard_normal(20000) * 10.0 ** rng.integers(-4, 3, 20000)).astype(np.float32),
        # ties between neighbouring E4M3 values (normal and subnormal)
        np.array([_e4m3_closed_form(c) for c in range(1, 0x7E)], np.float64).astype(np.float32),
    ])
    grid = np.array([_e4m3_closed_form(c) for c in range(0, 0x7F)])
    mids = ((grid[:-1] + grid[1:]) / 2).astype(np.float32)
    f = np.concatenate([f, mids])
    f = f[np.abs(f) <= 448.0]
    f = np.concatenate([f, -f])
    ref = torch.from_numpy(f).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([orc.e4m3_rne_satfinite(float(v)) for v in f], np.uint8)
    assert np.array_equal(got, ref)
    # satfinite: everything beyond the largest finite value clamps to +-448
    for v in (449.0, 464.0, 470.0, 1e9, math.inf):
        assert orc.e4m3_rne_satfinite(v) == 0x7E
        assert orc.e4m3_rne_satfinite(-v) == 0xFE
    assert orc.e4m3_rne_satfinite(-0.0) == 0x80
    assert orc.e4m3_rne_satfinite(math.nan) & 0x7F == 0x7F


@pytest.mark.parametrize("b", [0, 1, 3, 64, 117, 127, 128, 200, 254])
def test_mxfp8_single_codes_closed_form(orc, b):
    """Every E4M3 code at block exponent b: exact product rounded once to BF16."""
    codes = np.arange(256, dtype=np.uint8)
    words = codes.view(np.uint32).reshape(1, 64)
    scales = np.full((1, 8), b, np.uint8)
    got = orc.decode_mxfp8(words, scales, 1, 256)[0]
    v = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64) * 2.0 ** (b - 127)
    # the product has <= 4 significant bits and exponent >= -136: exact in float32
    ref = v.to(torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    for c in range(256):
        if (c & 0x7F) == 0x7F:
            assert got[c] == (0x7FC0 | ((c & 0x80) << 8)), c
        else:
            assert got[c] == ref[c], (c, hex(got[c]), hex(ref[c]))
