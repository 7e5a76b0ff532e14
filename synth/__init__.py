"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module draws random numbers and nothing else: it holds none of the
quantized-linear arithmetic (no scales, no codes, no dot products).  Both the
CUDA path and the CPU oracle receive the very same bytes from it.

Distributions follow the workloads the pages describe for a 27B-class decoder
(hidden 5120, FFN 17408): weights ~N(0, 0.02) with 1% of the rows scaled by 8
(outlier rows); activations ~N(0, 1) in BF16 with 0.5% of the channels scaled
by 20 for every token (outlier channels); MXFP8 sources with E4M3 codes of
N(0, 1) and block exponents b uniform in [117, 127]; MLX affine int8 sources
with uniform uint8 codes; block-wise FP8 sources with E4M3 codes of N(0, 1)
and random power-of-two-ish block scales.  No dataset or checkpoint is involved.

Generation runs on the requested torch device with a seeded torch.Generator;
the same (seed, device type) always yields the same bytes.
"""
import torch

SEED_BASE = 0xC0FFEE00


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def seed_for(config: int, tensor_id: int) -> int:
    return SEED_BASE + 16 * int(config) + int(tensor_id)


def weights_f32(n: int, k: int, seed: int, device="cpu", std=0.02, outlier_frac=0.01,
                outlier_mul=8.0) -> torch.Tensor:
    """W[n][k] float32 ~N(0, std); round(outlier_frac*n) seeded rows scaled by outlier_mul."""
    g = _gen(seed, device)
    w = torch.randn((n, k), generator=g, device=device, dtype=torch.float32) * std
    n_out = int(round(outlier_frac * n))
    if n_out > 0:
        rows = torch.randperm(n, generator=g, device=device)[:n_out]
        w[rows] *= outlier_mul
    return w


def activations_bf16(t: int, k: int, seed: int, device="cpu", outlier_frac=0.005,
                     outlier_mul=20.0) -> torch.Tensor:
    """x[t][k] bfloat16 ~N(0, 1); round(outlier_frac*k) seeded channels scaled by outlier_mul."""
    g = _gen(seed, device)
    x = torch.randn((t, k), generator=g, device=device, dtype=torch.float32)
    n_out = int(round(outlier_frac * k))
    if n_out > 0:
        ch = torch.randperm(k, generator=g, device=device)[:n_out]
        x[:, ch] *= outlier_mul
    return x.to(torch.bfloat16)


def mxfp8_source(rows: int, cols: int, seed: int, device="cpu", b_lo=117, b_hi=127):
    """(words int32[rows][cols/4] holding 4 E4M3 bytes each, little-endian; scales uint8[rows][cols/32])."""
    g = _gen(seed, device)
    v = torch.randn((rows, cols), generator=g, device=device, dtype=torch.float32)
    codes = v.to(torch.float8_e4m3fn).view(torch.uint8).contiguous()
    words = codes.view(torch.int32).reshape(rows, cols // 4)
    scales = torch.randint(b_lo, b_hi + 1, (rows, cols // 32), generator=g, device=device,
                           dtype=torch.int32).to(torch.uint8)
    return words, scales


def fp8_block128_source(rows: int, cols: int, seed: int, device="cpu", log2_lo=-8.0, log2_hi=-4.0):
    """(codes uint8[rows][cols] = E4M3 of N(0, 1) draws, no NaN; block scales
    float32[ceil(rows/128)][ceil(cols/128)] = 2^u with u uniform in [log2_lo, log2_hi]).
    The default range puts the decoded weights near N(0, 0.02) with blocks of
    different magnitude, as in a block-wise FP8 checkpoint."""
    g = _gen(seed, device)
    v = torch.randn((rows, cols), generator=g, device=device, dtype=torch.float32)
    codes = v.to(torch.float8_e4m3fn).view(torch.uint8).contiguous()
    gr, gc = (rows + 127) // 128, (cols + 127) // 128
    u = torch.rand((gr, gc), generator=g, device=device, dtype=torch.float32)
    scales = torch.exp2(log2_lo + (log2_hi - log2_lo) * u)
    return codes, scales


def mlx_affine_source(rows: int, cols: int, seed: int, device="cpu"):
    """(codes uint8[rows][cols], scales f16[rows][cols/128], biases f16[rows][cols/128])."""
    g = _gen(seed, device)
    q = torch.randint(0, 256, (rows, cols), generator=g, device=device, dtype=torch.int32)
    ng = cols // 128
    scale = (torch.rand((rows, ng), generator=g, device=device) * 4e-4 + 5e-5)
    bias = -128.0 * scale + torch.randn((rows, ng), generator=g, device=device) * 1e-3
    return q.to(torch.uint8), scale.to(torch.float16), bias.to(torch.float16)


def bf16_bits(x: torch.Tensor) -> torch.Tensor:
    """Reinterpret a bfloat16/float16 tensor as its 16-bit patterns (int16 view)."""
    return x.contiguous().view(torch.int16)
