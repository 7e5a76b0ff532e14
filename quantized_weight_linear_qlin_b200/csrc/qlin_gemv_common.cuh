// Pieces shared by the two GEMV kernels (tensor-core and CUDA-core): the
// packed formats' group geometry, the exact dequantization of one group of a
// row into BF16 pairs, and the stream-K unit bookkeeping.
#pragma once

#include "qlin_internal.cuh"

namespace qlin {
namespace gemv {

constexpr int BOX_BYTES = 128 * 128;  // one TMA box of codes: 128 rows x 128 bytes

// Per format: K per quantization group, groups per 128-byte box of codes,
// second (high-bit) plane and its bytes per row per 128-byte box of codes,
// per-group scales.
template <int FMT>
struct TcT;
template <>
struct TcT<QLIN_Q4_G64> {
  static constexpr int GK = 64, GPB = 4, HROW = 0;
  static constexpr bool PER_GROUP = true, HIB = false;
};
template <>
struct TcT<QLIN_Q5_G64> {
  static constexpr int GK = 64, GPB = 4, HROW = 32;  // one bit per element
  static constexpr bool PER_GROUP = true, HIB = true;
};
template <>
struct TcT<QLIN_Q3_G64> {
  static constexpr int GK = 64, GPB = 8, HROW = 64;  // 512 crumbs per box, one bit each
  static constexpr bool PER_GROUP = true, HIB = true;
};
template <>
struct TcT<QLIN_Q6_G64> {
  static constexpr int GK = 64, GPB = 4, HROW = 64;  // two bits per element
  static constexpr bool PER_GROUP = true, HIB = true;
};
template <>
struct TcT<QLIN_Q8_G32> {
  static constexpr int GK = 32, GPB = 4, HROW = 0;
  static constexpr bool PER_GROUP = true, HIB = false;
};
template <>
struct TcT<QLIN_FP8_ROW> {
  static constexpr int GK = 64, GPB = 2, HROW = 0;
  static constexpr bool PER_GROUP = false, HIB = false;  // one scale per row, applied at the end
};
template <>
struct TcT<QLIN_BF16> {
  static constexpr int GK = 64, GPB = 1, HROW = 0;
  static constexpr bool PER_GROUP = false, HIB = false;
};

// Bytes per row of a format's code plane and of its second plane (host side).
inline int64_t code_row_bytes(int fmt, int64_t k) {
  switch (fmt) {
    case QLIN_Q3_G64: return k / 4;
    case QLIN_Q4_G64:
    case QLIN_Q5_G64:
    case QLIN_Q6_G64: return k / 2;
    case QLIN_BF16: return k * 2;
    default: return k;  // Q8, FP8
  }
}
inline int64_t hib_row_bytes(int fmt, int64_t k) {
  return fmt == QLIN_Q6_G64 ? k / 4 : (fmt == QLIN_Q5_G64 || fmt == QLIN_Q3_G64) ? k / 8 : 0;
}
inline int hrow_of(int fmt) {
  return fmt == QLIN_Q5_G64 ? 32 : (fmt == QLIN_Q3_G64 || fmt == QLIN_Q6_G64) ? 64 : 0;
}

__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// ---- dequantization of one group of row r into BF16 pairs (element 2c in the
// low half of v[c]).  `codes` is the 128-byte-swizzled stage tile of the code
// plane; `hrow` points at row r's bytes of the second plane for this box.
template <int FMT>
__device__ __forceinline__ void dequant_group(const uint8_t* codes, const uint8_t* hrow, int r, int gi,
                                              uint32_t* v) {
  if constexpr (FMT == QLIN_Q4_G64 || FMT == QLIN_Q5_G64 || FMT == QLIN_Q6_G64) {
    const uint4 c0 = *(const uint4*)(codes + sw128_offset(r, 2 * gi));
    const uint4 c1 = *(const uint4*)(codes + sw128_offset(r, 2 * gi + 1));
    const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
    uint32_t h[4] = {0u, 0u, 0u, 0u};
    if constexpr (FMT == QLIN_Q5_G64) {
      const uint2 hh = *(const uint2*)(hrow + gi * 8);  // bit words of elements 0..31, 32..63
      h[0] = hh.x;
      h[1] = hh.y;
    } else if constexpr (FMT == QLIN_Q6_G64) {
      const uint4 hh = *(const uint4*)(hrow + gi * 16);  // crumb words of elements 16c..16c+15
      h[0] = hh.x;
      h[1] = hh.y;
      h[2] = hh.z;
      h[3] = hh.w;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        uint32_t m = ((w[j] >> (4 * s)) & 0x000F000Fu) | 0x43004300u;  // 128 + u, exact BF16
        if constexpr (FMT == QLIN_Q5_G64) {
          // bit of element 8j+2s+o at 16o + 4(j&3) + s -> bits 4 and 20
          const int sh = 4 * (j & 3) + s - 4;
          const uint32_t H = j < 4 ? h[0] : h[1];
          m |= (sh >= 0 ? (H >> sh) : (H << (-sh))) & 0x00100010u;
        } else if constexpr (FMT == QLIN_Q6_G64) {
          // crumb of element 8j+2s+o: word j/2, bits 16o + 8(j&1) + 2s -> bits 4..5 and 20..21
          const int sh = 8 * (j & 1) + 2 * s - 4;
          const uint32_t H = h[j >> 1];
          m |= (sh >= 0 ? (H >> sh) : (H << (-sh))) & 0x00300030u;
        }
        v[4 * j + s] = m;
      }
    }
    // 128 + u minus 128 + 2^(bits-1): the signed code, exact
    constexpr uint32_t OFF = FMT == QLIN_Q4_G64 ? 0x43084308u : FMT == QLIN_Q5_G64 ? 0x43104310u : 0x43204320u;
#pragma unroll
    for (int c = 0; c < 32; ++c) v[c] = bf16x2_sub(v[c], OFF);
  } else if constexpr (FMT == QLIN_Q3_G64) {
    const uint4 c = *(const uint4*)(codes + sw128_offset(r, gi));  // crumb words of the group
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
    const uint2 hh = *(const uint2*)(hrow + gi * 8);                // bit words
#pragma unroll
    for (int cw = 0; cw < 4; ++cw) {
      const uint32_t H = cw < 2 ? hh.x : hh.y;
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        // element 16cw+2s+o: crumb at 16o + 2s; its bit at 16o + 8(cw&1) + 4(s>>2) + (s&3) -> bit 2
        const int sh = 8 * (cw & 1) + 4 * (s >> 2) + (s & 3) - 2;
        const uint32_t hs = (sh >= 0 ? (H >> sh) : (H << (-sh))) & 0x00040004u;
        const uint32_t m = ((w[cw] >> (2 * s)) & 0x00030003u) | hs | 0x43004300u;  // 128 + u
        v[8 * cw + s] = bf16x2_sub(m, 0x43044304u);                             // - (128 + 4)
      }
    }
  } else if constexpr (FMT == QLIN_Q8_G32) {
    const uint4 c0 = *(const uint4*)(codes + sw128_offset(r, 2 * gi));
    const uint4 c1 = *(const uint4*)(codes + sw128_offset(r, 2 * gi + 1));
    const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t xw = w[j] ^ 0x80808080u;  // offset-binary bytes q + 128
      float f[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        f[i] = __uint_as_float(__byte_perm(xw, 0x4B000000u, 0x7540 + i)) - 8388736.0f;  // 2^23 + 128
      // exact small integers: their BF16 is the top half of the FP32 pattern
      v[2 * j] = __byte_perm(__float_as_uint(f[0]), __float_as_uint(f[1]), 0x7632);
      v[2 * j + 1] = __byte_perm(__float_as_uint(f[2]), __float_as_uint(f[3]), 0x7632);
    }
  } else if constexpr (FMT == QLIN_FP8_ROW) {
#pragma unroll
    for (int uq = 0; uq < 4; ++uq) {
      const uint4 c = *(const uint4*)(codes + sw128_offset(r, 4 * gi + uq));
      const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          // [0, b_lo, 0, b_hi]: each E4M3 byte in the high byte of a 16-bit half
          const uint32_t P = __byte_perm(w[j], 0u, h == 0 ? 0x1404 : 0x3424);
          // sign stays at bit 15; exponent+mantissa move to bits 4..10, which
          // reads as BF16 2^(e-127)(1+m/8) (or its subnormal); x 2^120 = E4M3 value
          const uint32_t bits = ((P >> 4) & 0x07F007F0u) | (P & 0x80008000u);
          v[8 * uq + 2 * j + h] = bf16x2_mul(bits, 0x7B807B80u);
        }
      }
    }
  } else {  // BF16 weights: straight copy
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const uint4 c = *(const uint4*)(codes + sw128_offset(r, u));
      v[4 * u] = c.x;
      v[4 * u + 1] = c.y;
      v[4 * u + 2] = c.z;
      v[4 * u + 3] = c.w;
    }
  }
}

__device__ __forceinline__ int64_t unit_start(int64_t i, int64_t U, int64_t P) { return i * U / P; }
// The CTA whose unit range holds unit u.
__device__ __forceinline__ int64_t unit_owner(int64_t u, int64_t U, int64_t P) {
  int64_t i = u * P / U;
  while (i + 1 < P && unit_start(i + 1, U, P) <= u) ++i;
  while (i > 0 && unit_start(i, U, P) > u) --i;
  return i;
}

// A ring position: slot index and the parity of its current use.  Advancing
// by one avoids integer division in the loops (64-bit divisions are slow).
struct Ring {
  int slot, phase;
  __device__ __forceinline__ void next(int n) {
    if (++slot == n) {
      slot = 0;
      phase ^= 1;
    }
  }
};

}  // namespace gemv
}  // namespace qlin
