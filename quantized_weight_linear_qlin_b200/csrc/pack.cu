// Weight packing and source decoding kernels (offline converter steps run on
// the device).  All of it is bit-exact by construction: IEEE division
// (__fdiv_rn), round-to-nearest-even conversions and fused multiply-adds only
// where the definition has one.
//
// Sources: "Qwen3.8-27B MXFP8-CRACK -- NInfer artifact", "How it was built"
// (step 1 MXFP8, step 2 MLX affine int8); "Qwen3.8-27B EfficientThink-
// Uncensored FP8 for NInfer", "Conversion and verification" (E4M3 codes with a
// weight_scale_inv per 128 x 128 block, re-encoded with fp8_row_maxabs);
// "Qwen3.8-27B for NInfer -- RTX 5080 16 GB", "Quantization profile"
// (Q3G64_F16S, Q4G64_F16S, Q5G64_F16S); "...MXFP8-CRACK", "Caveats" (Q6
// groupwise); "...NVFP4-NInferV3", "What is in the file" (Q8).
#include "qlin_internal.cuh"

namespace qlin {
namespace {

// ---- source element -> FP32 value -----------------------------------------
struct Src {
  int kind;
  const void* src;
  const void* aux0;
  const void* aux1;
  int64_t k;
};

// E4M3 byte -> float (exact; via the hardware E4M3 -> f16 conversion).
__device__ __forceinline__ float e4m3_to_float(uint8_t c) {
  __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)c, __NV_E4M3);
  return __half2float(__half(h));
}

// 2^(b-127) as a float (b in 0..254; b = 0 is the subnormal 2^-127).
__device__ __forceinline__ float ue8m0_to_float(uint32_t b) {
  return b == 0 ? __uint_as_float(0x00400000u) : __uint_as_float(b << 23);
}

// MXFP8 element -> bfloat16 bits (exact product, one BF16 rounding).
__device__ __forceinline__ uint16_t mxfp8_to_bf16(uint8_t c, uint32_t b) {
  if ((c & 0x7F) == 0x7F || b == 255) return (uint16_t)(0x7FC0 | ((c & 0x80) << 8));
  float v = __fmul_rn(e4m3_to_float(c), ue8m0_to_float(b));
  return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t h) {
  return __uint_as_float((uint32_t)h << 16);
}

__device__ __forceinline__ float source_value(const Src& s, int64_t r, int64_t c) {
  switch (s.kind) {
    case QLIN_SRC_F32:
      return ((const float*)s.src)[r * s.k + c];
    case QLIN_SRC_BF16:
      return bf16_bits_to_float(((const uint16_t*)s.src)[r * s.k + c]);
    case QLIN_SRC_MXFP8: {
      uint32_t w = ((const uint32_t*)s.src)[r * (s.k / 4) + c / 4];
      uint8_t code = (uint8_t)(w >> (8 * (c & 3)));
      uint32_t b = ((const uint8_t*)s.aux0)[r * (s.k / 32) + c / 32];
      return bf16_bits_to_float(mxfp8_to_bf16(code, b));
    }
    case QLIN_SRC_FP8_BLOCK128: {
      // E4M3 code times its 128 x 128 block's scale in FP32 (one rounding),
      // then BF16; an E4M3 NaN code gives the BF16 NaN with its sign
      const uint8_t code = ((const uint8_t*)s.src)[r * s.k + c];
      if ((code & 0x7F) == 0x7F) return bf16_bits_to_float((uint16_t)(0x7FC0 | ((code & 0x80) << 8)));
      const float sc = ((const float*)s.aux0)[(r >> 7) * ((s.k + 127) >> 7) + (c >> 7)];
      return __bfloat162float(__float2bfloat16_rn(__fmul_rn(e4m3_to_float(code), sc)));
    }
    default: {  // MLX affine int8: one FP32 fma, then BF16
      uint8_t q = ((const uint8_t*)s.src)[r * s.k + c];
      int64_t gi = r * (s.k / 128) + c / 128;
      float sc = __half2float(((const __half*)s.aux0)[gi]);
      float bi = __half2float(((const __half*)s.aux1)[gi]);
      float v = __fmaf_rn((float)q, sc, bi);
      return __bfloat162float(__float2bfloat16_rn(v));
    }
  }
}

__device__ __forceinline__ float warp_max(float v) {
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ uint32_t warp_or(uint32_t v, int width) {
  for (int o = 1; o < width; o <<= 1) v |= __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---- Q3 / Q4 / Q5 / Q6 group-64: one warp per (row, group); lane l owns
// elements 2l, 2l+1.  Planes (u = q + 2^(BITS-1)):
//   nibble plane (Q4, Q5, Q6: bits 0..3 of u): word j = elements 8j..8j+7,
//     element 8j+2s+o at bits 16o+4s;
//   crumb plane (Q3: bits 0..1 of u, as the codes; Q6: bits 4..5, as the high
//     plane): word c = elements 16c..16c+15, element 16c+2s+o at bits 16o+2s;
//   bit plane (Q5: bit 4, Q3: bit 2): word h = elements 32h..32h+31, element
//     32h+8jj+2s+o at bit 16o+4jj+s.
template <int BITS>
__global__ void pack_groupwise64_kernel(Src s, int64_t n, uint8_t* codes, uint8_t* hibits,
                                        __half* scales) {
  constexpr float QMAX = (float)((1 << (BITS - 1)) - 1);
  constexpr int OFF = 1 << (BITS - 1);
  const int64_t ng = s.k / 64;
  const int lane = threadIdx.x & 31;
  const int64_t item = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (item >= n * ng) return;
  const int64_t r = item / ng, g = item % ng;
  const int64_t e0 = g * 64 + 2 * lane;
  float v0 = source_value(s, r, e0), v1 = source_value(s, r, e0 + 1);
  float a = warp_max(fmaxf(fabsf(v0), fabsf(v1)));
  __half s16 = __float2half_rn(__fdiv_rn(a, QMAX));
  float sc = __half2float(s16);
  int q0 = 0, q1 = 0;
  if (sc != 0.0f) {
    q0 = (int)fminf(fmaxf(rintf(__fdiv_rn(v0, sc)), -QMAX - 1.0f), QMAX);
    q1 = (int)fminf(fmaxf(rintf(__fdiv_rn(v1, sc)), -QMAX - 1.0f), QMAX);
  }
  const uint32_t u0 = (uint32_t)(q0 + OFF), u1 = (uint32_t)(q1 + OFF);
  // the lane's pair inside its nibble word (lanes 4j..4j+3 share word j), its
  // crumb word (lanes 8c..8c+7) and its bit word (lanes 16h..16h+15)
  const int sn = lane & 3, sc2 = lane & 7, jj = (lane & 15) >> 2;
  auto crumb_word = [&](uint32_t f0, uint32_t f1) {
    return warp_or(((f0 & 3u) << (2 * sc2)) | ((f1 & 3u) << (16 + 2 * sc2)), 8);
  };
  auto bit_word = [&](uint32_t b0, uint32_t b1) {
    return warp_or(((b0 & 1u) << (4 * jj + sn)) | ((b1 & 1u) << (16 + 4 * jj + sn)), 16);
  };
  if constexpr (BITS == 3) {
    const uint32_t cw = crumb_word(u0, u1);
    if (sc2 == 0) ((uint32_t*)(codes + r * (s.k / 4)))[e0 >> 4] = cw;
    const uint32_t hw = bit_word(u0 >> 2, u1 >> 2);
    if ((lane & 15) == 0) ((uint32_t*)(hibits + r * (s.k / 8)))[e0 >> 5] = hw;
  } else {
    const uint32_t word = warp_or(((u0 & 0xFu) << (4 * sn)) | ((u1 & 0xFu) << (16 + 4 * sn)), 4);
    if (sn == 0) ((uint32_t*)(codes + r * (s.k / 2)))[e0 >> 3] = word;
    if constexpr (BITS == 5) {
      const uint32_t hw = bit_word(u0 >> 4, u1 >> 4);
      if ((lane & 15) == 0) ((uint32_t*)(hibits + r * (s.k / 8)))[e0 >> 5] = hw;
    }
    if constexpr (BITS == 6) {
      const uint32_t cw = crumb_word(u0 >> 4, u1 >> 4);
      if (sc2 == 0) ((uint32_t*)(hibits + r * (s.k / 4)))[e0 >> 4] = cw;
    }
  }
  if (lane == 0) scales[r * ng + g] = s16;
}

// ---- Q8 group-32: one warp per (row, group); lane l owns element l.
__global__ void pack_q8_kernel(Src s, int64_t n, int8_t* codes, __half* scales) {
  const int64_t ng = s.k / 32;
  const int lane = threadIdx.x & 31;
  const int64_t item = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (item >= n * ng) return;
  const int64_t r = item / ng, g = item % ng;
  const int64_t e = g * 32 + lane;
  float v = source_value(s, r, e);
  float a = warp_max(fabsf(v));
  __half s16 = __float2half_rn(__fdiv_rn(a, 127.0f));
  float sc = __half2float(s16);
  int q = 0;
  if (sc != 0.0f) q = (int)fminf(fmaxf(rintf(__fdiv_rn(v, sc)), -128.0f), 127.0f);
  codes[r * s.k + e] = (int8_t)q;
  if (lane == 0) scales[r * ng + g] = s16;
}

// ---- FP8 row (fp8_row_maxabs): one block per row.
__global__ void pack_fp8_row_kernel(Src s, int64_t n, uint8_t* codes, __nv_bfloat16* scales) {
  __shared__ float red[32];
  const int64_t r = blockIdx.x;
  float a = 0.0f;
  for (int64_t c = threadIdx.x; c < s.k; c += blockDim.x) a = fmaxf(a, fabsf(source_value(s, r, c)));
  a = warp_max(a);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < blockDim.x / 32 ? red[threadIdx.x] : 0.0f;
    v = warp_max(v);
    if (threadIdx.x == 0) red[0] = v;
  }
  __syncthreads();
  a = red[0];
  __nv_bfloat16 sc16 = __float2bfloat16_rn(__fdiv_rn(a, 448.0f));
  float sc = __bfloat162float(sc16);
  for (int64_t c = threadIdx.x; c < s.k; c += blockDim.x) {
    uint8_t code = 0;
    if (sc != 0.0f)
      code = (uint8_t)__nv_cvt_float_to_fp8(__fdiv_rn(source_value(s, r, c), sc), __NV_SATFINITE,
                                            __NV_E4M3);
    codes[r * s.k + c] = code;
  }
  if (threadIdx.x == 0) scales[r] = sc16;
}

// ---- BF16 target: BF16_rne of the source value.
__global__ void pack_bf16_kernel(Src s, int64_t n, uint16_t* out) {
  int64_t total = n * s.k;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    int64_t r = i / s.k, c = i % s.k;
    out[i] = __bfloat16_as_ushort(__float2bfloat16_rn(source_value(s, r, c)));
  }
}

// ---- MXFP8 -> BF16 streaming decode: each thread turns one 16-byte chunk of
// words (16 elements, half of a 32-element scale block) into 32 bytes of BF16.
// Fast path, two elements at a time: the E4M3 fields moved into BF16 position
// read as 2^(e-127)(1+m/8) (or its subnormal) and one exact BF16 multiply by
// 2^120 gives the E4M3 value; one BF16 multiply by 2^(b-127) rounds the
// product once (RNE, subnormals kept, overflow to infinity).  Chunks with a
// NaN code or b = 255 take the element-wise path.
__device__ __forceinline__ uint32_t bf16x2_mul_rn(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ void decode_chunk(const uint4 w, uint32_t b, uint4* __restrict__ out) {
  const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
  // a byte with (c & 0x7F) == 0x7F is a NaN code
  uint32_t nan_bytes = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t y = (wv[j] & 0x7F7F7F7Fu) ^ 0x7F7F7F7Fu;  // zero byte where the code is NaN
    nan_bytes |= (y - 0x01010101u) & ~y & 0x80808080u;
  }
  uint32_t o[8];
  if (nan_bytes == 0 && b != 255) {
    const uint32_t e = b == 0 ? 0x0040u : (b << 7);  // BF16 2^(b-127) (2^-127 is subnormal)
    const uint32_t scale2 = e | (e << 16);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        // [0, c_lo, 0, c_hi]: each E4M3 byte in the high byte of a 16-bit half
        const uint32_t P = __byte_perm(wv[j], 0u, h == 0 ? 0x1404 : 0x3424);
        const uint32_t bits = ((P >> 4) & 0x07F007F0u) | (P & 0x80008000u);
        o[2 * j + h] = bf16x2_mul_rn(bf16x2_mul_rn(bits, 0x7B807B80u), scale2);
      }
    }
  } else {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint16_t h0 = mxfp8_to_bf16((uint8_t)(wv[j]), b);
      const uint16_t h1 = mxfp8_to_bf16((uint8_t)(wv[j] >> 8), b);
      const uint16_t h2 = mxfp8_to_bf16((uint8_t)(wv[j] >> 16), b);
      const uint16_t h3 = mxfp8_to_bf16((uint8_t)(wv[j] >> 24), b);
      o[2 * j] = (uint32_t)h0 | ((uint32_t)h1 << 16);
      o[2 * j + 1] = (uint32_t)h2 | ((uint32_t)h3 << 16);
    }
  }
  __stcs(out, make_uint4(o[0], o[1], o[2], o[3]));
  __stcs(out + 1, make_uint4(o[4], o[5], o[6], o[7]));
}

// DU chunks per thread and iteration, all loaded before any is decoded.
constexpr int DU = 4;

__global__ void decode_mxfp8_kernel(const uint4* __restrict__ words, const uint8_t* __restrict__ sc,
                                    int64_t chunks, uint4* __restrict__ out) {
  const int64_t nthreads = (int64_t)gridDim.x * blockDim.x;
  const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  for (int64_t base = 0; base + tid < chunks; base += DU * nthreads) {
    uint4 w[DU];
    uint32_t b[DU];
#pragma unroll
    for (int j = 0; j < DU; ++j) {
      const int64_t i = base + j * nthreads + tid;
      w[j] = make_uint4(0, 0, 0, 0);
      b[j] = 0;
      if (i < chunks) {
        w[j] = __ldcs(words + i);
        b[j] = sc[i >> 1];  // cols % 32 == 0: chunk i lies in scale block i / 2
      }
    }
#pragma unroll
    for (int j = 0; j < DU; ++j) {
      const int64_t i = base + j * nthreads + tid;
      if (i < chunks) decode_chunk(w[j], b[j], out + 2 * i);
    }
  }
}

}  // namespace

int launch_pack(int src_kind, const void* src, const void* aux0, const void* aux1,
                const qlin_weights& dst, const Exec& ex) {
  Src s{src_kind, src, aux0, aux1, dst.k};
  const int64_t n = dst.n;
  switch (dst.fmt) {
    case QLIN_Q3_G64:
    case QLIN_Q4_G64:
    case QLIN_Q5_G64:
    case QLIN_Q6_G64: {
      const int64_t items = n * (dst.k / 64);
      const unsigned blocks = (unsigned)((items + 7) / 8);
      uint8_t* c = (uint8_t*)dst.codes;
      uint8_t* h = (uint8_t*)dst.hibits;
      __half* sc = (__half*)dst.scales;
      switch (dst.fmt) {
        case QLIN_Q3_G64: pack_groupwise64_kernel<3><<<blocks, 256, 0, ex.stream>>>(s, n, c, h, sc); break;
        case QLIN_Q4_G64: pack_groupwise64_kernel<4><<<blocks, 256, 0, ex.stream>>>(s, n, c, h, sc); break;
        case QLIN_Q5_G64: pack_groupwise64_kernel<5><<<blocks, 256, 0, ex.stream>>>(s, n, c, h, sc); break;
        default: pack_groupwise64_kernel<6><<<blocks, 256, 0, ex.stream>>>(s, n, c, h, sc); break;
      }
      break;
    }
    case QLIN_Q8_G32: {
      int64_t items = n * (dst.k / 32);
      pack_q8_kernel<<<(unsigned)((items + 7) / 8), 256, 0, ex.stream>>>(
          s, n, (int8_t*)dst.codes, (__half*)dst.scales);
      break;
    }
    case QLIN_FP8_ROW:
      pack_fp8_row_kernel<<<(unsigned)n, 256, 0, ex.stream>>>(s, n, (uint8_t*)dst.codes,
                                                              (__nv_bfloat16*)dst.scales);
      break;
    case QLIN_BF16: {
      int64_t total = n * dst.k;
      int64_t blocks = (total + 255) / 256;
      if (blocks > (int64_t)ex.num_sms * 32) blocks = (int64_t)ex.num_sms * 32;
      pack_bf16_kernel<<<(unsigned)blocks, 256, 0, ex.stream>>>(s, n, (uint16_t*)dst.codes);
      break;
    }
    default:
      return QLIN_ERR_INVALID_ARG;
  }
  return cuda_status(cudaGetLastError());
}

int launch_decode_mxfp8(const uint32_t* words, const uint8_t* scales, int64_t rows, int64_t cols,
                        uint16_t* out, const Exec& ex) {
  const int64_t chunks = rows * (cols / 16);
  int64_t blocks = (chunks / DU + 255) / 256;
  const int64_t cap = (int64_t)ex.num_sms * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  decode_mxfp8_kernel<<<(unsigned)blocks, 256, 0, ex.stream>>>((const uint4*)words, scales, chunks,
                                                               (uint4*)out);
  return cuda_status(cudaGetLastError());
}

}  // namespace qlin
