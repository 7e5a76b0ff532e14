// BF16-route projection on the CUDA cores: y[T][N] = x[T][K] * W^T with the
// packed weights dequantized in registers ("Qwen3.8-27B, NInfer int8-prefill
// artifact for the RTX 4090", "What changes": decode keeps the BF16 route;
// "Decode is bandwidth bound").
//
// Each warp streams two weight rows with 16-byte coalesced loads (lane i takes
// 16-byte chunks i, i+32, ...), unpacks the codes to exact FP32 integers in
// registers (a 2^23 exponent trick), multiplies with the activations staged
// in shared memory, applies the per-group scale to each group's partial dot
// and reduces across the warp with shuffles.  Long rows are split over CTAs
// (split-K); split partials meet in an FP32 workspace through atomics and a
// final pass converts them to the output type.
#include <algorithm>

#include "qlin_internal.cuh"

namespace qlin {
namespace {

constexpr int kThreads = 256;      // 8 warps
constexpr int kRowsPerWarp = 2;    // rows a warp streams together
constexpr int kRowsPerCta = 64;    // 8 warps x 4 passes x 2 rows
constexpr int kTokBlock = 4;       // tokens per pass over the weights
constexpr int kMaxKRange = 2048;   // columns of x staged per CTA (split-K beyond)

template <int FMT>
struct Traits;
template <>
struct Traits<QLIN_Q4_G64> { static constexpr int EPC = 32, GS = 64; };
template <>
struct Traits<QLIN_Q5_G64> { static constexpr int EPC = 32, GS = 64; };
template <>
struct Traits<QLIN_Q3_G64> { static constexpr int EPC = 64, GS = 64; };
template <>
struct Traits<QLIN_Q6_G64> { static constexpr int EPC = 32, GS = 64; };
template <>
struct Traits<QLIN_Q8_G32> { static constexpr int EPC = 16, GS = 32; };
template <>
struct Traits<QLIN_FP8_ROW> { static constexpr int EPC = 16, GS = 0; };
template <>
struct Traits<QLIN_BF16> { static constexpr int EPC = 8, GS = 0; };

// exact float of a small non-negative integer u (< 2^23) minus `off`
__device__ __forceinline__ float u_to_q(uint32_t u, float off_plus_magic) {
  return __uint_as_float(0x4B000000u | u) - off_plus_magic;
}

// Decode one 16-byte chunk of the code plane (plus the matching second-plane
// words hw) into EPC exact weight values (codes, not yet scaled).
// Element order: out[e] is element e of the chunk.
template <int FMT>
__device__ __forceinline__ void decode_chunk(uint4 c, uint2 hw, float* out) {
  uint32_t w[4] = {c.x, c.y, c.z, c.w};
  if constexpr (FMT == QLIN_Q4_G64 || FMT == QLIN_Q5_G64 || FMT == QLIN_Q6_G64) {
    constexpr float OFFM = 8388608.0f + (FMT == QLIN_Q4_G64 ? 8.0f : FMT == QLIN_Q5_G64 ? 16.0f : 32.0f);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
      for (int s = 0; s < 4; ++s) {
#pragma unroll
        for (int o = 0; o < 2; ++o) {
          uint32_t u = (w[j] >> (16 * o + 4 * s)) & 0xFu;
          // Q5: bit of element 8j+2s+o at 16o+4j+s; Q6: crumb of element
          // 8j+2s+o in word j/2 at bits 16o + 8(j&1) + 2s
          if constexpr (FMT == QLIN_Q5_G64) u |= ((hw.x >> (16 * o + 4 * j + s)) & 1u) << 4;
          if constexpr (FMT == QLIN_Q6_G64)
            u |= (((j < 2 ? hw.x : hw.y) >> (16 * o + 8 * (j & 1) + 2 * s)) & 3u) << 4;
          out[8 * j + 2 * s + o] = u_to_q(u, OFFM);
        }
      }
    }
  } else if constexpr (FMT == QLIN_Q3_G64) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
      for (int s = 0; s < 8; ++s) {
#pragma unroll
        for (int o = 0; o < 2; ++o) {
          // crumb of element 16j+2s+o at 16o+2s; its bit in word j/2 at
          // 16o + 8(j&1) + 4(s>>2) + (s&3)
          uint32_t u = (w[j] >> (16 * o + 2 * s)) & 3u;
          u |= (((j < 2 ? hw.x : hw.y) >> (16 * o + 8 * (j & 1) + 4 * (s >> 2) + (s & 3))) & 1u) << 2;
          out[16 * j + 2 * s + o] = u_to_q(u, 8388608.0f + 4.0f);
        }
      }
    }
  } else if constexpr (FMT == QLIN_Q8_G32) {
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int b = 0; b < 4; ++b) out[4 * j + b] = u_to_q(((w[j] >> (8 * b)) & 0xFFu) ^ 0x80u, 8388608.0f + 128.0f);
  } else if constexpr (FMT == QLIN_FP8_ROW) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[j] >> (16 * h)), __NV_E4M3);
        float2 f = __half22float2(__half2(hr));
        out[4 * j + 2 * h] = f.x;
        out[4 * j + 2 * h + 1] = f.y;
      }
    }
  } else {  // BF16
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      out[2 * j] = __uint_as_float(w[j] << 16);
      out[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
    }
  }
}

template <int FMT>
__device__ __forceinline__ float group_scale(const void* scales, int64_t r, int64_t k, int64_t e) {
  if constexpr (Traits<FMT>::GS > 0) {
    const __half* s = (const __half*)scales;
    return __half2float(s[r * (k / Traits<FMT>::GS) + e / Traits<FMT>::GS]);
  } else {
    return 1.0f;
  }
}

template <int FMT>
__global__ void __launch_bounds__(kThreads) gemv_cc_kernel(
    const uint8_t* __restrict__ codes, const uint8_t* __restrict__ hibits,
    const void* __restrict__ scales, const uint16_t* __restrict__ x, int64_t n, int64_t k, int64_t t,
    int64_t krange, void* __restrict__ y, int y_dtype, float* __restrict__ acc_ws) {
  constexpr int EPC = Traits<FMT>::EPC;
  // code-plane bits per element
  constexpr int CB = FMT == QLIN_BF16 ? 16 : (FMT == QLIN_Q8_G32 || FMT == QLIN_FP8_ROW) ? 8
                     : FMT == QLIN_Q3_G64 ? 2 : 4;
  extern __shared__ float xs[];  // [kTokBlock][krange]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t k0 = (int64_t)blockIdx.y * krange;
  const int64_t k1 = min(k, k0 + krange);
  const int64_t kr = k1 - k0;
  const int64_t row_bytes = k * CB / 8;
  const bool split = gridDim.y > 1;

  for (int64_t t0 = 0; t0 < t; t0 += kTokBlock) {
    const int tb = (int)min((int64_t)kTokBlock, t - t0);
    __syncthreads();
    for (int64_t i = threadIdx.x; i < (int64_t)kTokBlock * kr; i += kThreads) {
      int tt = (int)(i / kr);
      int64_t e = i % kr;
      xs[tt * krange + e] = tt < tb ? __uint_as_float((uint32_t)x[(t0 + tt) * k + k0 + e] << 16) : 0.0f;
    }
    __syncthreads();

    for (int pass = 0; pass < kRowsPerCta / (8 * kRowsPerWarp); ++pass) {
      const int64_t r0 = (int64_t)blockIdx.x * kRowsPerCta + (pass * 8 + warp) * kRowsPerWarp;
      float acc[kRowsPerWarp][kTokBlock];
#pragma unroll
      for (int rr = 0; rr < kRowsPerWarp; ++rr)
#pragma unroll
        for (int tt = 0; tt < kTokBlock; ++tt) acc[rr][tt] = 0.0f;

      for (int64_t ci = lane; ci * EPC < kr; ci += 32) {
        const int64_t e0 = k0 + ci * EPC;
#pragma unroll
        for (int rr = 0; rr < kRowsPerWarp; ++rr) {
          const int64_t r = r0 + rr;
          if (r >= n) break;
          const uint4 c = __ldcs((const uint4*)(codes + r * row_bytes + e0 * CB / 8));
          uint2 hw = make_uint2(0u, 0u);
          if constexpr (FMT == QLIN_Q5_G64) hw.x = __ldcs((const uint32_t*)(hibits + r * (k / 8) + e0 / 8));
          if constexpr (FMT == QLIN_Q3_G64) hw = __ldcs((const uint2*)(hibits + r * (k / 8) + e0 / 8));
          if constexpr (FMT == QLIN_Q6_G64) hw = __ldcs((const uint2*)(hibits + r * (k / 4) + e0 / 4));
          float wv[EPC];
          decode_chunk<FMT>(c, hw, wv);
          const float sc = group_scale<FMT>(scales, r, k, e0);
#pragma unroll
          for (int tt = 0; tt < kTokBlock; ++tt) {
            const float* xr = xs + tt * krange + (e0 - k0);
            float d = 0.0f;
#pragma unroll
            for (int e = 0; e < EPC; e += 4) {
              float4 xv = *(const float4*)(xr + e);
              d = fmaf(wv[e], xv.x, d);
              d = fmaf(wv[e + 1], xv.y, d);
              d = fmaf(wv[e + 2], xv.z, d);
              d = fmaf(wv[e + 3], xv.w, d);
            }
            acc[rr][tt] = fmaf(sc, d, acc[rr][tt]);
          }
        }
      }
#pragma unroll
      for (int rr = 0; rr < kRowsPerWarp; ++rr) {
        const int64_t r = r0 + rr;
        float rs = 1.0f;
        if constexpr (FMT == QLIN_FP8_ROW) {
          if (r < n) rs = __bfloat162float(((const __nv_bfloat16*)scales)[r]);
        }
#pragma unroll
        for (int tt = 0; tt < kTokBlock; ++tt) {
          float v = acc[rr][tt];
          for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
          if (lane == 0 && r < n && tt < tb) {
            v *= rs;
            const int64_t oi = (t0 + tt) * n + r;
            if (split) {
              atomicAdd(acc_ws + oi, v);
            } else if (y_dtype == QLIN_OUT_F32) {
              ((float*)y)[oi] = v;
            } else {
              ((__nv_bfloat16*)y)[oi] = __float2bfloat16_rn(v);
            }
          }
        }
      }
    }
  }
}

__global__ void finish_split_kernel(const float* __restrict__ acc, int64_t count, void* y,
                                    int y_dtype) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count;
       i += (int64_t)gridDim.x * blockDim.x) {
    float v = acc[i];
    if (y_dtype == QLIN_OUT_F32)
      ((float*)y)[i] = v;
    else
      ((__nv_bfloat16*)y)[i] = __float2bfloat16_rn(v);
  }
}

int64_t cc_krange(int64_t k) {
  int64_t ksplit = (k + kMaxKRange - 1) / kMaxKRange;
  int64_t kr = (k + ksplit - 1) / ksplit;
  return (kr + 63) / 64 * 64;
}

template <int FMT>
int launch_cc(const qlin_weights& w, const uint16_t* x, int64_t t, void* y, int y_dtype,
              const Exec& ex, float* acc_ws) {
  const int64_t kr = cc_krange(w.k);
  const int64_t ksplit = (w.k + kr - 1) / kr;
  dim3 grid((unsigned)((w.n + kRowsPerCta - 1) / kRowsPerCta), (unsigned)ksplit);
  // at most kTokBlock x kMaxKRange floats (32 KB): within the default 48 KB of
  // dynamic shared memory, so no attribute call is needed
  static_assert(kTokBlock * kMaxKRange * sizeof(float) <= 48 * 1024, "staged x exceeds 48 KB");
  size_t smem = (size_t)kTokBlock * kr * sizeof(float);
  if (ksplit > 1) {
    cudaError_t e = cudaMemsetAsync(acc_ws, 0, (size_t)t * w.n * sizeof(float), ex.stream);
    if (e != cudaSuccess) return QLIN_ERR_CUDA;
  }
  gemv_cc_kernel<FMT><<<grid, kThreads, smem, ex.stream>>>(
      (const uint8_t*)w.codes, (const uint8_t*)w.hibits, w.scales, x, w.n, w.k, t, kr, y, y_dtype,
      acc_ws);
  if (ksplit > 1) {
    int64_t count = t * w.n;
    int64_t blocks = std::min<int64_t>((count + 255) / 256, (int64_t)ex.num_sms * 8);
    finish_split_kernel<<<(unsigned)blocks, 256, 0, ex.stream>>>(acc_ws, count, y, y_dtype);
  }
  return cuda_status(cudaGetLastError());
}

}  // namespace

size_t gemv_cc_workspace_bytes(const qlin_weights& w, int64_t t) {
  const int64_t kr = cc_krange(w.k);
  const int64_t ksplit = (w.k + kr - 1) / kr;
  return ksplit > 1 ? (size_t)t * w.n * sizeof(float) : 0;
}

int launch_gemv_cc(const qlin_weights& w, const uint16_t* x, int64_t t, void* y, int y_dtype,
                   const Exec& ex, float* acc_ws) {
  switch (w.fmt) {
    case QLIN_Q4_G64: return launch_cc<QLIN_Q4_G64>(w, x, t, y, y_dtype, ex, acc_ws);
    case QLIN_Q5_G64: return launch_cc<QLIN_Q5_G64>(w, x, t, y, y_dtype, ex, acc_ws);
    case QLIN_Q3_G64: return launch_cc<QLIN_Q3_G64>(w, x, t, y, y_dtype, ex, acc_ws);
    case QLIN_Q6_G64: return launch_cc<QLIN_Q6_G64>(w, x, t, y, y_dtype, ex, acc_ws);
    case QLIN_Q8_G32: return launch_cc<QLIN_Q8_G32>(w, x, t, y, y_dtype, ex, acc_ws);
    case QLIN_FP8_ROW: return launch_cc<QLIN_FP8_ROW>(w, x, t, y, y_dtype, ex, acc_ws);
    case QLIN_BF16: return launch_cc<QLIN_BF16>(w, x, t, y, y_dtype, ex, acc_ws);
    default: return QLIN_ERR_INVALID_ARG;
  }
}

}  // namespace qlin
