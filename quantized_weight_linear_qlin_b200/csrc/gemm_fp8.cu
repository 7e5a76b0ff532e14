// The FP8-activation route for row-scaled FP8 weights ("Qwen3.8-27B
// EfficientThink-Uncensored FP8 for NInfer", "Conversion and verification":
// every large text projection sits in the row-scaled FP8 bank, and prefill and
// decode run FP8-activation tensor-core routes instead of dequantizing to BF16
// first).  The page fixes no activation scheme; this library's reading mirrors
// fp8_row_maxabs on the activation side: one FP32 scale per token,
// xs[t] = max_k |x[t][k]| / 448, codes xq = E4M3_rne_satfinite(x / xs).
// Then y[t][n] = FP32(ws[n] * xs[t]) * sum_k E4M3(w[n][k]) * E4M3(xq[t][k]),
// the products exact and the sum accumulated in FP32 by the tensor cores.
//
//   quantize_act_fp8_kernel  one block per token: amax, IEEE division,
//                            round-to-nearest-even with saturation;
//   gemm_fp8_kernel          persistent CTAs over 128-row x BN-token tiles:
//     warp 0     TMA: a 128 x 128 box of weight codes and a BN x 128 box of
//                activation codes per stage (128-byte swizzle), ring of stages;
//     warp 1     one elected thread issues tcgen05.mma.kind::f8f6f4 (E4M3 x
//                E4M3 -> FP32, M = 128, N = BN, K = 32) from both stages into a
//                tensor-memory accumulator (two, alternating between tiles);
//     warps 4-7  the epilogue reads a finished tile's accumulator with
//                tcgen05.ld, applies FP32(ws * xs) and writes y.
//   Tiles are taken row-tile-major (consecutive CTAs share a weight tile and
//   the activations stay in L2), so the weights stream from HBM once.
#include <algorithm>

#include "qlin_internal.cuh"

namespace qlin {
namespace {

constexpr int G8_BM = 128;          // weight rows per tile (MMA M)
constexpr int G8_BK = 128;          // K columns per stage: one 128-byte box
constexpr int G8_THREADS = 8 * 32;
constexpr int G8_WTMA = 0, G8_WMMA = 1, G8_WEPI0 = 4;
constexpr int G8_SMEM_BUDGET = 220 * 1024;

template <int BN>
struct G8Cfg {
  static constexpr int A_BYTES = G8_BM * 128;
  static constexpr int B_BYTES = BN * 128;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int NS = (G8_SMEM_BUDGET / STAGE) > 8 ? 8 : (G8_SMEM_BUDGET / STAGE);
  static constexpr size_t SMEM = (size_t)NS * STAGE + 1024 + 256;
  static constexpr uint32_t TMEM_COLS = 2 * BN < 32 ? 32 : 2 * BN;  // two accumulators
};

// Instruction descriptor: kind::f8f6f4 with E4M3 A and B, F32 accumulator, K-major.
__host__ __device__ constexpr uint32_t idesc_e4m3(int m, int n) {
  return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

__device__ __forceinline__ void mma_f8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

struct Ring {
  int slot, phase;
  __device__ __forceinline__ void next(int n) {
    if (++slot == n) {
      slot = 0;
      phase ^= 1;
    }
  }
};

struct G8Args {
  const __nv_bfloat16* ws;  // row scales [N]
  const float* xs;          // token scales [T]
  void* y;
  int32_t* dev_status;
  int64_t n, k, t;
  int64_t tiles_t, tiles;
  int y_dtype;
};

// ---------------------------------------------------------------------------
// Per-token E4M3 quantizer (one block per token).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) quantize_act_fp8_kernel(const uint16_t* __restrict__ x, int64_t k,
                                                               uint8_t* __restrict__ xq,
                                                               float* __restrict__ xs) {
  // the GEMM launched behind this kernel may start its prologue now
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ float red[8];
  const int64_t t = blockIdx.x;
  const uint4* row = (const uint4*)(x + t * k);
  uint2* orow = (uint2*)(xq + t * k);
  const int64_t n8 = k / 8;
  float a = 0.0f;
  for (int64_t i = threadIdx.x; i < n8; i += blockDim.x) {
    const uint4 v = row[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j)
      a = fmaxf(a, fmaxf(fabsf(__uint_as_float(w[j] << 16)), fabsf(__uint_as_float(w[j] & 0xFFFF0000u))));
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
  __syncthreads();
  a = 0.0f;
  for (int i = 0; i < (int)(blockDim.x >> 5); ++i) a = fmaxf(a, red[i]);
  const float s = __fdiv_rn(a, 448.0f);
  for (int64_t i = threadIdx.x; i < n8; i += blockDim.x) {
    const uint4 v = row[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[2] = {0u, 0u};
    if (s != 0.0f) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t lo = (uint32_t)__nv_cvt_float_to_fp8(__fdiv_rn(__uint_as_float(w[j] << 16), s),
                                                            __NV_SATFINITE, __NV_E4M3);
        const uint32_t hi = (uint32_t)__nv_cvt_float_to_fp8(__fdiv_rn(__uint_as_float(w[j] & 0xFFFF0000u), s),
                                                            __NV_SATFINITE, __NV_E4M3);
        o[j >> 1] |= (lo | (hi << 8)) << (16 * (j & 1));
      }
    }
    orow[i] = make_uint2(o[0], o[1]);
  }
  if (threadIdx.x == 0) xs[t] = s;
}

// ---------------------------------------------------------------------------
// FP8 x FP8 GEMM.
// ---------------------------------------------------------------------------
template <int BN>
__global__ void __launch_bounds__(G8_THREADS, 1)
    gemm_fp8_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                    G8Args args) {
  using C = G8Cfg<BN>;
  constexpr int NS = C::NS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* full = (uint64_t*)(base + NS * C::STAGE);
  uint64_t* empty = full + NS;
  uint64_t* acc_full = empty + NS;   // [2]
  uint64_t* acc_empty = acc_full + 2;  // [2]
  uint32_t* tmem_slot = (uint32_t*)(acc_empty + 2);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nkb = (int)((args.k + G8_BK - 1) / G8_BK);
  const int64_t my_tiles = (args.tiles - blockIdx.x + gridDim.x - 1) / gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == G8_WMMA) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == G8_WTMA && lane == 0) {
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_x);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  auto abort_now = [&]() {
    *abort_flag = 1;
    report_timeout(args.dev_status);
  };

  if (warp == G8_WTMA) {
    // activation codes may come from the quantizer launched just before
    asm volatile("griddepcontrol.wait;" ::: "memory");
    Ring ring{0, 0};
    int issued = 0;
    bool ok = true;
    for (int64_t it = 0; it < my_tiles && ok; ++it) {
      const int64_t tile = blockIdx.x + it * gridDim.x;
      const int rt = (int)(tile / args.tiles_t), tt = (int)(tile % args.tiles_t);
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = ring.slot;
        if (!__all_sync(0xffffffffu, !*abort_flag && mbar_wait(&empty[s], (uint32_t)(ring.phase ^ 1)))) {
          if (lane == 0) abort_now();
          ok = false;
          break;
        }
        if (elect_one()) {
          uint8_t* st = base + s * C::STAGE;
          mbar_arrive_expect_tx(&full[s], C::STAGE);
          tma_load_2d(st, &tm_w, &full[s], kb * G8_BK, rt * G8_BM);
          tma_load_2d(st + C::A_BYTES, &tm_x, &full[s], kb * G8_BK, tt * BN);
        }
        __syncwarp();
        ++issued;
        ring.next(NS);
      }
    }
    if (lane == 0)
      for (int i = issued > NS ? issued - NS : 0; i < issued; ++i)
        mbar_wait(&full[i % NS], (uint32_t)((i / NS) & 1));
  } else if (warp == G8_WMMA) {
    const uint32_t idesc = idesc_e4m3(G8_BM, BN);
    Ring ring{0, 0};
    bool ok = true;
    for (int64_t it = 0; it < my_tiles && ok; ++it) {
      const int b = (int)(it & 1);
      const uint32_t use_b = (uint32_t)(it >> 1);
      ok = __all_sync(0xffffffffu, !*abort_flag && mbar_wait(&acc_empty[b], (use_b & 1u) ^ 1u));
      const uint32_t d = tmem + b * BN;
      for (int kb = 0; kb < nkb && ok; ++kb) {
        const int s = ring.slot;
        ok = __all_sync(0xffffffffu, !*abort_flag && mbar_wait(&full[s], (uint32_t)ring.phase));
        if (!ok) break;
        tc_fence_after();
        const uint32_t as = smem_u32(base + s * C::STAGE);
        const uint64_t ad = sdesc_k_sw128(as), bd = sdesc_k_sw128(as + C::A_BYTES);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < G8_BK / 32; ++kk)  // 32 E4M3 = 32 bytes: +2 in descriptor units
            mma_f8_ss(d, ad + 2 * kk, bd + 2 * kk, idesc, (kb == 0 && kk == 0) ? 0u : 1u);
          tc_commit(&empty[s]);
          if (kb == nkb - 1) tc_commit(&acc_full[b]);
        }
        __syncwarp();
        ring.next(NS);
      }
    }
    if (!ok && lane == 0) abort_now();
  } else if (warp >= G8_WEPI0) {
    // token scales may come from the quantizer launched just before
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int quarter = warp & 3;
    const uint32_t lane_ofs = (uint32_t)(quarter * 32) << 16;
    bool dead = false;
    for (int64_t it = 0; it < my_tiles; ++it) {
      const int64_t tile = blockIdx.x + it * gridDim.x;
      const int64_t rt = tile / args.tiles_t, tt = tile % args.tiles_t;
      const int b = (int)(it & 1);
      const uint32_t use_b = (uint32_t)(it >> 1);
      const int64_t row = rt * G8_BM + quarter * 32 + lane;
      dead = dead || __any_sync(0xffffffffu, *abort_flag != 0);
      if (!dead && !__all_sync(0xffffffffu, mbar_wait(&acc_full[b], use_b & 1u))) {
        dead = true;
        abort_now();
      }
      if (dead) break;
      tc_fence_after();
      const float wsr = row < args.n ? __bfloat162float(args.ws[row]) : 0.0f;
      const int64_t t0 = tt * BN;
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 16) {
        if (t0 + c0 >= args.t) break;
        uint32_t v[16];
        tmem_ld_x16(tmem + lane_ofs + b * BN + c0, v);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) asm volatile("" : "+r"(v[j]));
        if (row < args.n) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int64_t t = t0 + c0 + j;
            if (t < args.t) {
              const float c = wsr * __ldg(args.xs + t);
              const float yv = c * __uint_as_float(v[j]);
              if (args.y_dtype == QLIN_OUT_F32)
                ((float*)args.y)[t * args.n + row] = yv;
              else
                ((__nv_bfloat16*)args.y)[t * args.n + row] = __float2bfloat16_rn(yv);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);
    }
  }

  // Every accumulator's completion was observed by the epilogue before this
  // point -- unless a wait timed out; then give the tensor core ample time
  // (1 ms) before the tensor memory is released.
  tc_fence_before();
  __syncthreads();
  if (warp == G8_WMMA) {
    if (*abort_flag) {
      const unsigned long long t0 = global_ns();
      while (global_ns() - t0 < 1000000ull) {
      }
    }
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

int bn_of(int64_t t) { return t <= 16 ? 16 : t <= 32 ? 32 : t <= 64 ? 64 : t <= 128 ? 128 : 256; }

template <int BN>
int launch_bn(const CUtensorMap& mw, const CUtensorMap& mx, G8Args a, const Exec& ex, bool pdl) {
  using C = G8Cfg<BN>;
  const cudaError_t e0 = set_smem_once<gemm_fp8_kernel<BN>>((int)C::SMEM);
  if (e0 != cudaSuccess) return cuda_status(e0);
  const int64_t rtiles = (a.n + G8_BM - 1) / G8_BM;
  a.tiles_t = (a.t + BN - 1) / BN;
  a.tiles = rtiles * a.tiles_t;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)std::min<int64_t>(a.tiles, ex.num_sms));
  cfg.blockDim = dim3(G8_THREADS);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = ex.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cuda_status(cudaLaunchKernelEx(&cfg, gemm_fp8_kernel<BN>, mw, mx, a));
}

}  // namespace

size_t gemm_fp8_workspace_bytes(int64_t t, int64_t k) {
  return ((size_t)t * k + 255) / 256 * 256 + (size_t)t * sizeof(float);
}

int launch_quantize_act_fp8(const uint16_t* x, int64_t t, int64_t k, uint8_t* xq, float* xs,
                            const Exec& ex) {
  quantize_act_fp8_kernel<<<(unsigned)t, 256, 0, ex.stream>>>(x, k, xq, xs);
  return cuda_status(cudaGetLastError());
}

int launch_gemm_fp8(const qlin_weights& w, const uint16_t* x, const uint8_t* xq, const float* xs,
                    int64_t t, void* y, int y_dtype, const Exec& ex) {
  const bool fused = x != nullptr;
  if (fused) {
    uint8_t* wq = (uint8_t*)ex.workspace;
    float* wsc = (float*)((uint8_t*)ex.workspace + ((size_t)t * w.k + 255) / 256 * 256);
    const int rc = launch_quantize_act_fp8(x, t, w.k, wq, wsc, ex);
    if (rc != QLIN_OK) return rc;
    xq = wq;
    xs = wsc;
  }
  const int bn = bn_of(t);
  CUtensorMap mw, mx;
  int rc = encode_tmap_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, w.codes, (uint64_t)w.k, (uint64_t)w.n,
                          (uint64_t)w.k, G8_BK, G8_BM, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return rc;
  rc = encode_tmap_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_UINT8, xq, (uint64_t)w.k, (uint64_t)t, (uint64_t)w.k,
                      G8_BK, (uint32_t)bn, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return rc;
  G8Args a;
  a.ws = (const __nv_bfloat16*)w.scales;
  a.xs = xs;
  a.y = y;
  a.dev_status = ex.dev_status;
  a.n = w.n;
  a.k = w.k;
  a.t = t;
  a.tiles_t = a.tiles = 0;
  a.y_dtype = y_dtype;
  switch (bn) {
    case 16: return launch_bn<16>(mw, mx, a, ex, fused);
    case 32: return launch_bn<32>(mw, mx, a, ex, fused);
    case 64: return launch_bn<64>(mw, mx, a, ex, fused);
    case 128: return launch_bn<128>(mw, mx, a, ex, fused);
    default: return launch_bn<256>(mw, mx, a, ex, fused);
  }
}

}  // namespace qlin
