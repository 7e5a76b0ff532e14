// The int8 prefill route ("Qwen3.8-27B, NInfer int8-prefill artifact for the
// RTX 4090", "What changes"): activations quantized per token and per 64
// channels (scale = amax / 127), integer MMAs over the Q4/Q5 weight codes give
// one int32 sum per 64-group, and each sum is scaled by weight_scale x
// activation_scale in FP32.
//
// B200 design:
//   * quantize_act_kernel: one warp per (token, 128 columns); lanes 0-15 and
//     16-31 each own one 64-group; amax by shuffles, IEEE division, RNE.
//   * gemm_a8_kernel: one CTA per 128 weight rows x 128 tokens.
//       - a TMA warp streams the packed weight codes (raw nibbles), the int8
//         activation codes and (for Q5) the high-bit plane into a 2-stage ring
//         of 256-column chunks (four 64-groups);
//       - four unpack warps expand the nibbles to signed int8 directly into the
//         128-byte-swizzled K-major operand layout the tensor core reads;
//       - one thread issues tcgen05.mma.kind::i8 (M=128, N=128, K=32) twice per
//         group into a fresh int32 accumulator in tensor memory, double-buffered
//         so the tensor core runs one group ahead of the epilogue;
//       - eight epilogue warps (two column halves x four lane quarters) read
//         each group's int32 sums with tcgen05.ld and apply
//         y += FP32(ws * as) * float(S) in registers; the output tile is
//         written once at the end.
//   The tensor core is idle part of the time: every group sum needs FP32 work
//   on the CUDA cores (the method's per-group promotion), which bounds this
//   kernel below the int8 tensor peak.
#include "qlin_internal.cuh"

namespace qlin {
namespace {

// ---------------------------------------------------------------------------
// Activation quantizer.
// ---------------------------------------------------------------------------
__global__ void quantize_act_kernel(const uint16_t* __restrict__ x, int64_t t, int64_t k,
                                    int8_t* __restrict__ xq, float* __restrict__ xs) {
  // let the GEMM that consumes these codes start its prologue now
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const int64_t chunks = (k + 127) / 128;
  const int64_t items = t * chunks;
  const int64_t warps_total = (int64_t)gridDim.x * (blockDim.x / 32);
  for (int64_t it = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5); it < items;
       it += warps_total) {
    const int64_t tt = it / chunks, ch = it % chunks;
    const int64_t e0 = ch * 128 + 4 * lane;
    const bool valid = e0 < k;  // k % 64 == 0: a 16-lane half is valid or not as a whole
    uint2 raw = make_uint2(0, 0);
    if (valid) raw = __ldcs((const uint2*)(x + tt * k + e0));
    float v[4] = {__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xFFFF0000u),
                  __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xFFFF0000u)};
    float a = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
    for (int o = 8; o; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    const float s = __fdiv_rn(a, 127.0f);
    uint32_t packed = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      int q = 0;
      if (s != 0.0f) q = (int)fminf(fmaxf(rintf(__fdiv_rn(v[i], s)), -127.0f), 127.0f);
      packed |= ((uint32_t)q & 0xFFu) << (8 * i);
    }
    if (valid) {
      __stcg((uint32_t*)(xq + tt * k + e0), packed);
      if ((lane & 15) == 0) xs[tt * (k / 64) + e0 / 64] = s;
    }
  }
}

// ---------------------------------------------------------------------------
// Int8 group-sum GEMM.
// ---------------------------------------------------------------------------
constexpr int BM = 128;         // weight rows per CTA (tensor-memory lanes)
constexpr int BN = 128;         // tokens per CTA (accumulator columns)
constexpr int BKC = 256;        // K columns per pipeline stage (four 64-groups)
constexpr int GPS = BKC / 64;   // groups per stage
constexpr int STAGES = 2;
constexpr int NUM_EPI_WARPS = 8;
constexpr int WARP_TMA = 8, WARP_MMA = 9, WARP_UNPACK0 = 10;
constexpr int NUM_UNPACK_THREADS = 64;  // two warps, two weight rows per thread
constexpr int NUM_THREADS = 12 * 32;

struct __align__(1024) StageSmem {
  uint8_t a[2][BM * 128];        // int8 weights, two 128-column swizzled atoms
  uint8_t b[2][BN * 128];        // int8 activations, two atoms
  uint8_t raw[BM * 128];         // packed nibbles of 256 columns (swizzled)
  uint8_t hib[BM * 32];          // Q5 high bits of 256 columns
  float xsb[GPS * BN];           // activation scales of the stage, [group][token]
  __half wsb[BM * GPS];          // weight scales of the stage, [row][group]
};

struct Smem {
  StageSmem st[STAGES];
  uint64_t full[STAGES], a_ready[STAGES], empty[STAGES];
  uint64_t d_full[2], d_empty[2], drain;
  uint32_t tmem_base;
  int abort_flag;
};

struct GemmArgs {
  const __half* ws;      // weight scales [N][K/64]
  const float* xs;       // activation scales [T][K/64]
  void* y;
  int32_t* sums_dbg;
  int32_t* dev_status;
  int64_t n, k, t;
  int y_dtype;
  int debug;
};

__device__ __forceinline__ void set_abort(Smem& sm, int32_t* dev_status) {
  *(volatile int*)&sm.abort_flag = 1;
  report_timeout(dev_status);
}
__device__ __forceinline__ bool aborted(Smem& sm) { return *(volatile int*)&sm.abort_flag != 0; }

// Expand 8 nibbles of one layout word into 8 signed int8 codes in element order.
template <int BITS>
__device__ __forceinline__ uint2 expand_word(uint32_t w, uint32_t h) {
  uint32_t lo = w & 0x0F0F0F0Fu;         // elements 0, 4, 1, 5
  uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;  // elements 2, 6, 3, 7
  uint32_t o0 = __byte_perm(lo, hi, 0x6420);  // elements 0..3
  uint32_t o1 = __byte_perm(lo, hi, 0x7531);  // elements 4..7
  if constexpr (BITS == 4) {
    o0 = (o0 + 0x78787878u) ^ 0x80808080u;
    o1 = (o1 + 0x78787878u) ^ 0x80808080u;
  } else {
    // h: this word's high bits shifted down to bits {0..3} (o = 0) and {16..19} (o = 1);
    // element 2s+o needs its bit at byte (2s+o) % 4, bit 4.
    uint32_t b0 = ((h << 4) & 0x10u) | ((h >> 4) & 0x1000u) | ((h << 19) & 0x100000u) |
                  ((h << 11) & 0x10000000u);
    uint32_t b1 = ((h << 2) & 0x10u) | ((h >> 6) & 0x1000u) | ((h << 17) & 0x100000u) |
                  ((h << 9) & 0x10000000u);
    o0 = ((o0 | b0) + 0x70707070u) ^ 0x80808080u;
    o1 = ((o1 | b1) + 0x70707070u) ^ 0x80808080u;
  }
  return make_uint2(o0, o1);
}

template <int BITS, bool DEBUG>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_a8_kernel(const __grid_constant__ CUtensorMap tm_codes,
                   const __grid_constant__ CUtensorMap tm_hib,
                   const __grid_constant__ CUtensorMap tm_act, GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((void*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t0 = (int64_t)blockIdx.x * BN;
  const int64_t n0 = (int64_t)blockIdx.y * BM;
  const int64_t ng = args.k / 64;
  const int64_t nchunks = (args.k + BKC - 1) / BKC;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&sm.full[s], 1 + 32);  // TMA issue + 32 scale-copy arrivals
      mbar_init(&sm.a_ready[s], NUM_UNPACK_THREADS);
      mbar_init(&sm.empty[s], 1 + NUM_EPI_WARPS * 32);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.d_full[b], 1);
      mbar_init(&sm.d_empty[b], NUM_EPI_WARPS * 32);
    }
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == WARP_MMA) {
    tmem_alloc(&sm.tmem_base, 256);
    tmem_relinquish();
  }
  if (warp == WARP_TMA && lane == 0) {
    tma_prefetch_desc(&tm_codes);
    tma_prefetch_desc(&tm_act);
    if (BITS == 5) tma_prefetch_desc(&tm_hib);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == WARP_TMA) {
    // lane 0 issues the TMA copies; all 32 lanes copy the stage's weight and
    // activation scales into shared memory with cp.async (same barrier).
    // The activations come from the quantizer kernel launched just before.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    int64_t issued = 0;
    for (int64_t kc = 0; kc < nchunks; ++kc) {
      const int s = (int)(kc % STAGES);
      const uint32_t par = (uint32_t)((kc / STAGES) & 1);
      if (!__all_sync(0xffffffffu, !aborted(sm) && mbar_wait(&sm.empty[s], par ^ 1))) {
        if (lane == 0) set_abort(sm, args.dev_status);
        break;
      }
      const int gcount = (int)min((int64_t)GPS, ng - kc * GPS);
      if (lane == 0) {
        uint32_t bytes = BM * 128 + 2 * BN * 128 + (BITS == 5 ? BM * 32 : 0);
        mbar_arrive_expect_tx(&sm.full[s], bytes);
        tma_load_2d(sm.st[s].raw, &tm_codes, &sm.full[s], (int)(kc * 128), (int)n0);
        if (BITS == 5) tma_load_2d(sm.st[s].hib, &tm_hib, &sm.full[s], (int)(kc * 32), (int)n0);
        tma_load_2d(sm.st[s].b[0], &tm_act, &sm.full[s], (int)(kc * BKC), (int)t0);
        tma_load_2d(sm.st[s].b[1], &tm_act, &sm.full[s], (int)(kc * BKC + 128), (int)t0);
      }
      // weight scales: two groups (4 bytes) per copy; K % 128 == 0 keeps them aligned
      for (int rr = lane; rr < BM; rr += 32) {
        const int64_t grow = n0 + rr;
        if (grow < args.n)
          for (int gp = 0; gp < gcount; gp += 2)
            cp_async_4(&sm.st[s].wsb[rr * GPS + gp], args.ws + grow * ng + kc * GPS + gp);
      }
      // activation scales, [group][token]
      for (int tt = lane; tt < BN; tt += 32) {
        const int64_t gt = t0 + tt;
        if (gt < args.t)
          for (int gi = 0; gi < gcount; ++gi)
            cp_async_4(&sm.st[s].xsb[gi * BN + tt], args.xs + gt * ng + kc * GPS + gi);
      }
      cp_async_arrive_noinc(&sm.full[s]);
      ++issued;
    }
    // let every copy in flight land before the CTA can leave
    if (lane == 0)
      for (int64_t kc = issued > STAGES ? issued - STAGES : 0; kc < issued; ++kc)
        mbar_wait(&sm.full[kc % STAGES], (uint32_t)((kc / STAGES) & 1));
  } else if (warp == WARP_MMA) {
    if (lane == 0) {
      const uint32_t idesc = idesc_i8(BM, BN);
      int64_t G = 0;
      for (int64_t kc = 0; kc < nchunks && !aborted(sm); ++kc) {
        const int s = (int)(kc % STAGES);
        const uint32_t par = (uint32_t)((kc / STAGES) & 1);
        if (!mbar_wait(&sm.full[s], par) || !mbar_wait(&sm.a_ready[s], par)) {
          set_abort(sm, args.dev_status);
          break;
        }
        tc_fence_after();
        const int gcount = (int)min((int64_t)GPS, ng - kc * GPS);
        bool ok = true;
        for (int gi = 0; gi < gcount; ++gi, ++G) {
          const int b = (int)(G & 1);
          if (!mbar_wait(&sm.d_empty[b], (uint32_t)(((G >> 1) & 1) ^ 1))) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sm.st[s].a[gi >> 1]) + (gi & 1) * 64;
          const uint32_t b_base = smem_u32(sm.st[s].b[gi >> 1]) + (gi & 1) * 64;
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            mma_i8_ss(tmem + b * BN, sdesc_k_sw128(a_base + kk * 32), sdesc_k_sw128(b_base + kk * 32),
                      idesc, kk);
          tc_commit(&sm.d_full[b]);
        }
        if (!ok) { set_abort(sm, args.dev_status); break; }
        tc_commit(&sm.empty[s]);
      }
      tc_commit(&sm.drain);
      mbar_wait(&sm.drain, 0);
    }
  } else if (warp >= WARP_UNPACK0) {
    const int ut = threadIdx.x - WARP_UNPACK0 * 32;  // rows ut and ut + 64 of the tile
    for (int64_t kc = 0; kc < nchunks; ++kc) {
      const int s = (int)(kc % STAGES);
      const uint32_t par = (uint32_t)((kc / STAGES) & 1);
      if (aborted(sm)) break;
      if (!mbar_wait(&sm.full[s], par)) { set_abort(sm, args.dev_status); break; }
      const uint8_t* raw = sm.st[s].raw;
#pragma unroll 1
      for (int rr = 0; rr < 2; ++rr) {
        const int r = ut + 64 * rr;
        uint32_t hw[8];
        if (BITS == 5) {
          const uint4* hp = (const uint4*)(sm.st[s].hib + r * 32);
          uint4 h0 = hp[0], h1 = hp[1];
          hw[0] = h0.x; hw[1] = h0.y; hw[2] = h0.z; hw[3] = h0.w;
          hw[4] = h1.x; hw[5] = h1.y; hw[6] = h1.z; hw[7] = h1.w;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {  // 16-byte unit u of the row = 32 elements
          uint4 c = *(const uint4*)(raw + sw128_offset(r, u));
          uint32_t wv[4] = {c.x, c.y, c.z, c.w};
          uint32_t o[8];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint32_t h = 0;
            if (BITS == 5) h = hw[u] >> (4 * j);
            uint2 e = expand_word<BITS>(wv[j], h);
            o[2 * j] = e.x;
            o[2 * j + 1] = e.y;
          }
          uint8_t* arow = sm.st[s].a[u >> 2];
          const uint32_t unit0 = (u & 3) * 2;
          *(uint4*)(arow + sw128_offset(r, unit0)) = make_uint4(o[0], o[1], o[2], o[3]);
          *(uint4*)(arow + sw128_offset(r, unit0 + 1)) = make_uint4(o[4], o[5], o[6], o[7]);
        }
      }
      fence_async_smem();
      mbar_arrive(&sm.a_ready[s]);
    }
  } else {
    // ---- epilogue: warps 0..7; warp w reads lanes 32*(w%4).., columns 64*(w/4)..
    const int quarter = warp & 3, half = warp >> 2;
    const int row = quarter * 32 + lane;
    const int64_t grow = n0 + row;
    const int col0 = half * 64;
    float acc[64];
#pragma unroll
    for (int j = 0; j < 64; ++j) acc[j] = 0.0f;
    int64_t G = 0;
    for (int64_t kc = 0; kc < nchunks; ++kc) {
      const int s = (int)(kc % STAGES);
      const int gcount = (int)min((int64_t)GPS, ng - kc * GPS);
      // acquire the stage (its scale copies landed when the barrier completed)
      if (__any_sync(0xffffffffu, aborted(sm)) ||
          !__all_sync(0xffffffffu, mbar_wait(&sm.full[s], (uint32_t)((kc / STAGES) & 1)))) {
        set_abort(sm, args.dev_status);
        break;
      }
      const float* xsb = sm.st[s].xsb;
      const uint2 wsr = *(const uint2*)(&sm.st[s].wsb[row * GPS]);
      const float ws0 = __low2float(*(const __half2*)&wsr.x), ws1 = __high2float(*(const __half2*)&wsr.x);
      const float ws2 = __low2float(*(const __half2*)&wsr.y), ws3 = __high2float(*(const __half2*)&wsr.y);
      bool ok = true;
      for (int gi = 0; gi < gcount; ++gi, ++G) {
        const int b = (int)(G & 1);
        const float wsc = gi == 0 ? ws0 : gi == 1 ? ws1 : gi == 2 ? ws2 : ws3;
        // warp-uniform: tcgen05.ld below needs the whole warp
        if (!__all_sync(0xffffffffu, mbar_wait(&sm.d_full[b], (uint32_t)((G >> 1) & 1)))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + b * BN + col0;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t sv[32];
          tmem_ld_x32(taddr + 32 * h, sv);
          tmem_ld_wait();
          if (h == 1) {
            tc_fence_before();
            mbar_arrive(&sm.d_empty[b]);
          }
          if (DEBUG && grow < args.n) {
            int32_t* dp = args.sums_dbg + ((t0 + col0 + 32 * h) * args.n + grow) * ng + kc * GPS + gi;
            const int64_t dstep = args.n * ng;
#pragma unroll
            for (int j = 0; j < 32; ++j, dp += dstep)
              if (t0 + col0 + 32 * h + j < args.t) *dp = (int32_t)sv[j];
          }
          const float4* xv4 = (const float4*)(xsb + gi * BN + col0 + 32 * h);
#pragma unroll
          for (int j4 = 0; j4 < 8; ++j4) {
            const float4 xv = xv4[j4];
            const int j = 4 * j4;
            acc[32 * h + j] = fmaf(wsc * xv.x, (float)(int32_t)sv[j], acc[32 * h + j]);
            acc[32 * h + j + 1] = fmaf(wsc * xv.y, (float)(int32_t)sv[j + 1], acc[32 * h + j + 1]);
            acc[32 * h + j + 2] = fmaf(wsc * xv.z, (float)(int32_t)sv[j + 2], acc[32 * h + j + 2]);
            acc[32 * h + j + 3] = fmaf(wsc * xv.w, (float)(int32_t)sv[j + 3], acc[32 * h + j + 3]);
          }
        }
      }
      if (!ok) {
        set_abort(sm, args.dev_status);
        break;
      }
      mbar_arrive(&sm.empty[s]);
    }
    if (!__any_sync(0xffffffffu, aborted(sm)) && grow < args.n) {
      const int64_t base = (t0 + col0) * args.n + grow;
      const int jmax = (int)min((int64_t)64, args.t - (t0 + col0));
      if (args.y_dtype == QLIN_OUT_F32) {
        float* yp = (float*)args.y + base;
#pragma unroll
        for (int j = 0; j < 64; ++j, yp += args.n)
          if (j < jmax) *yp = acc[j];
      } else {
        __nv_bfloat16* yp = (__nv_bfloat16*)args.y + base;
#pragma unroll
        for (int j = 0; j < 64; ++j, yp += args.n)
          if (j < jmax) *yp = __float2bfloat16_rn(acc[j]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace

size_t gemm_a8_workspace_bytes(int64_t t, int64_t n, int64_t k, int num_sms) {
  (void)n;
  (void)num_sms;
  size_t xq = ((size_t)t * k + 255) / 256 * 256;
  size_t xs = (size_t)t * (k / 64) * sizeof(float);
  return xq + xs;
}

int launch_quantize_act(const uint16_t* x, int64_t t, int64_t k, int8_t* xq, float* xs,
                        const Exec& ex) {
  const int64_t items = t * ((k + 127) / 128);
  int64_t blocks = (items + 7) / 8;
  const int64_t cap = (int64_t)ex.num_sms * 16;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  quantize_act_kernel<<<(unsigned)blocks, 256, 0, ex.stream>>>(x, t, k, xq, xs);
  return cuda_status(cudaGetLastError());
}

int launch_gemm_a8(const qlin_weights& w, const uint16_t* x, const int8_t* xq, const float* xs,
                   int64_t t, void* y, int y_dtype, uint32_t flags, int32_t* sums_dbg,
                   const Exec& ex) {
  const int64_t n = w.n, k = w.k;
  if (x != nullptr) {
    // quantize into the workspace first
    int8_t* wq = (int8_t*)ex.workspace;
    float* wsc = (float*)((uint8_t*)ex.workspace + ((size_t)t * k + 255) / 256 * 256);
    int rc = launch_quantize_act(x, t, k, wq, wsc, ex);
    if (rc != QLIN_OK) return rc;
    xq = wq;
    xs = wsc;
  }
  CUtensorMap tm_codes, tm_hib, tm_act;
  int rc = encode_tmap_2d(&tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, w.codes, (uint64_t)(k / 2),
                          (uint64_t)n, (uint64_t)(k / 2), 128, BM, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return rc;
  rc = encode_tmap_2d(&tm_act, CU_TENSOR_MAP_DATA_TYPE_UINT8, xq, (uint64_t)k, (uint64_t)t,
                      (uint64_t)k, 128, BN, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return rc;
  if (w.fmt == QLIN_Q5_G64) {
    rc = encode_tmap_2d(&tm_hib, CU_TENSOR_MAP_DATA_TYPE_UINT8, w.hibits, (uint64_t)(k / 8),
                        (uint64_t)n, (uint64_t)(k / 8), 32, BM, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (rc) return rc;
  } else {
    tm_hib = tm_codes;
  }
  GemmArgs args;
  args.ws = (const __half*)w.scales;
  args.xs = xs;
  args.y = y;
  args.sums_dbg = sums_dbg;
  args.dev_status = ex.dev_status;
  args.n = n;
  args.k = k;
  args.t = t;
  args.y_dtype = y_dtype;
  args.debug = (flags & QLIN_DEBUG_GROUP_SUMS) ? 1 : 0;

  const size_t smem = sizeof(Smem) + 1024;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((t + BN - 1) / BN), (unsigned)((n + BM - 1) / BM));
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = ex.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  auto kern = w.fmt == QLIN_Q4_G64 ? (args.debug ? gemm_a8_kernel<4, true> : gemm_a8_kernel<4, false>)
                                    : (args.debug ? gemm_a8_kernel<5, true> : gemm_a8_kernel<5, false>);
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  e = cudaLaunchKernelEx(&cfg, kern, tm_codes, tm_hib, tm_act, args);
  return cuda_status(e);
}

}  // namespace qlin
