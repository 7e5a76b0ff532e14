// BF16-weight projection at prefill sizes with the tokens on the MMA's M side:
// the GDN a/b gating projections, kept as direct BF16 weights ("Qwen3.8-27B
// EfficientThink-Uncensored FP8 for NInfer", "Conversion and verification":
// every text projection except the GDN a/b projections is row-scaled FP8; "...
// NVFP4-NInferV3", "How it was created").  y[T][N] = x[T][K] * W^T with a
// small N (96 for the a/b projections of a 27B-class layer) and many tokens.
//
// The work is reading x once: 8192 tokens x 5120 columns of BF16 are 84 MB,
// while W (96 x 5120, 1 MB) stays in L2.  So the tokens go on M (128 per tile)
// and the weight rows on N (N padded to a multiple of 16, at most 256); a CTA
// takes one or two 128-token sub-tiles, and the K range of a tile is split
// over the CTAs of one thread-block cluster (up to 16) so that all of them run
// in one wave:
//   warp 0     TMA: per stage a 64-column box of 128 token rows of x for each
//              sub-tile and one of the N weight rows (128-byte swizzle);
//   warp 1     one elected thread issues tcgen05.mma.kind::f16 (BF16 x BF16 ->
//              FP32, M = 128, N = NP, K = 16), four per stage and sub-tile,
//              one tensor-memory accumulator per sub-tile;
//   warps 4-7  the epilogue reads the accumulator with tcgen05.ld (thread =
//              token) and writes y, or, when K is split, the CTA's FP32
//              partial into its own shared memory; after a cluster barrier
//              every CTA of the cluster sums a share of the tile's outputs over
//              the parts' shared memories (distributed shared memory) in part
//              order and writes y.  No partial leaves the chip.
#include <algorithm>
#include <atomic>

#include "qlin_internal.cuh"

namespace qlin {
namespace {

constexpr int B16_BM = 128;   // tokens per tile (MMA M)
constexpr int B16_BK = 64;    // K columns per stage: one 128-byte box of BF16
constexpr int B16_THREADS = 8 * 32;
constexpr int B16_WTMA = 0, B16_WMMA = 1;
constexpr int B16_SMEM_BUDGET = 200 * 1024;

// MT 128-token sub-tiles per CTA share each stage's weight box (the weights
// come from L2 once per MT x 128 tokens instead of once per 128).
template <int NP, int MT>
struct B16Cfg {
  static constexpr int A_SUB = B16_BM * 128;          // one sub-tile's 64 columns of x
  static constexpr int A_BYTES = MT * A_SUB;
  static constexpr int B_BYTES = NP * 128;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int NS = (B16_SMEM_BUDGET / STAGE) > 8 ? 8 : (B16_SMEM_BUDGET / STAGE);
  static constexpr size_t SMEM = (size_t)NS * STAGE + 1024 + 256;
  static constexpr int COLS = MT * NP;                 // one accumulator per sub-tile
  static constexpr uint32_t TMEM_COLS = COLS <= 32 ? 32 : COLS <= 64 ? 64 : COLS <= 128 ? 128 : COLS <= 256 ? 256 : 512;
  static_assert(NP % 16 == 0 && NP <= 256, "N of an M = 128 MMA");
  static_assert(COLS <= 512, "tensor memory");
  static_assert(A_SUB % 1024 == 0 && STAGE % 1024 == 0, "1024-byte aligned operands");
  static_assert(NS >= 2, "pipeline needs two stages");
  static_assert((size_t)MT * B16_BM * (NP + 4) * 4 <= (size_t)NS * STAGE, "partial fits the stage buffers");
};

struct B16Args {
  void* out;          // y [T][N]
  int32_t* dev_status;
  int64_t n, k, t;
  int tiles, parts;   // token tiles, K parts per tile (= the cluster size)
  int out_dtype;      // QLIN_OUT_BF16 / QLIN_OUT_F32
};

constexpr int kMaxParts = 16;  // non-portable cluster size; 8 where the device refuses 16

// The FP32 partial of a CTA in its shared memory: [MT * 128 tokens][NP + 4]
// (the 4-float pad keeps the 16-byte row writes of a warp on distinct banks).
template <int NP>
constexpr int red_stride() { return NP + 4; }

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ float4 ld_dsmem_v4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

template <int NP, int MT>
__global__ void __launch_bounds__(B16_THREADS, 1)
    gemm_bf16_tok_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                         B16Args args) {
  using C = B16Cfg<NP, MT>;
  constexpr int NS = C::NS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* full = (uint64_t*)(base + NS * C::STAGE);
  uint64_t* empty = full + NS;
  uint64_t* acc_full = empty + NS;
  uint32_t* tmem_slot = (uint32_t*)(acc_full + 1);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = (int)(blockIdx.x / args.parts), part = (int)(blockIdx.x % args.parts);
  const int nkb = (int)(args.k / B16_BK);
  const int kb0 = (int)((int64_t)part * nkb / args.parts), kb1 = (int)((int64_t)(part + 1) * nkb / args.parts);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == B16_WMMA) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == B16_WTMA && lane == 0) {
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  auto abort_now = [&]() {
    *abort_flag = 1;
    report_timeout(args.dev_status);
  };

  if (warp == B16_WTMA) {
    const uint64_t pol_x = l2_evict_first(), pol_w = l2_evict_last();  // x streams once; W serves every tile
    int slot = 0, phase = 0, issued = 0;
    for (int kb = kb0; kb < kb1; ++kb) {
      if (!__all_sync(0xffffffffu, !*abort_flag && mbar_wait(&empty[slot], (uint32_t)(phase ^ 1)))) {
        if (lane == 0) abort_now();
        break;
      }
      if (elect_one()) {
        uint8_t* st = base + slot * C::STAGE;
        mbar_arrive_expect_tx(&full[slot], C::STAGE);
#pragma unroll
        for (int m = 0; m < MT; ++m)
          tma_load_2d_hint(st + m * C::A_SUB, &tm_x, &full[slot], kb * B16_BK, (tile * MT + m) * B16_BM, pol_x);
        tma_load_2d_hint(st + C::A_BYTES, &tm_w, &full[slot], kb * B16_BK, 0, pol_w);
      }
      __syncwarp();
      ++issued;
      if (++slot == NS) {
        slot = 0;
        phase ^= 1;
      }
    }
    // let every copy in flight land before the CTA can leave
    if (lane == 0)
      for (int i = issued > NS ? issued - NS : 0; i < issued; ++i)
        mbar_wait(&full[i % NS], (uint32_t)((i / NS) & 1));
  } else if (warp == B16_WMMA) {
    const uint32_t idesc = idesc_bf16(B16_BM, NP);
    int slot = 0, phase = 0;
    bool ok = true;
    for (int kb = kb0; kb < kb1 && ok; ++kb) {
      ok = __all_sync(0xffffffffu, !*abort_flag && mbar_wait(&full[slot], (uint32_t)phase));
      if (!ok) break;
      tc_fence_after();
      const uint32_t as = smem_u32(base + slot * C::STAGE);
      if (elect_one()) {
#pragma unroll
        for (int m = 0; m < MT; ++m)
#pragma unroll
          for (int kk = 0; kk < B16_BK / 16; ++kk)  // 16 BF16 = 32 bytes along the swizzled row
            mma_f16_ss(tmem + m * NP, sdesc_k_sw128(as + m * C::A_SUB + kk * 32),
                       sdesc_k_sw128(as + C::A_BYTES + kk * 32), idesc, (kb == kb0 && kk == 0) ? 0u : 1u);
        tc_commit(&empty[slot]);
        if (kb == kb1 - 1) tc_commit(acc_full);
      }
      __syncwarp();
      if (++slot == NS) {
        slot = 0;
        phase ^= 1;
      }
    }
    if (!ok && lane == 0) abort_now();
  } else if (warp >= 4) {
    const int quarter = warp & 3;
    if (!__any_sync(0xffffffffu, *abort_flag != 0) && __all_sync(0xffffffffu, mbar_wait(acc_full, 0))) {
      tc_fence_after();
      const uint32_t lane_ofs = (uint32_t)(quarter * 32) << 16;
      const bool f32 = args.out_dtype == QLIN_OUT_F32;
      const bool vec = (args.n & 3) == 0;  // rows of y start on 16 bytes (FP32) / 8 bytes (BF16)
      float* red = (float*)base;           // the stage buffers are idle once the accumulator is complete
#pragma unroll 1
      for (int m = 0; m < MT; ++m) {
        const int ltok = m * B16_BM + quarter * 32 + lane;
        const int64_t tok = (int64_t)tile * MT * B16_BM + ltok;
        const int64_t obase = tok * args.n;
#pragma unroll 1
        for (int c0 = 0; c0 < NP; c0 += 16) {
          if (c0 >= args.n) break;
          uint32_t v[16];
          tmem_ld_x16(tmem + lane_ofs + m * NP + c0, v);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) asm volatile("" : "+r"(v[j]));
          if (args.parts > 1) {
            float4* o = (float4*)(red + ltok * red_stride<NP>() + c0);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
              o[q4] = make_float4(__uint_as_float(v[4 * q4]), __uint_as_float(v[4 * q4 + 1]),
                                  __uint_as_float(v[4 * q4 + 2]), __uint_as_float(v[4 * q4 + 3]));
            continue;
          }
          if (tok >= args.t) continue;
          if (vec && c0 + 16 <= args.n) {
            if (f32) {
              float4* o = (float4*)((float*)args.out + obase + c0);
#pragma unroll
              for (int q4 = 0; q4 < 4; ++q4)
                o[q4] = make_float4(__uint_as_float(v[4 * q4]), __uint_as_float(v[4 * q4 + 1]),
                                    __uint_as_float(v[4 * q4 + 2]), __uint_as_float(v[4 * q4 + 3]));
            } else {
              uint2* o = (uint2*)((__nv_bfloat16*)args.out + obase + c0);
#pragma unroll
              for (int q4 = 0; q4 < 4; ++q4) {
                const __nv_bfloat162 lo = __floats2bfloat162_rn(__uint_as_float(v[4 * q4]), __uint_as_float(v[4 * q4 + 1]));
                const __nv_bfloat162 hi = __floats2bfloat162_rn(__uint_as_float(v[4 * q4 + 2]), __uint_as_float(v[4 * q4 + 3]));
                o[q4] = make_uint2(*(const uint32_t*)&lo, *(const uint32_t*)&hi);
              }
            }
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              if (c0 + j < args.n) {
                if (f32)
                  ((float*)args.out)[obase + c0 + j] = __uint_as_float(v[j]);
                else
                  ((__nv_bfloat16*)args.out)[obase + c0 + j] = __float2bfloat16_rn(__uint_as_float(v[j]));
              }
            }
          }
        }
      }
    } else if (lane == 0) {
      abort_now();
    }
  }

  if (args.parts > 1) {
    // Every CTA of the cluster reaches both barriers, on every path (a timed
    // out CTA contributes whatever its partial holds; its status is set).
    __syncthreads();
    cluster_sync_all();
    // rank r sums outputs [r * E / P, (r + 1) * E / P) of the tile, E = its
    // tokens x NP / 4 four-column groups, over the P partials in part order
    constexpr int C4 = NP / 4;
    constexpr int E = MT * B16_BM * C4;
    const int P = args.parts;
    const uint32_t r = cluster_rank();
    const int lo = (int)((int64_t)r * E / P), hi = (int)((int64_t)(r + 1) * E / P);
    const uint32_t red_s = smem_u32(base);
    const bool f32 = args.out_dtype == QLIN_OUT_F32;
    const bool vec = (args.n & 3) == 0;
    for (int idx = lo + (int)threadIdx.x; idx < hi; idx += B16_THREADS) {
      const int ltok = idx / C4, col = (idx - ltok * C4) * 4;
      const int64_t tok = (int64_t)tile * MT * B16_BM + ltok;
      if (tok >= args.t || col >= args.n) continue;
      const uint32_t off = (uint32_t)(ltok * red_stride<NP>() + col) * 4u;
      // all P loads in flight at once (one distributed-shared-memory latency),
      // then the sum in part order
      float4 v[kMaxParts];
#pragma unroll
      for (int p = 0; p < kMaxParts; ++p)
        if (p < P) v[p] = ld_dsmem_v4(map_to_rank(red_s + off, (uint32_t)p));
      float4 acc = v[0];
#pragma unroll
      for (int p = 1; p < kMaxParts; ++p) {
        if (p < P) {
          acc.x += v[p].x;
          acc.y += v[p].y;
          acc.z += v[p].z;
          acc.w += v[p].w;
        }
      }
      const int64_t o = tok * args.n + col;
      if (vec) {
        if (f32) {
          *(float4*)((float*)args.out + o) = acc;
        } else {
          const __nv_bfloat162 a01 = __floats2bfloat162_rn(acc.x, acc.y);
          const __nv_bfloat162 a23 = __floats2bfloat162_rn(acc.z, acc.w);
          *(uint2*)((__nv_bfloat16*)args.out + o) = make_uint2(*(const uint32_t*)&a01, *(const uint32_t*)&a23);
        }
      } else {
        const float a[4] = {acc.x, acc.y, acc.z, acc.w};
        for (int j = 0; j < 4 && col + j < args.n; ++j) {
          if (f32)
            ((float*)args.out)[o + j] = a[j];
          else
            ((__nv_bfloat16*)args.out)[o + j] = __float2bfloat16_rn(a[j]);
        }
      }
    }
    // no CTA leaves (and frees its shared memory) while another still reads it
    cluster_sync_all();
  }

  // The accumulator's completion was observed by the epilogue before this
  // point -- unless a wait timed out; then give the tensor core ample time
  // (1 ms) before the tensor memory is released.
  tc_fence_before();
  __syncthreads();
  if (warp == B16_WMMA) {
    if (*abort_flag) {
      const unsigned long long t0 = global_ns();
      while (global_ns() - t0 < 1000000ull) {
      }
    }
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

int np_of(int64_t n) { return n <= 64 ? 64 : n <= 96 ? 96 : n <= 128 ? 128 : 256; }
// 128-token sub-tiles per CTA: two from 1024 tokens on (the weight box is then
// read once per 256 tokens), one below (more CTAs for short prompts) and for
// N = 256 (the partial of two sub-tiles would not fit the stage buffers).
int mt_of(int64_t t, int np) { return t >= 1024 && np <= 128 ? 2 : 1; }


// Clusters of `p` CTAs that can be resident at once on this device (cached per
// device and configuration); 0 when the device refuses the cluster size.
template <int NP, int MT>
int max_clusters(int p) {
  static std::atomic<int> cache[64][kMaxParts + 1];  // value + 1; 0 = not asked yet
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  const int c = cache[dev][p].load(std::memory_order_relaxed);
  if (c > 0) return c - 1;
  using C = B16Cfg<NP, MT>;
  int n = 0;
  if (set_smem_once<gemm_bf16_tok_kernel<NP, MT>>((int)C::SMEM) == cudaSuccess &&
      (p <= 8 || cudaFuncSetAttribute(gemm_bf16_tok_kernel<NP, MT>, cudaFuncAttributeNonPortableClusterSizeAllowed,
                                      1) == cudaSuccess)) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p);
    cfg.blockDim = dim3(B16_THREADS);
    cfg.dynamicSmemBytes = C::SMEM;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)p;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, gemm_bf16_tok_kernel<NP, MT>, &cfg) != cudaSuccess) n = 0;
  }
  (void)cudaGetLastError();  // a refused size is an answer, not an error of this call
  cache[dev][p].store(n + 1, std::memory_order_relaxed);
  return n;
}

// K parts per token tile (the cluster size): as many as keep every tile's
// cluster resident in one wave, at most one per SM per tile and each part at
// least two 64-column stages.
template <int NP, int MT>
int parts_for(int64_t tiles, int64_t k, int num_sms) {
  const int64_t nkb = k / B16_BK;
  int64_t p = std::max<int64_t>(1, num_sms / tiles);
  p = std::min<int64_t>({p, std::max<int64_t>(1, nkb / 2), (int64_t)kMaxParts});
  for (; p > 1; --p)
    if (max_clusters<NP, MT>((int)p) >= tiles) break;
  return (int)p;
}

template <int NP, int MT>
int launch_np(const CUtensorMap& mx, const CUtensorMap& mw, const B16Args& a, int num_sms, cudaStream_t st) {
  using C = B16Cfg<NP, MT>;
  const cudaError_t e0 = set_smem_once<gemm_bf16_tok_kernel<NP, MT>>((int)C::SMEM);
  if (e0 != cudaSuccess) return cuda_status(e0);
  B16Args args = a;
  args.parts = parts_for<NP, MT>(a.tiles, a.k, num_sms);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(args.tiles * args.parts));
  cfg.blockDim = dim3(B16_THREADS);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)args.parts;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_status(cudaLaunchKernelEx(&cfg, gemm_bf16_tok_kernel<NP, MT>, mx, mw, args));
}

template <int MT>
int launch_mt(int np, const CUtensorMap& mx, const CUtensorMap& mw, const B16Args& a, int num_sms,
              cudaStream_t st) {
  switch (np) {
    case 64: return launch_np<64, MT>(mx, mw, a, num_sms, st);
    case 96: return launch_np<96, MT>(mx, mw, a, num_sms, st);
    case 128: return launch_np<128, MT>(mx, mw, a, num_sms, st);
    default: return launch_np<256, 1>(mx, mw, a, num_sms, st);
  }
}

}  // namespace

// BF16 weights with N <= 256, K a multiple of 64 (the prefill path of the
// small BF16 projections; decode sizes stay on the GEMV kernels).
bool gemm_bf16_tok_supported(const qlin_weights& w, int64_t t) {
  return w.fmt == QLIN_BF16 && w.n <= 256 && w.k % B16_BK == 0 && t > 64 && t <= (int64_t)INT32_MAX / 2;
}

size_t gemm_bf16_tok_workspace_bytes(const qlin_weights&, int64_t, int) { return 0; }

int launch_gemm_bf16_tok(const qlin_weights& w, const uint16_t* x, int64_t t, void* y, int y_dtype,
                         const Exec& ex) {
  const int np = np_of(w.n);
  CUtensorMap mx, mw;
  int rc = encode_tmap_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, (uint64_t)w.k, (uint64_t)t,
                          (uint64_t)w.k * 2, B16_BK, B16_BM, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return rc;
  rc = encode_tmap_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w.codes, (uint64_t)w.k, (uint64_t)w.n,
                      (uint64_t)w.k * 2, B16_BK, (uint32_t)np, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return rc;
  B16Args a;
  const int mt = mt_of(t, np);
  a.tiles = (int)((t + (int64_t)B16_BM * mt - 1) / ((int64_t)B16_BM * mt));
  a.parts = 1;  // launch_np sets the cluster size
  a.out = y;
  a.dev_status = ex.dev_status;
  a.n = w.n;
  a.k = w.k;
  a.t = t;
  a.out_dtype = y_dtype;
  return mt == 2 ? launch_mt<2>(np, mx, mw, a, ex.num_sms, ex.stream)
                 : launch_mt<1>(np, mx, mw, a, ex.num_sms, ex.stream);
}

}  // namespace qlin
