// The int8 prefill route ("Qwen3.8-27B, NInfer int8-prefill artifact for the
// RTX 4090", "What changes"): activations quantized per token and per 64
// channels (scale = amax / 127), integer MMAs over the Q4/Q5 weight codes give
// one int32 sum per 64-group, and each sum is scaled by weight_scale x
// activation_scale in FP32.
//
// B200 design:
//   * quantize_act_kernel: eight lanes per (token, 64-group), 16-byte loads
//     (two per thread in flight, and the next two); amax by shuffles, the
//     scale by IEEE division, the codes rint(x / scale) through the correctly
//     rounded reciprocal with the IEEE division taking over near a
//     half-integer (bit-identical to one division per element, see
//     code_fast).
//   * with the full workspace: expand_i8_kernel writes the weights as int8
//     once per call and gemm_i8x_kernel (below) runs SS-operand integer MMAs
//     fed by TMA, y in registers, full waves of tiles then a stream-K tail;
//   * with only the activation part of the workspace:
//     gemm_a8_kernel: persistent, one CTA per SM walking 128-row x 128-token
//     tiles (neighbouring CTAs share weight rows; the activations stay in L2):
//       - a TMA warp streams the packed weight codes, the int8 activation codes
//         and (Q5) the high-bit plane into a 4-stage ring of 256-column chunks
//         (four 64-groups), its lanes cp.async the stage's scales;
//       - four unpack warps (one per tensor-memory lane quarter, thread = row)
//         expand each group's nibbles to signed int8 and write them with
//         tcgen05.st into an 8-slot ring of A operands in tensor memory;
//       - one thread issues tcgen05.mma.kind::i8 (A in tensor memory, B = the
//         activation codes in shared memory, M = 128, N = 128, K = 32) twice
//         per group into one of two group-sum slots, pre-armed with a bias so
//         that one FP32 subtraction turns the sum into a float;
//       - eight epilogue warps read each group's sums with tcgen05.ld and do
//         y += FP32(ws * as) * S, y itself being an FP32 tile in tensor memory
//         (keeps registers free), then write y once per tile.
//   Every group sum needs three FP32 operations on the CUDA cores (the
//   method's per-group promotion), which bounds this kernel below the int8
//   tensor peak.
#include <algorithm>

#include "qlin_internal.cuh"

namespace qlin {
namespace {

// ---------------------------------------------------------------------------
// Activation quantizer.
// ---------------------------------------------------------------------------
// Eight lanes per 64-group (8 elements = 16 bytes each), four groups per warp;
// x is [T][K] with K % 64 == 0, so group g covers elements [64g, 64g + 64) of
// the flattened array and its scale is xs[g].
// rint(x / sc) in FP32 without a division per element: with rc = 1/sc
// correctly rounded, t = x * rc differs from the exact quotient Q by at most
// 2^-23 |Q| <= 2^-16 (|Q| <= 127.5), and the IEEE quotient fl(Q) by at most
// 2^-24 |Q|.  So when t lies farther than 2^-13 from every half-integer,
// rint(t) and rint(fl(Q)) are the same integer; near a half-integer (exact
// ties included) the IEEE division decides.  rint(t) comes from one FP32 add
// of 1.5 * 2^23: the sum's ulp is 1, so it rounds t to the nearest integer
// (ties to even), the integer sits in the low bits of the sum's bit pattern
// (its low byte is the int8 code), and t minus it is exact.  Any inf / NaN on
// the way (a subnormal scale whose reciprocal overflows, non-finite inputs)
// fails the distance test and also takes the division.
constexpr float RND_MAGIC = 12582912.0f;  // 1.5 * 2^23

// int8 code byte of x, or -1 when the IEEE division must decide
__device__ __forceinline__ int code_fast(float x, float rc) {
  const float t = x * rc;
  const float m = t + RND_MAGIC;
  const float r = t - (m - RND_MAGIC);
  return fabsf(r) <= 0.5f - 0x1p-13f ? (int)(__float_as_uint(m) & 0xFFu) : -1;
}
__device__ __forceinline__ int code_div(float x, float sc) {
  return ((int)fminf(fmaxf(rintf(__fdiv_rn(x, sc)), -127.0f), 127.0f)) & 0xFF;
}

__device__ __forceinline__ void quantize_group8(uint4 raw, int lane, bool valid, int64_t idx,
                                                int8_t* __restrict__ xq, float* __restrict__ xs) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
  float v[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(v[i]));
  // the 8 lanes of a group are consecutive and aligned to 8 within the warp
#pragma unroll
  for (int o = 4; o; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  const float sc = __fdiv_rn(a, 127.0f);
  uint32_t packed[2] = {0u, 0u};
  if (sc != 0.0f) {
    const float rc = __frcp_rn(sc);
    int c[8];
    bool slow = false;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      c[i] = code_fast(v[i], rc);
      slow |= c[i] < 0;
    }
    if (slow) {  // rare: a code near a half-integer (or a non-finite value)
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (c[i] < 0) c[i] = code_div(v[i], sc);
    }
    packed[0] = (uint32_t)c[0] | ((uint32_t)c[1] << 8) | ((uint32_t)c[2] << 16) | ((uint32_t)c[3] << 24);
    packed[1] = (uint32_t)c[4] | ((uint32_t)c[5] << 8) | ((uint32_t)c[6] << 16) | ((uint32_t)c[7] << 24);
  }
  if (valid) {
    __stcg((uint2*)(xq + idx * 8), make_uint2(packed[0], packed[1]));
    if ((lane & 7) == 0) xs[idx >> 3] = sc;
  }
}

__global__ void __launch_bounds__(512) quantize_act_kernel(const uint16_t* __restrict__ x, int64_t groups,
                                                           int8_t* __restrict__ xq, float* __restrict__ xs) {
  // let the GEMM that consumes these codes start its prologue now
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const int64_t total = groups * 8;  // 8 lanes per group
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  // whole warps iterate together (the shuffles need every lane); two 16-byte
  // loads per thread per step, and the next step's two loads are issued before
  // this step's codes are computed (four in flight)
  int64_t wbase = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31);
  // x is read once: its lines go first when L2 needs room (they do not push
  // out the dirty lines of earlier kernels, which would cost a write-back)
  const uint64_t pol = l2_evict_first();
  auto load = [&](int64_t i) {
    uint4 v = make_uint4(0, 0, 0, 0);
    if (i < total)
      asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
                   : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                   : "l"(x + i * 8), "l"(pol));
    return v;
  };
  uint4 r0 = load(wbase + lane), r1 = load(wbase + stride + lane);
  for (; wbase < total; wbase += 2 * stride) {
    const int64_t i0 = wbase + lane, i1 = wbase + stride + lane;
    const bool v0 = i0 < total, v1 = i1 < total;  // total % 8 == 0: a group is valid or not as a whole
    const uint4 n0 = load(i0 + 2 * stride), n1 = load(i1 + 2 * stride);
    quantize_group8(r0, lane, v0, i0, xq, xs);
    if (__any_sync(0xffffffffu, v1)) quantize_group8(r1, lane, v1, i1, xq, xs);
    r0 = n0;
    r1 = n1;
  }
}

// ---------------------------------------------------------------------------
// Int8 group-sum GEMM.
// ---------------------------------------------------------------------------
constexpr int BM = 128;         // weight rows per tile (tensor-memory lanes)
constexpr int BN = 128;         // tokens per tile (accumulator columns)
constexpr int BKC = 256;        // K columns per pipeline stage (four 64-groups)
constexpr int GPS = BKC / 64;   // groups per stage
constexpr int NDS = 2;          // group-sum slots (128 columns each)
constexpr int NAS = 8;          // A slots (one group of int8 codes: 16 columns each)
constexpr int Y_COL0 = NDS * BN;        // the tile's FP32 output accumulator (128 columns)
constexpr int A_COL0 = Y_COL0 + BN;
constexpr int NUM_EPI_WARPS = 8;
// warp w accesses tensor-memory lanes 32 * (w % 4) ..: four consecutive warps
// cover all 128 rows
constexpr int WARP_TMA = 0, WARP_MMA = 1, WARP_UNPACK0 = 4, WARP_EPI0 = 8;
constexpr int NUM_THREADS = 16 * 32;
// Accumulators start at this bit pattern (FP32 1.5 * 2^23): after the integer
// MMAs add a group sum S (|S| < 2^22) the word reads as the float 1.5 * 2^23 + S,
// so one FP32 subtraction recovers S exactly.
constexpr uint32_t ACC_BIAS = 0x4B400000u;
constexpr float ACC_BIAS_F = 12582912.0f;

// Per code width: bytes per row and stage (256 columns) of the code plane and
// of the second plane, and the pipeline depth that fits shared memory.
//   Q3: crumb plane 64 B (unswizzled) + bit plane 32 B;  Q4: nibble plane
//   128 B (128-byte swizzle);  Q5: + bit plane 32 B;  Q6: + crumb plane 64 B.
template <int BITS>
struct A8Fmt {
  static constexpr int RAW_ROW = BITS == 3 ? 64 : 128;
  static constexpr int HIB_ROW = BITS == 6 ? 64 : (BITS == 3 || BITS == 5) ? 32 : 0;
  static constexpr int STAGES = BITS == 6 ? 3 : 4;
};

template <int BITS>
struct __align__(1024) StageSmem {
  uint8_t b[2][BN * 128];        // int8 activations, two 128-column swizzled atoms
  uint8_t raw[BM * 128];         // code plane of 256 columns
  uint8_t hib[BM * (A8Fmt<BITS>::HIB_ROW ? A8Fmt<BITS>::HIB_ROW : 16)];  // second plane
  float xsb[GPS * BN];           // activation scales of the stage, [group][token]
  __half wsb[BM * GPS];          // weight scales of the stage, [row][group]
};

template <int BITS>
struct Smem {
  static constexpr int STAGES = A8Fmt<BITS>::STAGES;
  StageSmem<BITS> st[STAGES];
  uint64_t full[STAGES], empty[STAGES];
  uint64_t a_full[NAS], a_free[NAS];
  uint64_t d_full[NDS], d_empty[NDS];
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
  int64_t tiles_t;       // token tiles
  int64_t tiles;         // row tiles x token tiles
  int y_dtype;
  float* partials;       // stream-K split tiles: [CTAs][2][BN tokens][BM rows] FP32
  int* counters;         // stream-K split tiles: [tiles][epilogue warps], zero at launch
};

template <class SM>
__device__ __forceinline__ void set_abort(SM& sm, int32_t* dev_status) {
  *(volatile int*)&sm.abort_flag = 1;
  report_timeout(dev_status);
}
template <class SM>
__device__ __forceinline__ bool aborted(SM& sm) { return *(volatile int*)&sm.abort_flag != 0; }

// A ring position: slot index and the parity of its current use.
struct Ring {
  int slot, phase;
  __device__ __forceinline__ void next(int n) {
    if (++slot == n) {
      slot = 0;
      phase ^= 1;
    }
  }
};

// Expand 8 nibbles of one layout word into the offset codes u (bytes, element
// order): element 8j+2s+o sits at bits 16o+4s.  `b0`, `b1` are the higher bits
// of u already in place (bit 4 and up of each byte).
__device__ __forceinline__ uint2 nibble_bytes(uint32_t w) {
  const uint32_t lo = w & 0x0F0F0F0Fu;         // elements 0, 4, 1, 5
  const uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;  // elements 2, 6, 3, 7
  return make_uint2(__byte_perm(lo, hi, 0x6420),   // elements 0..3
                    __byte_perm(lo, hi, 0x7531));  // elements 4..7
}

// One 64-group as 64 signed int8 codes q = u - 2^(BITS-1) in element order
// (16 words), from its code-plane words `cw` (Q3: 4 crumb words; else 8 nibble
// words) and second-plane words `hw` (Q3 / Q5: 2 bit words; Q6: 4 crumb words).
template <int BITS>
__device__ __forceinline__ void expand_group_words(const uint32_t* cw, const uint32_t* hw, uint32_t* o) {
  // u + (128 - 2^(BITS-1)) then flip bit 7: the two's complement byte of q
  constexpr uint32_t ADD = BITS == 3 ? 0x7C7C7C7Cu : BITS == 4 ? 0x78787878u : BITS == 5 ? 0x70707070u
                                                                             : 0x60606060u;
  if constexpr (BITS == 3) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {  // crumb word c: elements 16c + 2s + o
      const uint32_t m0 = cw[c] & 0x03030303u;         // elements 0, 8, 1, 9
      const uint32_t m1 = (cw[c] >> 2) & 0x03030303u;  // 2, 10, 3, 11
      const uint32_t m2 = (cw[c] >> 4) & 0x03030303u;  // 4, 12, 5, 13
      const uint32_t m3 = (cw[c] >> 6) & 0x03030303u;  // 6, 14, 7, 15
      const uint32_t e[4] = {__byte_perm(m0, m1, 0x6420), __byte_perm(m2, m3, 0x6420),
                             __byte_perm(m0, m1, 0x7531), __byte_perm(m2, m3, 0x7531)};
      // bit of element 2s+o of this crumb word: bit 16o + s of Hc
      const uint32_t Hc = hw[c >> 1] >> (8 * (c & 1));
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t Hq = Hc >> (2 * q);  // elements 4q, 4q+1, 4q+2, 4q+3 at bits 0, 16, 1, 17
        const uint32_t b = ((Hq << 2) & 0x4u) | ((Hq >> 6) & 0x400u) | ((Hq << 17) & 0x40000u) |
                           ((Hq << 9) & 0x4000000u);
        o[4 * c + q] = ((e[q] | b) + ADD) ^ 0x80808080u;
      }
    }
  } else {
#pragma unroll
    for (int jw = 0; jw < 8; ++jw) {  // nibble word jw: elements 8jw .. 8jw+7
      uint2 e = nibble_bytes(cw[jw]);
      if constexpr (BITS == 5) {
        // bit of element 8jw+2s+o at 16o + 4(jw&3) + s of word jw/4 -> bit 4 of its byte
        const uint32_t h = hw[jw >> 2] >> (4 * (jw & 3));
        e.x |= ((h << 4) & 0x10u) | ((h >> 4) & 0x1000u) | ((h << 19) & 0x100000u) |
               ((h << 11) & 0x10000000u);
        e.y |= ((h << 2) & 0x10u) | ((h >> 6) & 0x1000u) | ((h << 17) & 0x100000u) |
               ((h << 9) & 0x10000000u);
      } else if constexpr (BITS == 6) {
        // crumb of element 8jw+2s+o at 16o + 8(jw&1) + 2s of word jw/2 -> bits 4..5 of its byte
        const uint32_t cj = hw[jw >> 1] >> (8 * (jw & 1));
        e.x |= ((cj << 4) & 0x30u) | ((cj >> 4) & 0x3000u) | ((cj << 18) & 0x300000u) |
               ((cj << 10) & 0x30000000u);
        e.y |= (cj & 0x30u) | ((cj >> 8) & 0x3000u) | ((cj << 14) & 0x300000u) |
               ((cj << 6) & 0x30000000u);
      }
      o[2 * jw] = (e.x + ADD) ^ 0x80808080u;
      o[2 * jw + 1] = (e.y + ADD) ^ 0x80808080u;
    }
  }
}

// The same for group gi of row r of a stage: `raw` is the stage's code plane
// (128-byte swizzled nibbles, or for Q3 unswizzled 64-byte crumb rows), `hib`
// its second plane.
template <int BITS>
__device__ __forceinline__ void expand_group(const uint8_t* raw, const uint8_t* hib, int r, int gi,
                                             uint32_t* o) {
  uint32_t cw[8], hw[4] = {0u, 0u, 0u, 0u};
  if constexpr (BITS == 3) {
    const uint4 c = *(const uint4*)(raw + r * 64 + gi * 16);
    cw[0] = c.x; cw[1] = c.y; cw[2] = c.z; cw[3] = c.w;
  } else {
#pragma unroll
    for (int uu = 0; uu < 2; ++uu) {  // 16-byte units 2gi, 2gi+1 of the row
      const uint4 c = *(const uint4*)(raw + sw128_offset(r, 2 * gi + uu));
      cw[4 * uu] = c.x; cw[4 * uu + 1] = c.y; cw[4 * uu + 2] = c.z; cw[4 * uu + 3] = c.w;
    }
  }
  if constexpr (BITS == 3 || BITS == 5) {
    const uint2 hh = *(const uint2*)(hib + r * 32 + gi * 8);
    hw[0] = hh.x; hw[1] = hh.y;
  } else if constexpr (BITS == 6) {
    const uint4 hh = *(const uint4*)(hib + r * 64 + gi * 16);
    hw[0] = hh.x; hw[1] = hh.y; hw[2] = hh.z; hw[3] = hh.w;
  }
  expand_group_words<BITS>(cw, hw, o);
}

template <int BITS, bool DEBUG>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_a8_kernel(const __grid_constant__ CUtensorMap tm_codes,
                   const __grid_constant__ CUtensorMap tm_hib,
                   const __grid_constant__ CUtensorMap tm_act, GemmArgs args) {
  using F = A8Fmt<BITS>;
  constexpr int STAGES = F::STAGES;
  extern __shared__ uint8_t smem_raw[];
  Smem<BITS>& sm = *reinterpret_cast<Smem<BITS>*>((void*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t ng = args.k / 64;
  const int nchunks = (int)((args.k + BKC - 1) / BKC);
  // tiles of this CTA: blockIdx.x, + gridDim.x, ...; tile i covers rows
  // (i / tiles_t) * BM and tokens (i % tiles_t) * BN (neighbouring CTAs share
  // weight rows, the activations stay in L2)
  const int64_t my_tiles = (args.tiles - blockIdx.x + gridDim.x - 1) / gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&sm.full[s], 1 + 32);                 // TMA issue + 32 scale-copy arrivals
      mbar_init(&sm.empty[s], 4 + 1 + NUM_EPI_WARPS);  // unpack warps, MMA commit, epilogue warps
    }
    for (int j = 0; j < NAS; ++j) {
      mbar_init(&sm.a_full[j], 4);  // unpack warps
      mbar_init(&sm.a_free[j], 1);  // MMA commit
    }
    for (int d = 0; d < NDS; ++d) {
      mbar_init(&sm.d_full[d], 1);
      mbar_init(&sm.d_empty[d], NUM_EPI_WARPS);
    }
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == WARP_MMA) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == WARP_TMA && lane == 0) {
    tma_prefetch_desc(&tm_codes);
    tma_prefetch_desc(&tm_act);
    if (F::HIB_ROW) tma_prefetch_desc(&tm_hib);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  if (warp >= WARP_EPI0) {  // arm every group-sum slot with the bias; zero the output accumulator
    const int quarter = warp & 3, half = (warp - WARP_EPI0) >> 2;
    const uint32_t lo = (uint32_t)(quarter * 32) << 16;
    for (int d = 0; d < NDS; ++d)
      for (int c = 0; c < 64; c += 32) tmem_fill_x32(tmem + lo + d * BN + half * 64 + c, ACC_BIAS);
    for (int c = 0; c < 64; c += 32) tmem_fill_x32(tmem + lo + Y_COL0 + half * 64 + c, 0u);
    tmem_st_wait();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (warp == WARP_TMA) {
    // lane 0 issues the TMA copies; all 32 lanes copy the stage's weight and
    // activation scales into shared memory with cp.async (same barrier).
    // The activations come from the quantizer kernel launched just before.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    int issued = 0;
    Ring ring{0, 0};
    bool ok = true;
    for (int64_t it = 0; it < my_tiles && ok; ++it) {
      const int64_t tile = blockIdx.x + it * gridDim.x;
      const int64_t n0 = (tile / args.tiles_t) * BM, t0 = (tile % args.tiles_t) * BN;
      for (int kc = 0; kc < nchunks; ++kc) {
        const int s = ring.slot;
        if (!__all_sync(0xffffffffu, !aborted(sm) && mbar_wait(&sm.empty[s], (uint32_t)(ring.phase ^ 1)))) {
          if (lane == 0) set_abort(sm, args.dev_status);
          ok = false;
          break;
        }
        const int gcount = (int)min((int64_t)GPS, ng - (int64_t)kc * GPS);
        if (lane == 0) {
          uint32_t bytes = BM * F::RAW_ROW + 2 * BN * 128 + BM * F::HIB_ROW;
          mbar_arrive_expect_tx(&sm.full[s], bytes);
          tma_load_2d(sm.st[s].raw, &tm_codes, &sm.full[s], kc * F::RAW_ROW, (int)n0);
          if (F::HIB_ROW) tma_load_2d(sm.st[s].hib, &tm_hib, &sm.full[s], kc * F::HIB_ROW, (int)n0);
          tma_load_2d(sm.st[s].b[0], &tm_act, &sm.full[s], kc * BKC, (int)t0);
          tma_load_2d(sm.st[s].b[1], &tm_act, &sm.full[s], kc * BKC + 128, (int)t0);
        }
        // weight scales: two groups (4 bytes) per copy; K % 128 == 0 keeps them aligned
        for (int rr = lane; rr < BM; rr += 32) {
          const int64_t grow = n0 + rr;
          if (grow < args.n)
            for (int gp = 0; gp < gcount; gp += 2)
              cp_async_4(&sm.st[s].wsb[rr * GPS + gp], args.ws + grow * ng + (int64_t)kc * GPS + gp);
        }
        // activation scales, [group][token]
        for (int tt = lane; tt < BN; tt += 32) {
          const int64_t gt = t0 + tt;
          if (gt < args.t)
            for (int gi = 0; gi < gcount; ++gi)
              cp_async_4(&sm.st[s].xsb[gi * BN + tt], args.xs + gt * ng + (int64_t)kc * GPS + gi);
        }
        cp_async_arrive_noinc(&sm.full[s]);
        ++issued;
        ring.next(STAGES);
      }
    }
    // let every copy in flight land before the CTA can leave
    if (lane == 0) {
      Ring r2{0, 0};
      for (int i = 0; i < issued; ++i) {
        if (i + STAGES >= issued) mbar_wait(&sm.full[r2.slot], (uint32_t)r2.phase);
        r2.next(STAGES);
      }
    }
  } else if (warp == WARP_MMA) {
    if (lane == 0) {
      const uint32_t idesc = idesc_i8(BM, BN);
      Ring ring{0, 0}, ar{0, 0}, dr{0, 0};
      bool ok = true;
      for (int64_t it = 0; it < my_tiles && ok; ++it) {
        for (int kc = 0; kc < nchunks && ok; ++kc) {
          const int s = ring.slot;
          ok = !aborted(sm) && mbar_wait(&sm.full[s], (uint32_t)ring.phase);
          const int gcount = (int)min((int64_t)GPS, ng - (int64_t)kc * GPS);
          for (int gi = 0; gi < gcount && ok; ++gi) {
            ok = mbar_wait(&sm.a_full[ar.slot], (uint32_t)ar.phase) &&
                 mbar_wait(&sm.d_empty[dr.slot], (uint32_t)(dr.phase ^ 1)) && !aborted(sm);
            if (!ok) break;
            tc_fence_after();
            const uint32_t b_base = smem_u32(sm.st[s].b[gi >> 1]) + (gi & 1) * 64;
            const uint32_t a_col = tmem + A_COL0 + ar.slot * 16;
#pragma unroll
            for (int kk = 0; kk < 2; ++kk)
              mma_i8_ts(tmem + dr.slot * BN, a_col + kk * 8, sdesc_k_sw128(b_base + kk * 32), idesc, 1u);
            tc_commit(&sm.a_free[ar.slot]);
            tc_commit(&sm.d_full[dr.slot]);
            ar.next(NAS);
            dr.next(NDS);
          }
          if (ok) tc_commit(&sm.empty[s]);  // the activation tile is free once these MMAs finish
          ring.next(STAGES);
        }
      }
      if (!ok) set_abort(sm, args.dev_status);
    }
    __syncwarp();
  } else if (warp >= WARP_UNPACK0 && warp < WARP_EPI0) {
    // ---- unpack: thread = weight row; nibbles (+ high bits) -> signed int8
    // codes written with tcgen05.st as the MMA's A operand, one group per A slot
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_ofs = (uint32_t)(quarter * 32) << 16;
    Ring ring{0, 0}, ar{0, 0};
    bool ok = true;
    for (int64_t it = 0; it < my_tiles && ok; ++it) {
      for (int kc = 0; kc < nchunks; ++kc) {
        const int s = ring.slot;
        if (!__all_sync(0xffffffffu, !aborted(sm) && mbar_wait(&sm.full[s], (uint32_t)ring.phase))) {
          if (lane == 0) set_abort(sm, args.dev_status);
          ok = false;
          break;
        }
        const int gcount = (int)min((int64_t)GPS, ng - (int64_t)kc * GPS);
        const uint8_t* raw = sm.st[s].raw;
        for (int gi = 0; gi < gcount; ++gi) {
          // the MMAs that last read this A slot are complete
          if (!__all_sync(0xffffffffu, mbar_wait(&sm.a_free[ar.slot], (uint32_t)(ar.phase ^ 1)))) {
            if (lane == 0) set_abort(sm, args.dev_status);
            ok = false;
            break;
          }
          tc_fence_after();
          uint32_t o[16];
          expand_group<BITS>(raw, sm.st[s].hib, r, gi, o);
          tmem_st_x16(tmem + lane_ofs + A_COL0 + ar.slot * 16, o);
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.a_full[ar.slot]);
          ar.next(NAS);
        }
        if (!ok) break;
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty[s]);  // codes and high bits consumed
        ring.next(STAGES);
      }
    }
  } else if (warp >= WARP_EPI0) {
    // ---- epilogue: warp w reads lanes 32*(w%4).., token columns 64*half..; the
    // tile's FP32 accumulator y lives in tensor memory next to the group sums:
    // per group and 16-column chunk, y += FP32(ws * as) * S
    const int quarter = warp & 3, half = (warp - WARP_EPI0) >> 2;
    const int row = quarter * 32 + lane;
    const int col0 = half * 64;
    const uint32_t lane_ofs = (uint32_t)(quarter * 32) << 16;
    const uint32_t yaddr = tmem + lane_ofs + Y_COL0 + col0;
    Ring ring{0, 0}, dr{0, 0};
    bool ok = true;
    for (int64_t it = 0; it < my_tiles && ok; ++it) {
      const int64_t tile = blockIdx.x + it * gridDim.x;
      const int64_t n0 = (tile / args.tiles_t) * BM, t0 = (tile % args.tiles_t) * BN;
      const int64_t grow = n0 + row;
      for (int kc = 0; kc < nchunks && ok; ++kc) {
        const int s = ring.slot;
        const int gcount = (int)min((int64_t)GPS, ng - (int64_t)kc * GPS);
        // acquire the stage (its scale copies landed when the barrier completed)
        if (__any_sync(0xffffffffu, aborted(sm)) ||
            !__all_sync(0xffffffffu, mbar_wait(&sm.full[s], (uint32_t)ring.phase))) {
          ok = false;
          break;
        }
        const float* xsb = sm.st[s].xsb;
        const uint2 wsr = *(const uint2*)(&sm.st[s].wsb[row * GPS]);
        for (int gi = 0; gi < gcount; ++gi) {
          const uint32_t wsw = (gi & 2) ? wsr.y : wsr.x;
          const float wsc = __half2float(__ushort_as_half((unsigned short)(wsw >> ((gi & 1) * 16))));
          // warp-uniform: tcgen05.ld below needs the whole warp
          if (!__all_sync(0xffffffffu, mbar_wait(&sm.d_full[dr.slot], (uint32_t)dr.phase))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t saddr = tmem + lane_ofs + dr.slot * BN + col0;
          // four 16-column chunks, software-pipelined: chunk h+1's tensor-memory
          // loads are in flight while chunk h is computed
          uint32_t s0[16], y0[16], s1[16], y1[16];
          tmem_ld_x16(saddr, s0);
          tmem_ld_x16(yaddr, y0);
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            uint32_t* sv = (h & 1) ? s1 : s0;
            uint32_t* yv = (h & 1) ? y1 : y0;
            tmem_ld_wait();
            if (h < 3) {
              tmem_ld_x16(saddr + 16 * (h + 1), (h & 1) ? s0 : s1);
              tmem_ld_x16(yaddr + 16 * (h + 1), (h & 1) ? y0 : y1);
            }
            tmem_fill_x16(saddr + 16 * h, ACC_BIAS);  // re-arm for a later group
            if (DEBUG && grow < args.n) {
              int32_t* dp = args.sums_dbg + ((t0 + col0 + 16 * h) * args.n + grow) * ng + (int64_t)kc * GPS + gi;
              const int64_t dstep = args.n * ng;
#pragma unroll
              for (int j = 0; j < 16; ++j, dp += dstep)
                if (t0 + col0 + 16 * h + j < args.t) *dp = (int32_t)(sv[j] - ACC_BIAS);
            }
            const float4* xv4 = (const float4*)(xsb + gi * BN + col0 + 16 * h);
#pragma unroll
            for (int j4 = 0; j4 < 4; ++j4) {
              const float4 xv = xv4[j4];
              const float xa[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int j = 4 * j4 + e;
                yv[j] = __float_as_uint(
                    fmaf(wsc * xa[e], __uint_as_float(sv[j]) - ACC_BIAS_F, __uint_as_float(yv[j])));
              }
            }
            tmem_st_x16(yaddr + 16 * h, yv);
          }
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.d_empty[dr.slot]);
          dr.next(NDS);
        }
        if (!ok) break;
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty[s]);  // the stage's scales are consumed
        ring.next(STAGES);
      }
      if (!ok) {
        set_abort(sm, args.dev_status);
        break;
      }
      // the tile is complete: write y, zero the accumulator for the next tile
      const int jmax = (int)min((int64_t)64, args.t - (t0 + col0));
#pragma unroll 1
      for (int h = 0; h < 4; ++h) {
        uint32_t yv[16];
        tmem_ld_x16(yaddr + 16 * h, yv);
        tmem_ld_wait();
        tmem_fill_x16(yaddr + 16 * h, 0u);
        if (grow < args.n) {
          const int64_t base = (t0 + col0 + 16 * h) * args.n + grow;
          if (args.y_dtype == QLIN_OUT_F32) {
            float* yp = (float*)args.y + base;
#pragma unroll
            for (int j = 0; j < 16; ++j, yp += args.n)
              if (16 * h + j < jmax) *yp = __uint_as_float(yv[j]);
          } else {
            __nv_bfloat16* yp = (__nv_bfloat16*)args.y + base;
#pragma unroll
            for (int j = 0; j < 16; ++j, yp += args.n)
              if (16 * h + j < jmax) *yp = __float2bfloat16_rn(__uint_as_float(yv[j]));
          }
        }
      }
      tmem_st_wait();
    }
  }

  // Every group's completion was observed by the epilogue before this point,
  // so no MMA is in flight -- unless a wait timed out; then give the tensor
  // core ample time (1 ms) before the tensor memory is released.
  tc_fence_before();
  __syncthreads();
  if (warp == WARP_MMA) {
    if (aborted(sm)) {
      const unsigned long long t0 = global_ns();
      while (global_ns() - t0 < 1000000ull) {
      }
    }
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}


// ---------------------------------------------------------------------------
// Int8 group-sum GEMM on int8 weights expanded once per call.
//   expand_i8_kernel  packed Q3..Q6 codes -> int8 [N][K] in the workspace
//                     (one thread per (row, 64-group), bandwidth-bound);
//   gemm_i8x_kernel   persistent CTAs over 128-row x 128-token tiles, row-tile
//                     major (consecutive CTAs share a weight tile, which L2
//                     then serves); with fewer than X_SK_MAX_WAVES full waves
//                     of tiles, the tiles after the last full wave are split
//                     over all CTAs by their K chunks (stream-K, SK = true):
//     warp 0     TMA: per stage a 128 x 128 B box of int8 weights and one of
//                int8 activation codes (two 64-groups, 128-byte swizzle); its
//                lanes cp.async the stage's weight and activation scales;
//     warp 1     one elected thread issues tcgen05.mma.kind::i8 from both
//                shared-memory operands (M = N = 128, K = 32), two per group,
//                the first overwriting its accumulator, into one of three
//                group-sum slots in tensor memory, and commits per group;
//     warps 4-19 sixteen epilogue warps (row = lane of the warp's lane
//                quarter, 32 tokens each, four warps per scheduler): read a
//                group's sums with one tcgen05.ld, release the slot, and fold
//                y += FP32(ws * as) * S in registers with paired FP32 multiplies
//                and FMAs (S converts to FP32 exactly: |S| < 2^22); y is
//                written once per tile.
// No code expansion, no A operand written by the CUDA cores, and no output
// tile in tensor memory: the tensor memory traffic per group is one read of
// the sums.
// ---------------------------------------------------------------------------
constexpr int X_BK = 128;                   // K columns per stage: two 64-groups
constexpr int X_NDS = 3;                    // group-sum slots
constexpr int X_NEPI = 16;                  // epilogue warps: 4 lane quarters x 4 token blocks
constexpr int X_WEPI0 = 4;
constexpr int X_THREADS = (X_WEPI0 + X_NEPI) * 32;  // warps 0..3 control, 4..19 epilogue

struct __align__(1024) XStage {
  uint8_t a[BM * 128];      // int8 weights, 128 rows x 128 columns (swizzled)
  uint8_t b[BN * 128];      // int8 activations, 128 tokens x 128 columns (swizzled)
  float xsb[2 * BN];        // activation scales [group][token]
  __half wsb[BM * 2];       // weight scales [row][group]
};
constexpr int X_NS = 6;
constexpr int X_SK_MAX_WAVES = 8;           // stream-K for the last wave only below this many waves
struct XSmem {
  XStage st[X_NS];
  uint64_t full[X_NS], empty[X_NS];
  uint64_t sfull[X_NDS], sfree[X_NDS];
  uint32_t tmem_base;
  int abort_flag;
};

template <int BITS>
__global__ void expand_i8_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ hib,
                                 int64_t n, int64_t k, int8_t* __restrict__ out, int* __restrict__ counters,
                                 int64_t ncounters) {
  // the GEMM's split-tile counters start the call at zero
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < ncounters;
       i += (int64_t)gridDim.x * blockDim.x)
    counters[i] = 0;
  const int64_t ng = k / 64;
  for (int64_t item = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; item < n * ng;
       item += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = item / ng, g = item - r * ng;
    uint32_t cw[8], hw[4] = {0u, 0u, 0u, 0u};
    if constexpr (BITS == 3) {
      const uint4 c = __ldcs((const uint4*)(codes + r * (k / 4) + g * 16));
      cw[0] = c.x; cw[1] = c.y; cw[2] = c.z; cw[3] = c.w;
    } else {
      const uint4* src = (const uint4*)(codes + r * (k / 2) + g * 32);
      const uint4 c0 = __ldcs(src), c1 = __ldcs(src + 1);
      cw[0] = c0.x; cw[1] = c0.y; cw[2] = c0.z; cw[3] = c0.w;
      cw[4] = c1.x; cw[5] = c1.y; cw[6] = c1.z; cw[7] = c1.w;
    }
    if constexpr (BITS == 3 || BITS == 5) {
      const uint2 hh = __ldcs((const uint2*)(hib + r * (k / 8) + g * 8));
      hw[0] = hh.x; hw[1] = hh.y;
    } else if constexpr (BITS == 6) {
      const uint4 hh = __ldcs((const uint4*)(hib + r * (k / 4) + g * 16));
      hw[0] = hh.x; hw[1] = hh.y; hw[2] = hh.z; hw[3] = hh.w;
    }
    uint32_t o[16];
    expand_group_words<BITS>(cw, hw, o);
    uint4* dst = (uint4*)(out + r * k + g * 64);
#pragma unroll
    for (int q = 0; q < 4; ++q) dst[q] = make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
  }
}

template <bool DEBUG, bool SK>
__global__ void __launch_bounds__(X_THREADS, 1)
    gemm_i8x_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_act,
                    GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  XSmem& sm = *reinterpret_cast<XSmem*>((void*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t ng = args.k / 64;
  const int nchunks = (int)(args.k / X_BK);
  // Whole tiles in full waves (tile = CTA + round * CTAs: the CTAs that run at
  // the same time share weight row tiles, which L2 then serves), then the
  // tiles left over after the last full wave split evenly over all CTAs by
  // their (tile, K chunk) iterations (stream-K), so that no SM idles through a
  // partial last wave.
  // (32-bit counts: tiles x chunks < 2^31 is checked on the host)
  // SK = false (eight or more full waves: the idle part of the last one is
  // small, and splitting it costs about as much): every tile whole, round
  // robin, this CTA's rounds including the last, partial wave.
  const int P = (int)gridDim.x, ntiles = (int)args.tiles;
  const int rounds = SK ? ntiles / P : (ntiles - (int)blockIdx.x + P - 1) / P;
  const int dp_tiles = SK ? rounds * P : ntiles;
  const int iters = (ntiles - dp_tiles) * nchunks;  // stream-K iterations
  const int it0 = (int)((int64_t)blockIdx.x * iters / P), it1 = (int)(((int64_t)blockIdx.x + 1) * iters / P);
  const int dp_jobs = rounds * nchunks;
  const int njobs = dp_jobs + (it1 - it0);  // this CTA's (tile, chunk) steps

  if (threadIdx.x == 0) {
    for (int s = 0; s < X_NS; ++s) {
      mbar_init(&sm.full[s], 1 + 32);  // TMA issue + 32 scale-copy arrivals
      mbar_init(&sm.empty[s], 1 + X_NEPI);  // the MMA commit + the epilogue warps (scales read)
    }
    for (int d = 0; d < X_NDS; ++d) {
      mbar_init(&sm.sfull[d], 1);
      mbar_init(&sm.sfree[d], X_NEPI);
    }
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_act);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    // the activation codes and the expanded weights come from the kernels
    // launched just before
    asm volatile("griddepcontrol.wait;" ::: "memory");
    int issued = 0;
    Ring ring{0, 0};
    bool ok = true;
    // the steps' tile and K chunk, advanced incrementally (no division per step)
    int tile = (int)blockIdx.x, kc = 0;
    if (dp_jobs == 0) {
      tile = dp_tiles + it0 / nchunks;
      kc = it0 - (it0 / nchunks) * nchunks;
    }
    const int tiles_t = (int)args.tiles_t;
    int rt = tile / tiles_t, tt = tile - rt * tiles_t;  // row tile, token tile
    for (int j = 0; j < njobs && ok; ++j) {
      if (j == dp_jobs && j > 0) {  // from the full waves into the stream-K range
        tile = dp_tiles + it0 / nchunks;
        kc = it0 - (it0 / nchunks) * nchunks;
        rt = tile / tiles_t;
        tt = tile - rt * tiles_t;
      }
      const int64_t n0 = (int64_t)rt * BM, t0 = (int64_t)tt * BN;
      {
        const int s = ring.slot;
        if (!__all_sync(0xffffffffu, !aborted(sm) && mbar_wait(&sm.empty[s], (uint32_t)(ring.phase ^ 1)))) {
          if (lane == 0) set_abort(sm, args.dev_status);
          ok = false;
          break;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(&sm.full[s], (uint32_t)(BM * 128 + BN * 128));
          tma_load_2d(sm.st[s].a, &tm_w, &sm.full[s], kc * X_BK, (int)n0);
          tma_load_2d(sm.st[s].b, &tm_act, &sm.full[s], kc * X_BK, (int)t0);
        }
        // weight scales: two groups (4 bytes) per row; activation scales [group][token]
        for (int rr = lane; rr < BM; rr += 32) {
          const int64_t grow = n0 + rr;
          if (grow < args.n) cp_async_4(&sm.st[s].wsb[rr * 2], args.ws + grow * ng + (int64_t)kc * 2);
        }
        for (int tt = lane; tt < BN; tt += 32) {
          const int64_t gt = t0 + tt;
          if (gt < args.t)
            for (int gi = 0; gi < 2; ++gi)
              cp_async_4(&sm.st[s].xsb[gi * BN + tt], args.xs + gt * ng + (int64_t)kc * 2 + gi);
        }
        cp_async_arrive_noinc(&sm.full[s]);
        ++issued;
        ring.next(X_NS);
      }
      if (++kc == nchunks) {  // next tile: the next wave's, or the next one in the range
        kc = 0;
        tile += j < dp_jobs ? P : 1;
        rt = tile / tiles_t;
        tt = tile - rt * tiles_t;
      }
    }
    if (lane == 0) {
      Ring r2{0, 0};
      for (int i = 0; i < issued; ++i) {
        if (i + X_NS >= issued) mbar_wait(&sm.full[r2.slot], (uint32_t)r2.phase);
        r2.next(X_NS);
      }
    }
  } else if (warp == 1) {
    const uint32_t idesc = idesc_i8(BM, BN);
    Ring ring{0, 0}, dr{0, 0};
    bool ok = true;
    for (int j = 0; j < njobs && ok; ++j) {
      {
        const int s = ring.slot;
        ok = __all_sync(0xffffffffu, !aborted(sm) && mbar_wait(&sm.full[s], (uint32_t)ring.phase));
        if (!ok) break;
        const uint32_t as = smem_u32(sm.st[s].a), bs = smem_u32(sm.st[s].b);
        for (int gi = 0; gi < 2 && ok; ++gi) {
          ok = __all_sync(0xffffffffu, mbar_wait(&sm.sfree[dr.slot], (uint32_t)(dr.phase ^ 1)) && !aborted(sm));
          if (!ok) break;
          tc_fence_after();
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < 2; ++kk)  // K = 32 int8 = 32 bytes of the swizzled rows
              mma_i8_ss(tmem + dr.slot * BN, sdesc_k_sw128(as + gi * 64 + kk * 32),
                        sdesc_k_sw128(bs + gi * 64 + kk * 32), idesc, kk ? 1u : 0u);
            tc_commit(&sm.sfull[dr.slot]);
          }
          __syncwarp();
          dr.next(X_NDS);
        }
        if (!ok) break;
        if (elect_one()) tc_commit(&sm.empty[s]);  // the stage's operands are read once these finish
        __syncwarp();
        ring.next(X_NS);
      }
    }
    if (!ok && lane == 0) set_abort(sm, args.dev_status);
  } else if (warp >= X_WEPI0) {
    // warp w reads tensor-memory lanes 32 * (w % 4) .. +31 (its rows) and the
    // 32 tokens of its column block
    const int quarter = warp & 3, cblk = (warp - X_WEPI0) >> 2;
    const int row = quarter * 32 + lane;
    const int col0 = cblk * 32;
    const uint32_t lane_ofs = (uint32_t)(quarter * 32) << 16;
    // the split-tile counters come from the kernels launched just before
    asm volatile("griddepcontrol.wait;" ::: "memory");
    Ring ring{0, 0}, dr{0, 0};
    bool ok = true;
    // y (this thread's row, 32 tokens) of one tile over chunks [kc0, kc1)
    auto run = [&](int tile, int kc0, int kc1, float2 (&y2)[16]) {
      const int64_t n0 = (int64_t)(tile / (int)args.tiles_t) * BM, t0 = (int64_t)(tile % (int)args.tiles_t) * BN;
      const int64_t grow = n0 + row;
#pragma unroll
      for (int j = 0; j < 16; ++j) y2[j] = make_float2(0.0f, 0.0f);
      for (int kc = kc0; kc < kc1 && ok; ++kc) {
        const int s = ring.slot;
        // the stage's scales have landed once its barrier completed (acquire)
        ok = __all_sync(0xffffffffu, !aborted(sm) && mbar_wait(&sm.full[s], (uint32_t)ring.phase));
        if (!ok) break;
        const uint32_t wsw = *(const uint32_t*)&sm.st[s].wsb[row * 2];
        for (int gi = 0; gi < 2 && ok; ++gi) {
          ok = __all_sync(0xffffffffu, mbar_wait(&sm.sfull[dr.slot], (uint32_t)dr.phase));
          if (!ok) break;
          tc_fence_after();
          uint32_t sv[32];
          tmem_ld_x32(tmem + lane_ofs + dr.slot * BN + col0, sv);
          tmem_ld_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.sfree[dr.slot]);  // the slot may be overwritten now
          if (DEBUG && grow < args.n) {
            int32_t* dp = args.sums_dbg + ((t0 + col0) * args.n + grow) * ng + (int64_t)kc * 2 + gi;
            const int64_t dstep = args.n * ng;
#pragma unroll 4
            for (int j = 0; j < 32; ++j, dp += dstep)
              if (t0 + col0 + j < args.t) *dp = (int32_t)sv[j];
          }
          const float wsc = __half2float(__ushort_as_half((unsigned short)(wsw >> (16 * gi))));
          const float2 w2 = make_float2(wsc, wsc);
          const float4* xsg = (const float4*)(sm.st[s].xsb + gi * BN + col0);
#pragma unroll
          for (int j4 = 0; j4 < 8; ++j4) {
            const float4 xv = xsg[j4];
            // |S| < 2^22: the int32 sum converts to FP32 exactly
            const float2 f0 = make_float2(__int2float_rn((int)sv[4 * j4]), __int2float_rn((int)sv[4 * j4 + 1]));
            const float2 f1 =
                make_float2(__int2float_rn((int)sv[4 * j4 + 2]), __int2float_rn((int)sv[4 * j4 + 3]));
            y2[2 * j4] = __ffma2_rn(__fmul2_rn(w2, make_float2(xv.x, xv.y)), f0, y2[2 * j4]);
            y2[2 * j4 + 1] = __ffma2_rn(__fmul2_rn(w2, make_float2(xv.z, xv.w)), f1, y2[2 * j4 + 1]);
          }
          dr.next(X_NDS);
        }
        if (!ok) break;
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty[s]);  // the stage's scales are consumed
        ring.next(X_NS);
      }
    };
    auto store = [&](int tile, const float2 (&y2)[16]) {
      const int64_t n0 = (int64_t)(tile / (int)args.tiles_t) * BM, t0 = (int64_t)(tile % (int)args.tiles_t) * BN;
      const int64_t grow = n0 + row;
      if (grow >= args.n) return;
      const int jmax = (int)min((int64_t)32, args.t - (t0 + col0));
      const int64_t base = (t0 + col0) * args.n + grow;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if (j < jmax) {
          const float v = (j & 1) ? y2[j >> 1].y : y2[j >> 1].x;
          if (args.y_dtype == QLIN_OUT_F32)
            ((float*)args.y)[base + (int64_t)j * args.n] = v;
          else
            ((__nv_bfloat16*)args.y)[base + (int64_t)j * args.n] = __float2bfloat16_rn(v);
        }
      }
    };
    float2 y2[16];
    // full waves: whole tiles
    for (int r = 0; r < rounds && ok; ++r) {
      const int tile = (int)blockIdx.x + r * P;
      run(tile, 0, nchunks, y2);
      if (!ok) break;
      store(tile, y2);
    }
    // the stream-K range: segments of whole tiles, or the first and last tile
    // of the range shared with neighbouring CTAs
    for (int g = it0; SK && g < it1 && ok;) {
      const int tile = dp_tiles + g / nchunks;
      const int kc0 = g - (g / nchunks) * nchunks;
      const int kc1 = min(nchunks, kc0 + (it1 - g));
      g += kc1 - kc0;
      run(tile, kc0, kc1, y2);
      if (!ok) break;
      if (kc0 != 0 || kc1 != nchunks) {
        // a split tile: publish this part ([token][row] FP32, slot 0 for the
        // CTA's first tile, 1 for its last); the warp that arrives last for
        // this block of the tile sums every part in CTA order and writes y
        const int ew = warp - X_WEPI0;
        const int slot = tile == dp_tiles + it0 / nchunks ? 0 : 1;
        float* mine = args.partials + ((int64_t)blockIdx.x * 2 + slot) * (BM * BN) + (int64_t)col0 * BM + row;
#pragma unroll
        for (int j = 0; j < 32; ++j) mine[j * BM] = (j & 1) ? y2[j >> 1].y : y2[j >> 1].x;
        __threadfence();
        __syncwarp();
        int old = 0;
        if (lane == 0) old = atomicAdd(&args.counters[(int64_t)tile * X_NEPI + ew], 1);
        old = __shfl_sync(0xffffffffu, old, 0);
        // the CTAs that own the tile's first and last stream-K iterations
        const int64_t g0 = (int64_t)(tile - dp_tiles) * nchunks;
        const int i_first = (int)(((g0 + 1) * P - 1) / iters);
        const int i_last = (int)(((g0 + nchunks) * P - 1) / iters);
        if (old != i_last - i_first) continue;
        __threadfence();
#pragma unroll
        for (int j = 0; j < 16; ++j) y2[j] = make_float2(0.0f, 0.0f);
        for (int i = i_first; i <= i_last; ++i) {
          const int si = tile == dp_tiles + (int)((int64_t)i * iters / P) / nchunks ? 0 : 1;
          const float* part = args.partials + ((int64_t)i * 2 + si) * (BM * BN) + (int64_t)col0 * BM + row;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            y2[j].x += __ldcg(part + (2 * j) * BM);
            y2[j].y += __ldcg(part + (2 * j + 1) * BM);
          }
        }
      }
      store(tile, y2);
    }
    if (!ok) set_abort(sm, args.dev_status);
  }

  // Every group sum's completion was observed by the epilogue before this
  // point -- unless a wait timed out; then give the tensor core ample time
  // (1 ms) before the tensor memory is released.
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (aborted(sm)) {
      const unsigned long long t0 = global_ns();
      while (global_ns() - t0 < 1000000ull) {
      }
    }
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

// Workspace: xq int8 [T][K] | xs FP32 [T][K/64] | the weights expanded to int8
// [N][K] (each part 256-byte aligned).  A workspace too small for the last
// part runs the kernel that expands the codes in tensor memory instead.
struct A8Ws {
  size_t xq, xs, w8, counters, partials, total, act_total;
  int64_t ncounters;
};
static size_t up256(size_t v) { return (v + 255) / 256 * 256; }
static A8Ws a8_ws(int64_t t, int64_t n, int64_t k, int num_sms) {
  A8Ws L;
  L.xq = 0;
  L.xs = up256((size_t)t * k);
  L.act_total = L.xs + (size_t)t * (k / 64) * sizeof(float);
  L.w8 = up256(L.act_total);
  const int64_t tiles = ((n + BM - 1) / BM) * ((t + BN - 1) / BN);
  L.ncounters = tiles * X_NEPI;
  L.counters = up256(L.w8 + (size_t)n * k);
  L.partials = up256(L.counters + (size_t)L.ncounters * sizeof(int));
  L.total = L.partials + (size_t)(num_sms > 0 ? num_sms : 1) * 2 * BM * BN * sizeof(float);
  return L;
}

size_t gemm_a8_workspace_bytes(int64_t t, int64_t n, int64_t k, int num_sms) {
  return a8_ws(t, n, k, num_sms).total;
}
size_t gemm_a8_act_workspace_bytes(int64_t t, int64_t k) { return a8_ws(t, 0, k, 1).act_total; }

int launch_quantize_act(const uint16_t* x, int64_t t, int64_t k, int8_t* xq, float* xs,
                        const Exec& ex) {
  const int64_t groups = t * (k / 64);
  const int64_t threads = groups * 8;
  int64_t blocks = (threads + 511) / 512;
  // four 512-thread blocks per SM (two are resident at a time): measured
  // faster than one resident wave or than eight blocks per SM
  const int64_t cap = (int64_t)ex.num_sms * 4;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  quantize_act_kernel<<<(unsigned)blocks, 512, 0, ex.stream>>>(x, groups, xq, xs);
  return cuda_status(cudaGetLastError());
}

template <int BITS, bool DEBUG>
static int launch_a8(const CUtensorMap& tm_codes, const CUtensorMap& tm_hib, const CUtensorMap& tm_act,
                     const GemmArgs& args, int grid, const Exec& ex) {
  const size_t smem = sizeof(Smem<BITS>) + 1024;
  const cudaError_t e0 = set_smem_once<gemm_a8_kernel<BITS, DEBUG>>((int)smem);
  if (e0 != cudaSuccess) return cuda_status(e0);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = ex.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_status(cudaLaunchKernelEx(&cfg, gemm_a8_kernel<BITS, DEBUG>, tm_codes, tm_hib, tm_act, args));
}

template <bool DEBUG, bool SK>
static int launch_i8x(const CUtensorMap& tm_w, const CUtensorMap& tm_act, const GemmArgs& args, int grid,
                      const Exec& ex) {
  const size_t smem = sizeof(XSmem) + 1024;
  const cudaError_t e0 = set_smem_once<gemm_i8x_kernel<DEBUG, SK>>((int)smem);
  if (e0 != cudaSuccess) return cuda_status(e0);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(X_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = ex.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_status(cudaLaunchKernelEx(&cfg, gemm_i8x_kernel<DEBUG, SK>, tm_w, tm_act, args));
}

int launch_gemm_a8(const qlin_weights& w, const uint16_t* x, const int8_t* xq, const float* xs,
                   int64_t t, void* y, int y_dtype, uint32_t flags, int32_t* sums_dbg,
                   const Exec& ex) {
  const int64_t n = w.n, k = w.k;
  const A8Ws wl = a8_ws(t, n, k, ex.num_sms);
  // (the expanded-weight kernel counts its (tile, K chunk) steps in 32 bits)
  const int64_t xtiles = ((n + BM - 1) / BM) * ((t + BN - 1) / BN);
  const bool expanded = ex.workspace != nullptr && ex.workspace_bytes >= wl.total &&
                        xtiles * (k / X_BK) < (int64_t)INT32_MAX;
  const int bits = w.fmt == QLIN_Q3_G64 ? 3 : w.fmt == QLIN_Q4_G64 ? 4 : w.fmt == QLIN_Q5_G64 ? 5 : 6;
  int8_t* w8 = expanded ? (int8_t*)((uint8_t*)ex.workspace + wl.w8) : nullptr;
  if (expanded) {
    // the codes as int8 [N][K], once per call (bandwidth-bound)
    const int64_t items = n * (k / 64);
    const int64_t blocks = std::min<int64_t>((items + 255) / 256, (int64_t)ex.num_sms * 16);
    const uint8_t* c = (const uint8_t*)w.codes;
    const uint8_t* h = (const uint8_t*)w.hibits;
    int* cnt = (int*)((uint8_t*)ex.workspace + wl.counters);
    switch (bits) {
      case 3: expand_i8_kernel<3><<<(unsigned)blocks, 256, 0, ex.stream>>>(c, h, n, k, w8, cnt, wl.ncounters); break;
      case 4: expand_i8_kernel<4><<<(unsigned)blocks, 256, 0, ex.stream>>>(c, h, n, k, w8, cnt, wl.ncounters); break;
      case 5: expand_i8_kernel<5><<<(unsigned)blocks, 256, 0, ex.stream>>>(c, h, n, k, w8, cnt, wl.ncounters); break;
      default: expand_i8_kernel<6><<<(unsigned)blocks, 256, 0, ex.stream>>>(c, h, n, k, w8, cnt, wl.ncounters); break;
    }
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_status(e);
  }
  if (x != nullptr) {
    // quantize into the workspace first
    int8_t* wq = (int8_t*)ex.workspace;
    float* wsc = (float*)((uint8_t*)ex.workspace + wl.xs);
    int rc = launch_quantize_act(x, t, k, wq, wsc, ex);
    if (rc != QLIN_OK) return rc;
    xq = wq;
    xs = wsc;
  }
  if (expanded) {
    CUtensorMap tm_w, tm_act;
    int rc = encode_tmap_2d(&tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, w8, (uint64_t)k, (uint64_t)n, (uint64_t)k,
                            128, BM, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;
    rc = encode_tmap_2d(&tm_act, CU_TENSOR_MAP_DATA_TYPE_UINT8, xq, (uint64_t)k, (uint64_t)t, (uint64_t)k,
                        128, BN, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;
    GemmArgs args;
    args.ws = (const __half*)w.scales;
    args.xs = xs;
    args.y = y;
    args.sums_dbg = sums_dbg;
    args.dev_status = ex.dev_status;
    args.n = n;
    args.k = k;
    args.t = t;
    args.tiles_t = (t + BN - 1) / BN;
    args.tiles = args.tiles_t * ((n + BM - 1) / BM);
    args.y_dtype = y_dtype;
    args.partials = (float*)((uint8_t*)ex.workspace + wl.partials);
    args.counters = (int*)((uint8_t*)ex.workspace + wl.counters);
    // stream-K: every SM takes an equal share of the (tile, K chunk) iterations
    const int grid = (int)std::min<int64_t>(args.tiles * (k / X_BK), ex.num_sms);
    // stream-K for the tail only below X_SK_MAX_WAVES full waves
    const bool sk = args.tiles < (int64_t)X_SK_MAX_WAVES * grid;
    if (flags & QLIN_DEBUG_GROUP_SUMS)
      return sk ? launch_i8x<true, true>(tm_w, tm_act, args, grid, ex) : launch_i8x<true, false>(tm_w, tm_act, args, grid, ex);
    return sk ? launch_i8x<false, true>(tm_w, tm_act, args, grid, ex) : launch_i8x<false, false>(tm_w, tm_act, args, grid, ex);
  }
  // code plane: 128-byte swizzled nibble rows, or (Q3) unswizzled 64-byte crumb rows per stage
  const uint64_t crow = (uint64_t)(bits == 3 ? k / 4 : k / 2);
  CUtensorMap tm_codes, tm_hib, tm_act;
  int rc = encode_tmap_2d(&tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, w.codes, crow, (uint64_t)n, crow,
                          bits == 3 ? 64 : 128, BM,
                          bits == 3 ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return rc;
  rc = encode_tmap_2d(&tm_act, CU_TENSOR_MAP_DATA_TYPE_UINT8, xq, (uint64_t)k, (uint64_t)t,
                      (uint64_t)k, 128, BN, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return rc;
  if (bits != 4) {
    // second plane: 32 (bit plane) or 64 (crumb plane) bytes per row per stage
    const uint64_t hrow = (uint64_t)(bits == 6 ? k / 4 : k / 8);
    rc = encode_tmap_2d(&tm_hib, CU_TENSOR_MAP_DATA_TYPE_UINT8, w.hibits, hrow, (uint64_t)n, hrow,
                        bits == 6 ? 64 : 32, BM, CU_TENSOR_MAP_SWIZZLE_NONE);
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
  args.tiles_t = (t + BN - 1) / BN;
  args.tiles = args.tiles_t * ((n + BM - 1) / BM);
  args.y_dtype = y_dtype;
  args.partials = nullptr;
  args.counters = nullptr;
  const bool debug = (flags & QLIN_DEBUG_GROUP_SUMS) != 0;
  const int grid = (int)std::min<int64_t>(args.tiles, ex.num_sms);
  switch (bits) {
    case 3: return debug ? launch_a8<3, true>(tm_codes, tm_hib, tm_act, args, grid, ex)
                         : launch_a8<3, false>(tm_codes, tm_hib, tm_act, args, grid, ex);
    case 4: return debug ? launch_a8<4, true>(tm_codes, tm_hib, tm_act, args, grid, ex)
                         : launch_a8<4, false>(tm_codes, tm_hib, tm_act, args, grid, ex);
    case 5: return debug ? launch_a8<5, true>(tm_codes, tm_hib, tm_act, args, grid, ex)
                         : launch_a8<5, false>(tm_codes, tm_hib, tm_act, args, grid, ex);
    default: return debug ? launch_a8<6, true>(tm_codes, tm_hib, tm_act, args, grid, ex)
                          : launch_a8<6, false>(tm_codes, tm_hib, tm_act, args, grid, ex);
  }
}

}  // namespace qlin
