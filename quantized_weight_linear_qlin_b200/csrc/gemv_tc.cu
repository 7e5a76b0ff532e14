// BF16-route projection on the 5th-generation tensor cores (decode / MTP /
// verify steps, T <= 64): y[T][N] = x[T][K] * W^T with the packed weights
// dequantized on the fly ("Qwen3.8-27B, NInfer int8-prefill artifact for the
// RTX 4090", "What changes": decode keeps the BF16 route; "...NVFP4-
// NInferV3", "How it was created": the FP8 head op over T = 1..33).
//
// Why tensor cores for a bandwidth-bound GEMV: at T >= 2 the CUDA cores cannot
// both unpack the codes and do T FMAs per weight at HBM speed.  Here the CUDA
// cores only unpack; the tcgen05 MMA does the dot products.
//
// One persistent CTA per SM walks a contiguous range of (128-row tile, K-chunk)
// units (stream-K), so every SM streams the same number of weight bytes:
//   warp 0      TMA: 128 rows x 128 bytes of packed codes (+ the Q5 high-bit
//               plane) and the matching activation columns, into a ring of
//               shared-memory stages;
//   warps 4-7   dequantize: thread r owns weight row r; it expands one group's
//               codes to exact BF16 integers (exponent-bias tricks, no
//               conversions) and writes them with tcgen05.st as the MMA's A
//               operand straight into tensor memory (lane r);
//   warp 1      issues tcgen05.mma.kind::f16 (A from tensor memory, B = the
//               activations from shared memory, M = 128, N = T padded to 16)
//               into a fresh FP32 accumulator per quantization group;
//   warps 8-11  epilogue: tcgen05.ld each group's 128 x T sums and apply the
//               group's FP16 scale in FP32 registers (row-scaled FP8 and BF16
//               weights accumulate a whole tile segment in the tensor core).
// Tiles split between two CTAs meet in a workspace; the last CTA to arrive
// sums the parts in a fixed order (deterministic) and writes y.
#include "qlin_internal.cuh"

namespace qlin {
namespace {

constexpr int TC_THREADS = 16 * 32;
constexpr int W_TMA = 0, W_MMA = 1, W_DQ0 = 4, W_EPI0 = 8, W_DQB0 = 12;
constexpr int NA = 4;  // A stages in tensor memory
constexpr int ND = 4;  // accumulator stages in tensor memory
constexpr uint32_t TMEM_COLS = 512;
constexpr int CODES_BYTES = 128 * 128;
constexpr int SMEM_BUDGET = 212992;

template <int FMT>
struct TcT;
template <>
struct TcT<QLIN_Q4_G64> {
  static constexpr int KC = 256, GK = 64, GPC = 4, BOXES = 4;
  static constexpr bool PER_GROUP = true, HIB = false;
};
template <>
struct TcT<QLIN_Q5_G64> {
  static constexpr int KC = 256, GK = 64, GPC = 4, BOXES = 4;
  static constexpr bool PER_GROUP = true, HIB = true;
};
template <>
struct TcT<QLIN_Q8_G32> {
  static constexpr int KC = 128, GK = 32, GPC = 4, BOXES = 2;
  static constexpr bool PER_GROUP = true, HIB = false;
};
template <>
struct TcT<QLIN_FP8_ROW> {
  static constexpr int KC = 128, GK = 64, GPC = 2, BOXES = 2;
  static constexpr bool PER_GROUP = false, HIB = false;
};
template <>
struct TcT<QLIN_BF16> {
  static constexpr int KC = 64, GK = 64, GPC = 1, BOXES = 1;
  static constexpr bool PER_GROUP = false, HIB = false;
};

template <int FMT, int TP>
struct Cfg {
  using Tr = TcT<FMT>;
  static constexpr int X_BYTES = Tr::BOXES * TP * 128;
  static constexpr int HIB_BYTES = Tr::HIB ? 128 * 32 : 0;
  static constexpr int SC_BYTES = Tr::PER_GROUP ? 128 * Tr::GPC * 2 : 0;  // 8 B of scales per row
  static constexpr int TMA_BYTES = CODES_BYTES + X_BYTES + HIB_BYTES;
  static constexpr int STAGE = TMA_BYTES + SC_BYTES;
  static constexpr int NS = (SMEM_BUDGET / STAGE) > 8 ? 8 : (SMEM_BUDGET / STAGE);
  static constexpr int ACOLS = Tr::GK / 2;  // tensor-memory columns of one A stage
  static constexpr size_t SMEM = (size_t)NS * STAGE + 1024 + 512;
};

struct TcArgs {
  const void* scales;
  void* y;
  float* partials;  // [P][2][T][128]
  int* counters;    // [tiles]
  int32_t* dev_status;
  int64_t n, k, t;
  int64_t cpt;      // K-chunks per tile
  int64_t units;    // tiles * cpt
  int y_dtype;
};

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
// low half of v[c]).  `codes` is the 128-byte-swizzled stage tile.
template <int FMT>
__device__ __forceinline__ void dequant_group(const uint8_t* codes, const uint8_t* hib, int r, int gi,
                                              uint32_t* v) {
  if constexpr (FMT == QLIN_Q4_G64 || FMT == QLIN_Q5_G64) {
    const uint4 c0 = *(const uint4*)(codes + sw128_offset(r, 2 * gi));
    const uint4 c1 = *(const uint4*)(codes + sw128_offset(r, 2 * gi + 1));
    const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
    uint32_t h0 = 0, h1 = 0;
    if constexpr (FMT == QLIN_Q5_G64) {
      const uint2 hh = *(const uint2*)(hib + r * 32 + gi * 8);
      h0 = hh.x;
      h1 = hh.y;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        uint32_t m = ((w[j] >> (4 * s)) & 0x000F000Fu) | 0x43004300u;  // 128 + u, exact BF16
        if constexpr (FMT == QLIN_Q5_G64) {
          const uint32_t H = j < 4 ? h0 : h1;
          const int sh = 4 * (j & 3) + s - 4;  // high bits of the pair -> bits 4 and 20
          const uint32_t hs = sh >= 0 ? (H >> sh) : (H << (-sh));
          m |= hs & 0x00100010u;
          v[4 * j + s] = bf16x2_sub(m, 0x43104310u);  // - 144 = -(128 + 16)
        } else {
          v[4 * j + s] = bf16x2_sub(m, 0x43084308u);  // - 136 = -(128 + 8)
        }
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

template <int FMT, int TP>
__global__ void __launch_bounds__(TC_THREADS, 1)
    gemv_tc_kernel(const __grid_constant__ CUtensorMap tm_codes,
                   const __grid_constant__ CUtensorMap tm_hib,
                   const __grid_constant__ CUtensorMap tm_x, TcArgs args) {
  using Tr = TcT<FMT>;
  using C = Cfg<FMT, TP>;
  constexpr int NS = C::NS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* codes_s = base;
  uint8_t* x_s = codes_s + NS * CODES_BYTES;
  uint8_t* hib_s = x_s + NS * C::X_BYTES;
  uint8_t* sc_s = hib_s + NS * C::HIB_BYTES;
  uint64_t* full = (uint64_t*)(sc_s + NS * C::SC_BYTES);
  uint64_t* empty = full + NS;
  uint64_t* a_full = empty + NS;
  uint64_t* a_empty = a_full + NA;
  uint64_t* d_full = a_empty + NA;
  uint64_t* d_empty = d_full + ND;
  uint64_t* drain = d_empty + ND;
  uint32_t* tmem_slot = (uint32_t*)(drain + 1);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  volatile int* fix_slot = (volatile int*)(tmem_slot + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t P = gridDim.x;
  const int64_t U = args.units;
  const int64_t u0 = unit_start(blockIdx.x, U, P), u1 = unit_start(blockIdx.x + 1, U, P);
  const int64_t ng = args.k / Tr::GK;  // groups per row
  const int T = (int)args.t;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1 + 32);             // TMA issue + 32 scale-copy arrivals
      mbar_init(&empty[s], 1 + 2 * 128 + 128);  // MMA commit + both dequant groups + epilogue
    }
    for (int a = 0; a < NA; ++a) {
      mbar_init(&a_full[a], 128);
      mbar_init(&a_empty[a], 1);
    }
    for (int d = 0; d < ND; ++d) {
      mbar_init(&d_full[d], 1);
      mbar_init(&d_empty[d], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == W_MMA) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == W_TMA && lane == 0) {
    tma_prefetch_desc(&tm_codes);
    tma_prefetch_desc(&tm_x);
    if (Tr::HIB) tma_prefetch_desc(&tm_hib);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_a = tmem;
  const uint32_t tmem_d = tmem + NA * C::ACOLS;

  auto abort_now = [&]() {
    *abort_flag = 1;
    report_timeout(args.dev_status);
  };

  if (warp == W_TMA) {
    // lane 0 issues the TMA copies; all 32 lanes copy the stage's group scales
    // (8 bytes per row) with cp.async, tracked by the same barrier.
    int64_t issued = 0;
    for (int64_t u = u0; u < u1; ++u) {
      const int64_t cu = u - u0;
      const int s = (int)(cu % NS);
      if (!__all_sync(0xffffffffu, !*abort_flag && mbar_wait(&empty[s], (uint32_t)(((cu / NS) & 1) ^ 1)))) {
        if (lane == 0) abort_now();
        break;
      }
      const int64_t tile = u / args.cpt, ch = u % args.cpt;
      if (lane == 0) {
        mbar_arrive_expect_tx(&full[s], C::TMA_BYTES);
        tma_load_2d(codes_s + s * CODES_BYTES, &tm_codes, &full[s], (int)(ch * 128), (int)(tile * 128));
        if (Tr::HIB)
          tma_load_2d(hib_s + s * C::HIB_BYTES, &tm_hib, &full[s], (int)(ch * 32), (int)(tile * 128));
#pragma unroll
        for (int b = 0; b < Tr::BOXES; ++b)
          tma_load_2d(x_s + s * C::X_BYTES + b * TP * 128, &tm_x, &full[s],
                      (int)(ch * Tr::KC + b * 64), 0);
      }
      if constexpr (Tr::PER_GROUP) {
        const __half* src = (const __half*)args.scales + ch * Tr::GPC;
        uint8_t* dst = sc_s + s * C::SC_BYTES;
#pragma unroll
        for (int rr = lane; rr < 128; rr += 32) {
          const int64_t row = tile * 128 + rr;
          if (row < args.n) cp_async_8(dst + rr * 8, src + row * ng);
        }
      }
      cp_async_arrive_noinc(&full[s]);
      ++issued;
    }
    if (lane == 0)
      for (int64_t cu = issued > NS ? issued - NS : 0; cu < issued; ++cu)
        mbar_wait(&full[cu % NS], (uint32_t)((cu / NS) & 1));
  } else if (warp == W_MMA) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, TP);
      int64_t G = 0, D = 0;
      for (int64_t u = u0; u < u1 && !*abort_flag; ++u) {
        const int64_t cu = u - u0;
        const int s = (int)(cu % NS);
        if (!mbar_wait(&full[s], (uint32_t)((cu / NS) & 1))) { abort_now(); break; }
        const int64_t ch = u % args.cpt;
        const int gcount = (int)min((int64_t)Tr::GPC, ng - ch * Tr::GPC);
        const bool seg_first = (u == u0) || ch == 0;
        const bool seg_last = (u + 1 == u1) || ((u + 1) % args.cpt == 0);
        const uint32_t xs_base = smem_u32(x_s + s * C::X_BYTES);
        bool ok = true;
        for (int gi = 0; gi < gcount; ++gi, ++G) {
          const int a = (int)(G % NA);
          const bool new_acc = Tr::PER_GROUP || (seg_first && gi == 0);
          const bool close_acc = Tr::PER_GROUP || (seg_last && gi == gcount - 1);
          const int d = (int)(D % ND);
          if (!mbar_wait(&a_full[a], (uint32_t)((G / NA) & 1))) { ok = false; break; }
          if (new_acc && !mbar_wait(&d_empty[d], (uint32_t)(((D / ND) & 1) ^ 1))) { ok = false; break; }
          tc_fence_after();
          const int kofs = gi * Tr::GK;  // K offset of the group inside the chunk
          const uint32_t xaddr = xs_base + (kofs / 64) * TP * 128 + (kofs % 64) * 2;
#pragma unroll
          for (int kk = 0; kk < Tr::GK / 16; ++kk)
            mma_f16_ts(tmem_d + d * TP, tmem_a + a * C::ACOLS + kk * 8, sdesc_k_sw128(xaddr + kk * 32),
                       idesc, (kk > 0 || !new_acc) ? 1u : 0u);
          tc_commit(&a_empty[a]);
          if (close_acc) {
            tc_commit(&d_full[d]);
            ++D;
          }
        }
        if (!ok) { abort_now(); break; }
        tc_commit(&empty[s]);
      }
      tc_commit(drain);
      mbar_wait(drain, 0);
    }
  } else if ((warp >= W_DQ0 && warp < W_DQ0 + 4) || warp >= W_DQB0) {
    // two dequantizing warpgroups take alternate groups (A stages of matching parity)
    const int wg = warp >= W_DQB0 ? 1 : 0;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_ofs = (uint32_t)(quarter * 32) << 16;
    int64_t G = 0;
    for (int64_t u = u0; u < u1; ++u) {
      const int64_t cu = u - u0;
      const int s = (int)(cu % NS);
      if (!__all_sync(0xffffffffu, !*abort_flag && mbar_wait(&full[s], (uint32_t)((cu / NS) & 1)))) {
        abort_now();
        break;
      }
      const int64_t ch = u % args.cpt;
      const int gcount = (int)min((int64_t)Tr::GPC, ng - ch * Tr::GPC);
      const uint8_t* cs = codes_s + s * CODES_BYTES;
      const uint8_t* hs = hib_s + s * C::HIB_BYTES;
      bool ok = true;
      for (int gi = 0; gi < gcount; ++gi, ++G) {
        if ((int)(G & 1) != wg) continue;
        uint32_t v[C::ACOLS];
        dequant_group<FMT>(cs, hs, r, gi, v);
        const int a = (int)(G % NA);
        if (!__all_sync(0xffffffffu, mbar_wait(&a_empty[a], (uint32_t)(((G / NA) & 1) ^ 1)))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if constexpr (C::ACOLS == 32)
          tmem_st_x32(tmem_a + lane_ofs + a * C::ACOLS, v);
        else
          tmem_st_x16(tmem_a + lane_ofs + a * C::ACOLS, v);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&a_full[a]);
      }
      if (!ok) { abort_now(); break; }
      mbar_arrive(&empty[s]);
    }
  } else if (warp >= W_EPI0 && warp < W_EPI0 + 4) {
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int et = threadIdx.x - W_EPI0 * 32;  // 0..127
    const uint32_t lane_ofs = (uint32_t)(quarter * 32) << 16;
    float acc[TP];
#pragma unroll
    for (int t = 0; t < TP; ++t) acc[t] = 0.0f;
    int64_t D = 0;
    bool dead = false;  // after a timed-out wait: skip waits and work, keep the barrier sequence
    for (int64_t u = u0; u < u1; ++u) {
      const int64_t cu = u - u0;
      const int s = (int)(cu % NS);
      const int64_t tile = u / args.cpt, ch = u % args.cpt;
      const int64_t row = tile * 128 + r;
      const int gcount = (int)min((int64_t)Tr::GPC, ng - ch * Tr::GPC);
      const bool seg_first = (u == u0) || ch == 0;
      const bool seg_last = (u + 1 == u1) || ((u + 1) % args.cpt == 0);
      if (seg_first) {
#pragma unroll
        for (int t = 0; t < TP; ++t) acc[t] = 0.0f;
      }
      dead = dead || __any_sync(0xffffffffu, *abort_flag != 0);
      // the stage's scales have landed once its barrier completed (acquire)
      if (!dead && !__all_sync(0xffffffffu, mbar_wait(&full[s], (uint32_t)((cu / NS) & 1)))) {
        dead = true;
        abort_now();
      }
      const __half* sc_row = (const __half*)(sc_s + s * C::SC_BYTES) + r * Tr::GPC;
      for (int gi = 0; gi < gcount; ++gi) {
        const bool close_acc = Tr::PER_GROUP || (seg_last && gi == gcount - 1);
        if (!close_acc) continue;
        const int d = (int)(D % ND);
        const uint32_t dpar = (uint32_t)((D / ND) & 1);
        ++D;
        if (dead) continue;
        float sc = 1.0f;
        if constexpr (Tr::PER_GROUP) sc = __half2float(sc_row[gi]);
        if (!__all_sync(0xffffffffu, mbar_wait(&d_full[d], dpar))) {
          dead = true;
          abort_now();
          continue;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < TP; c += 16) {
          if (c < T) {
            uint32_t vr[16];
            tmem_ld_x16(tmem_d + lane_ofs + d * TP + c, vr);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j) acc[c + j] = fmaf(sc, __uint_as_float(vr[j]), acc[c + j]);
          }
        }
        tc_fence_before();
        mbar_arrive(&d_empty[d]);
      }
      if (!dead) mbar_arrive(&empty[s]);
      if (!seg_last) continue;
      // ---- the CTA's part of this tile is complete
      float rs = 1.0f;
      if constexpr (FMT == QLIN_FP8_ROW) {
        if (row < args.n) rs = __bfloat162float(((const __nv_bfloat16*)args.scales)[row]);
      }
      const int64_t tstart = tile * args.cpt, tend = tstart + args.cpt;
      const bool whole = u0 <= tstart && u1 >= tend;
      if (whole) {
        if (!dead && row < args.n) {
#pragma unroll
          for (int t = 0; t < TP; ++t) {
            if (t < T) {
              if (args.y_dtype == QLIN_OUT_F32)
                ((float*)args.y)[(int64_t)t * args.n + row] = acc[t] * rs;
              else
                ((__nv_bfloat16*)args.y)[(int64_t)t * args.n + row] = __float2bfloat16_rn(acc[t] * rs);
            }
          }
        }
        continue;
      }
      // split tile: publish this part, the last contributor reduces
      const int slot = (tile == u0 / args.cpt) ? 0 : 1;
      float* mine = args.partials + ((int64_t)blockIdx.x * 2 + slot) * T * 128;
      if (!dead) {
#pragma unroll
        for (int t = 0; t < TP; ++t)
          if (t < T) mine[t * 128 + et] = acc[t];
      }
      __threadfence();
      asm volatile("bar.sync 2, 128;" ::: "memory");
      if (et == 0) *fix_slot = dead ? -1 : atomicAdd(&args.counters[tile], 1);
      asm volatile("bar.sync 2, 128;" ::: "memory");
      const int old = *fix_slot;
      const int64_t i_first = unit_owner(tstart, U, P), i_last = unit_owner(tend - 1, U, P);
      if (old == (int)(i_last - i_first)) {
        __threadfence();
#pragma unroll
        for (int t = 0; t < TP; ++t) acc[t] = 0.0f;
        for (int64_t i = i_first; i <= i_last; ++i) {
          const int si = (tile == unit_start(i, U, P) / args.cpt) ? 0 : 1;
          const float* part = args.partials + (i * 2 + si) * T * 128;
#pragma unroll
          for (int t = 0; t < TP; ++t)
            if (t < T) acc[t] += __ldcg(part + t * 128 + et);
        }
        if (row < args.n) {
#pragma unroll
          for (int t = 0; t < TP; ++t) {
            if (t < T) {
              if (args.y_dtype == QLIN_OUT_F32)
                ((float*)args.y)[(int64_t)t * args.n + row] = acc[t] * rs;
              else
                ((__nv_bfloat16*)args.y)[(int64_t)t * args.n + row] = __float2bfloat16_rn(acc[t] * rs);
            }
          }
        }
        if (et == 0) args.counters[tile] = 0;  // leave the counter ready for the next call
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == W_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

template <int FMT>
int64_t chunk_k() {
  return TcT<FMT>::KC;
}

int64_t tc_chunk_k(int fmt) {
  switch (fmt) {
    case QLIN_Q4_G64: return TcT<QLIN_Q4_G64>::KC;
    case QLIN_Q5_G64: return TcT<QLIN_Q5_G64>::KC;
    case QLIN_Q8_G32: return TcT<QLIN_Q8_G32>::KC;
    case QLIN_FP8_ROW: return TcT<QLIN_FP8_ROW>::KC;
    default: return TcT<QLIN_BF16>::KC;
  }
}

int tpad_of(int64_t t) { return t <= 16 ? 16 : t <= 32 ? 32 : t <= 48 ? 48 : 64; }

template <int FMT, int TP>
int launch_tp(const CUtensorMap& mc, const CUtensorMap& mh, const CUtensorMap& mx, const TcArgs& a,
              int grid, cudaStream_t st) {
  using C = Cfg<FMT, TP>;
  static_assert(C::NS >= 2, "pipeline needs two stages");
  static_assert(NA * C::ACOLS + ND * TP <= (int)TMEM_COLS, "tensor memory budget");
  auto kern = gemv_tc_kernel<FMT, TP>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
  kern<<<grid, TC_THREADS, C::SMEM, st>>>(mc, mh, mx, a);
  return cuda_status(cudaGetLastError());
}

template <int FMT>
int launch_fmt(int tp, const CUtensorMap& mc, const CUtensorMap& mh, const CUtensorMap& mx,
               const TcArgs& a, int grid, cudaStream_t st) {
  switch (tp) {
    case 16: return launch_tp<FMT, 16>(mc, mh, mx, a, grid, st);
    case 32: return launch_tp<FMT, 32>(mc, mh, mx, a, grid, st);
    case 48: return launch_tp<FMT, 48>(mc, mh, mx, a, grid, st);
    default: return launch_tp<FMT, 64>(mc, mh, mx, a, grid, st);
  }
}

}  // namespace

// Q4/Q5 need whole 256-column chunks (8-byte scale rows per chunk), Q8 whole
// 128-column chunks; other shapes take the CUDA-core kernel.
bool gemv_tc_supported(const qlin_weights& w, int64_t t) {
  if (t < 1 || t > 64) return false;
  if ((w.fmt == QLIN_Q4_G64 || w.fmt == QLIN_Q5_G64) && w.k % 256 != 0) return false;
  if (w.fmt == QLIN_Q8_G32 && w.k % 128 != 0) return false;
  return true;
}

size_t gemv_tc_workspace_bytes(const qlin_weights& w, int64_t t, int num_sms) {
  const int64_t tiles = (w.n + 127) / 128;
  const size_t counters = ((size_t)tiles * sizeof(int) + 255) / 256 * 256;
  return counters + (size_t)num_sms * 2 * t * 128 * sizeof(float);
}

int launch_gemv_tc(const qlin_weights& w, const uint16_t* x, int64_t t, void* y, int y_dtype,
                   const Exec& ex) {
  const int64_t tiles = (w.n + 127) / 128;
  const int64_t kc = tc_chunk_k(w.fmt);
  const int64_t cpt = (w.k + kc - 1) / kc;
  const int64_t units = tiles * cpt;
  const int grid = (int)std::min<int64_t>(ex.num_sms, units);
  const int tp = tpad_of(t);
  const int64_t row_bytes = w.fmt == QLIN_Q4_G64 || w.fmt == QLIN_Q5_G64 ? w.k / 2
                            : w.fmt == QLIN_BF16                      ? w.k * 2
                                                                      : w.k;
  CUtensorMap mc, mh, mx;
  int rc = encode_tmap_2d(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, w.codes, (uint64_t)row_bytes,
                          (uint64_t)w.n, (uint64_t)row_bytes, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return rc;
  rc = encode_tmap_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, (uint64_t)w.k, (uint64_t)t,
                      (uint64_t)w.k * 2, 64, (uint32_t)tp, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return rc;
  if (w.fmt == QLIN_Q5_G64) {
    rc = encode_tmap_2d(&mh, CU_TENSOR_MAP_DATA_TYPE_UINT8, w.hibits, (uint64_t)(w.k / 8),
                        (uint64_t)w.n, (uint64_t)(w.k / 8), 32, 128, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (rc) return rc;
  } else {
    mh = mc;
  }
  TcArgs a;
  a.scales = w.scales;
  a.y = y;
  const size_t counters = ((size_t)tiles * sizeof(int) + 255) / 256 * 256;
  a.counters = (int*)ex.workspace;
  a.partials = (float*)((uint8_t*)ex.workspace + counters);
  a.dev_status = ex.dev_status;
  a.n = w.n;
  a.k = w.k;
  a.t = t;
  a.cpt = cpt;
  a.units = units;
  a.y_dtype = y_dtype;
  switch (w.fmt) {
    case QLIN_Q4_G64: return launch_fmt<QLIN_Q4_G64>(tp, mc, mh, mx, a, grid, ex.stream);
    case QLIN_Q5_G64: return launch_fmt<QLIN_Q5_G64>(tp, mc, mh, mx, a, grid, ex.stream);
    case QLIN_Q8_G32: return launch_fmt<QLIN_Q8_G32>(tp, mc, mh, mx, a, grid, ex.stream);
    case QLIN_FP8_ROW: return launch_fmt<QLIN_FP8_ROW>(tp, mc, mh, mx, a, grid, ex.stream);
    default: return launch_fmt<QLIN_BF16>(tp, mc, mh, mx, a, grid, ex.stream);
  }
}

}  // namespace qlin
