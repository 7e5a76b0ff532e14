// BF16-route projection of FP8-row and Q8 group-32 weights on the
// 5th-generation tensor cores, 1 <= T <= 64 tokens (decode / MTP / verify
// steps and the output head): y[T][N] = x[T][K] * W^T with the weights
// dequantized on the fly ("Qwen3.8-27B, NInfer int8-prefill artifact for the
// RTX 4090", "What changes": decode keeps the BF16 route and is bandwidth
// bound; "...NVFP4-NInferV3", "How it was created": the head op, row-FP8 or
// Q8 group-32, over T).
//
// Operands.  The weight's scale is folded into the MMA's A operand:
//   Q8:  A[r][k] = FP16_rn(q[r][k] * s[r][g]) from one packed half2 multiply
//        of the exact integer code by the stored FP16 group scale (relative
//        error <= 2^-11, exact when the product is an FP16 subnormal: every
//        FP16 value is a multiple of 2^-24);
//   FP8: A[r][k] = the E4M3 value, exact in FP16; the row scale multiplies the
//        finished sum.
// The activations enter as FP16 too, scaled per token by a power of two 2^e_t
// chosen so that the token's largest magnitude lies in [2^14, 2^15): every
// BF16 value within 2^-31 of that maximum is exact in FP16.  The scaling is
// undone on the output (exact).  So one FP32 tensor-memory accumulator per
// issuer spans the whole of a CTA's part of a tile: no per-group accumulator,
// no per-group epilogue.
//
// Rows whose FP16 group scale could overflow FP16 in q * s (|s| > 511.75:
// weights beyond ~65,000 in magnitude) are recomputed exactly on the CUDA
// cores by the epilogue (never at the workloads of the pages, but the result
// stays correct for any input).
//
// One persistent CTA per SM walks a contiguous range of units (a unit is one
// 128-row tile x 256 columns, 32 KB of codes), so every SM streams the same
// number of weight bytes (stream-K):
//   warp 0      TMA: the unit's codes (two 128-byte-wide boxes, 128-byte
//               swizzle), its group scales (one 16-byte box per row) and the
//               FP16 activation columns into a ring of shared-memory stages.
//               The codes of the first stages are requested before the
//               activation conversion has finished (programmatic dependent
//               launch);
//   warps 4..19 four warpgroups; warpgroup g expands chunk g (64 columns) of
//               every unit: thread = weight row, FP16 pairs written with
//               tcgen05.st into one of the warpgroup's A slots in tensor
//               memory; in rotation one warpgroup also writes out each finished
//               segment (accumulators double-buffered where tensor memory
//               allows, so the next segment's MMAs run meanwhile);
//   warps 1, 2  issuer i issues the tcgen05.mma.kind::f16 of chunks 2i, 2i+1
//               (A in tensor memory, B = the activations in shared memory,
//               M = 128, N = T rounded up to 16) into its own accumulator.  One
//               thread issues an MMA only every ~48 cycles (its own latency),
//               while the tensor pipe needs N/2 cycles for one, so the
//               expansion never waits for a single issuing thread.
// Tiles split between CTAs meet in the workspace; the last CTA to arrive sums
// the parts in CTA order (deterministic) and writes y.
#include "qlin_gemv_common.cuh"

namespace qlin {
namespace {
using namespace gemv;

constexpr uint32_t F_TMEM_COLS = 512;
constexpr int F_SMEM_BUDGET = 225 * 1024;
// Warp roles: 0 producer, 1..2 MMA issuers, 4..19 four dequantizing
// warpgroups.  Warpgroup g always expands chunk g (a quarter of the unit's K
// columns) of every unit, and the epilogue of every fourth segment; issuer i
// issues the MMAs of chunks 2i and 2i + 1 into its own accumulator.  One
// thread issues an MMA only every ~48 cycles (its own issue latency) while the
// tensor pipe needs just N/2 cycles for an M = 128, K = 16 MMA, so two issuers
// keep it fed, and the expansion never waits for an issuing thread.  Twenty
// warps leave 96 registers per thread.
constexpr int F_NDQ = 4;                       // dequantizing warpgroups = chunks per unit
constexpr int F_CPU = F_NDQ;
constexpr int F_NISS = 2;                      // MMA issuers (two chunks each)
constexpr int F_NAW_MAX = 2;                   // A slots per warpgroup where tensor memory allows
constexpr int FW_PROD = 0, FW_ISS0 = 1, FW_DQ0 = 4;
constexpr int F_THREADS = (FW_DQ0 + 4 * F_NDQ) * 32;

// Per format: K elements per 128-byte code box, group size, scale kind, and
// (Q8) the largest FP16 scale bit pattern for which every q * s stays finite.
template <int FMT>
struct FT;
template <>
struct FT<QLIN_Q8_G32> {
  static constexpr int E128 = 128, GK = 32;
  static constexpr bool PER_GROUP = true;
  static constexpr uint32_t S_LIMIT = 0x5FFF;  // 511.75: 128 * 511.75 <= 65504
};
template <>
struct FT<QLIN_FP8_ROW> {
  static constexpr int E128 = 128, GK = 64;
  static constexpr bool PER_GROUP = false;
};
constexpr int up1k(int v) { return (v + 1023) / 1024 * 1024; }

template <int FMT, int TP, int UB>
struct FLayout {
  using Tr = FT<FMT>;
  static constexpr int KC = UB * Tr::E128;              // K columns per unit
  static constexpr int XBOXES = KC / 64;                // activation boxes (64 columns x TP rows)
  static constexpr int X_BYTES = XBOXES * TP * 128;
  static constexpr int GPC = Tr::PER_GROUP ? KC / Tr::GK : 0;  // scale groups per unit
  // one TMA box of 8 FP16 scales (16 bytes) per row: the unit's groups
  static constexpr int SC_ROW = Tr::PER_GROUP ? 16 : 0;
  static constexpr int SC_BYTES = 128 * SC_ROW;
  static constexpr int TMA_BYTES = UB * BOX_BYTES + X_BYTES + SC_BYTES;
  static constexpr int OFF_X = UB * BOX_BYTES;
  static constexpr int OFF_SC = OFF_X + up1k(X_BYTES);
  static constexpr int STAGE = OFF_SC + up1k(SC_BYTES);
  static constexpr int NS = (F_SMEM_BUDGET / STAGE) > 8 ? 8 : (F_SMEM_BUDGET / STAGE);
  static constexpr int CHUNK_K = KC / F_CPU;             // K columns of one chunk (64)
  static constexpr int A_COLS = CHUNK_K / 2;             // tensor-memory columns of its FP16 pairs
};

template <int FMT, int TP>
struct FCfg {
  // two code boxes per unit while three stages still fit, else one
  static constexpr int UB = FLayout<FMT, TP, 2>::NS >= 3 ? 2 : 1;
  using L = FLayout<FMT, TP, UB>;
  static_assert(L::NS >= 2, "pipeline needs two stages");
  static_assert(L::CHUNK_K % 64 == 0, "a chunk holds whole 64-column halves");
  static constexpr size_t SMEM = (size_t)L::NS * L::STAGE + 1024 + 512;
  // tensor memory: accumulators [buffer][warpgroup] of TP columns, then two A
  // slots per warpgroup; two accumulator buffers (the epilogue drains one
  // segment while the next is computed) where they fit
  static constexpr int NACC = F_NISS;
  static constexpr int NAW = 2 * NACC * TP + F_NDQ * F_NAW_MAX * L::A_COLS <= (int)F_TMEM_COLS ? F_NAW_MAX : 1;
  static constexpr int A_TOTAL = F_NDQ * NAW * L::A_COLS;
  static constexpr int NB = 2 * NACC * TP + A_TOTAL <= (int)F_TMEM_COLS ? 2 : 1;
  static constexpr int A0 = NB * NACC * TP;
  static_assert(A0 + A_TOTAL <= (int)F_TMEM_COLS, "tensor memory budget");
};

struct FArgs {
  const void* scales;      // FP16 group scales (Q8) or BF16 row scales (FP8)
  const uint8_t* codes;    // the codes, read again only by the exact CUDA-core
                           //   path of overflowing rows
  const uint16_t* x;       // the BF16 activations (same)
  const float* inv;        // per token 2^-e_t (NULL: activations used unscaled)
  void* y;
  float* partials;         // [P][2][T][128]
  int* counters;           // [tiles]
  int32_t* dev_status;
  int64_t n, k, t;
  int64_t cpt;             // units per tile
  int64_t units;           // tiles * cpt
  int y_dtype;
};

__device__ __forceinline__ uint32_t h2_sub(uint32_t a, __half2 b) {
  const __half2 r = __hsub2(*(const __half2*)&a, b);
  return *(const uint32_t*)&r;
}
__device__ __forceinline__ uint32_t h2_mul(uint32_t a, __half2 b) {
  const __half2 r = __hmul2_rn(*(const __half2*)&a, b);
  return *(const uint32_t*)&r;
}
__device__ __forceinline__ __half2 h2_const(uint32_t bits) { return *(const __half2*)&bits; }
__device__ __forceinline__ uint32_t e4m3x2_to_h2(uint32_t two_bytes) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)two_bytes, __NV_E4M3);
  return (uint32_t)h.x | ((uint32_t)h.y << 16);
}

// Two 32-element Q8 groups (64 elements, 32 pairs) of row r: units u0, u0+1
// hold group 0, u0+2, u0+3 group 1.
__device__ __forceinline__ void dq_q8(const uint8_t* box, int r, int u0, __half2 s2a, __half2 s2b,
                                      uint32_t* v) {
  const __half2 off = h2_const(0x64806480u);  // 1024 + 128
#pragma unroll
  for (int uq = 0; uq < 4; ++uq) {
    const uint4 c = *(const uint4*)(box + sw128_offset(r, u0 + uq));
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
    const __half2 s2 = uq < 2 ? s2a : s2b;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t xw = w[j] ^ 0x80808080u;  // offset-binary bytes q + 128
      // [b0, 0x64, b1, 0x64] = FP16 (1024 + u0, 1024 + u1), exact
      const uint32_t p0 = __byte_perm(xw, 0x64u, 0x4140);
      const uint32_t p1 = __byte_perm(xw, 0x64u, 0x4342);
      v[8 * uq + 2 * j] = h2_mul(h2_sub(p0, off), s2);
      v[8 * uq + 2 * j + 1] = h2_mul(h2_sub(p1, off), s2);
    }
  }
}

// 64 E4M3 codes of row r (units u0..u0+3) widened to FP16 pairs (exact).
__device__ __forceinline__ void dq_fp8(const uint8_t* box, int r, int u0, uint32_t* v) {
#pragma unroll
  for (int uq = 0; uq < 4; ++uq) {
    const uint4 c = *(const uint4*)(box + sw128_offset(r, u0 + uq));
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[8 * uq + 2 * j] = e4m3x2_to_h2(w[j] & 0xFFFFu);
      v[8 * uq + 2 * j + 1] = e4m3x2_to_h2(w[j] >> 16);
    }
  }
}

__device__ __forceinline__ __half2 h2_bcast(uint16_t h) { return __half2half2(*(const __half*)&h); }

// Integer code of element e of row `row` (Q8: two's complement bytes).
__device__ __forceinline__ int code_at(const FArgs& a, int64_t row, int64_t e) {
  return (int)(int8_t)__ldg(a.codes + row * a.k + e);
}

// Does any group scale of `row` over columns [k0, k1) exceed the format's
// FP16-safe limit (so that q * s could overflow FP16)?
template <int FMT>
__device__ __forceinline__ bool row_overflows(const FArgs& a, int64_t row, int64_t k0, int64_t k1) {
  using Tr = FT<FMT>;
  if constexpr (!Tr::PER_GROUP) {
    return false;
  } else {
    // K is a whole number of units, so a row's scales and the segment's first
    // scale are 8-byte aligned: four scales per load, eight loads in flight
    const int64_t ng = a.k / Tr::GK;
    const uint2* s = (const uint2*)((const uint16_t*)a.scales + row * ng + k0 / Tr::GK);
    const int n4 = (int)((k1 - k0) / Tr::GK / 4);
    uint32_t mx = 0;
    int i = 0;
    for (; i + 8 <= n4; i += 8) {
      uint2 v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = __ldg(s + i + j);
#pragma unroll
      for (int j = 0; j < 8; ++j) mx = max(mx, __vmaxu2(v[j].x & 0x7FFF7FFFu, v[j].y & 0x7FFF7FFFu));
    }
    for (; i < n4; ++i) {
      const uint2 v = __ldg(s + i);
      mx = max(mx, __vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu));
    }
    mx = max(mx & 0xFFFFu, mx >> 16);
    return mx > Tr::S_LIMIT;
  }
}

// The exact CUDA-core result of `row` over columns [k0, k1) for token t:
// sum_g s_g * sum_{k in g} q * x in FP32 (BF16 x, exact products).
template <int FMT>
__device__ float row_dot_exact(const FArgs& a, int64_t row, int64_t k0, int64_t k1, int t) {
  using Tr = FT<FMT>;
  const int64_t ng = a.k / Tr::GK;
  const __half* s = (const __half*)a.scales + row * ng;
  const uint16_t* xr = a.x + (int64_t)t * a.k;
  float acc = 0.0f;
  for (int64_t g0 = k0; g0 < k1; g0 += Tr::GK) {
    float part = 0.0f;
    for (int64_t e = g0; e < g0 + Tr::GK; ++e)
      part = fmaf((float)code_at(a, row, e), __uint_as_float((uint32_t)__ldg(xr + e) << 16), part);
    acc = fmaf(__half2float(s[g0 / Tr::GK]), part, acc);
  }
  return acc;
}

template <int FMT, int TP>
__global__ void __launch_bounds__(F_THREADS, 1)
    gemv_f16_kernel(const __grid_constant__ CUtensorMap tm_codes,
                    const __grid_constant__ CUtensorMap tm_x,
                    const __grid_constant__ CUtensorMap tm_sc, FArgs args) {
  using Tr = FT<FMT>;
  using C = FCfg<FMT, TP>;
  using L = typename C::L;
  constexpr int NS = L::NS, UB = C::UB, KC = L::KC, CK = L::CHUNK_K;
  constexpr int NACC = C::NACC, NB = C::NB, NAW = C::NAW;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* full = (uint64_t*)(base + NS * L::STAGE);
  uint64_t* empty = full + NS;
  uint64_t* a_full = empty + NS;               // [F_NDQ][NAW]: slot written by its warpgroup
  uint64_t* a_free = a_full + F_NDQ * NAW;     // [F_NDQ][NAW]: slot read by the MMAs
  uint64_t* acc_full = a_free + F_NDQ * NAW;   // [2]
  uint64_t* acc_empty = acc_full + 2;          // [2]
  uint32_t* tmem_slot = (uint32_t*)(acc_empty + 2);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  volatile int* fix_slot = (volatile int*)(tmem_slot + 2);  // [F_NDQ]
  auto stage = [&](int s) { return base + s * L::STAGE; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t P = gridDim.x;
  const int64_t U = args.units;
  const int64_t u0 = unit_start(blockIdx.x, U, P), u1 = unit_start(blockIdx.x + 1, U, P);
  const int T = (int)args.t;
  const int cpt = (int)args.cpt;
  const int nunits = (int)(u1 - u0);
  const int tile0 = (int)(u0 / cpt), ch0 = (int)(u0 % cpt);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);                             // the TMA issue (bytes tracked)
      mbar_init(&empty[s], NACC);                         // one MMA commit per issuer and unit
    }
    for (int j = 0; j < F_NDQ * NAW; ++j) {
      mbar_init(&a_full[j], 4);  // the warpgroup's four warps
      mbar_init(&a_free[j], 1);  // the issuer's commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], NACC);
      mbar_init(&acc_empty[b], 4);  // the four warps of the segment's epilogue warpgroup
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == FW_ISS0) {
    tmem_alloc(tmem_slot, F_TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == FW_PROD && lane == 0) {
    tma_prefetch_desc(&tm_codes);
    tma_prefetch_desc(&tm_x);
    if (Tr::PER_GROUP) tma_prefetch_desc(&tm_sc);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto abort_now = [&]() {
    *abort_flag = 1;
    report_timeout(args.dev_status);
  };

  if (warp == FW_PROD) {
    // ---- producer.  The codes of the first stages go out before the wait for
    // the activation conversion (programmatic dependent launch); their
    // activation boxes follow once it has completed.
    const uint64_t pol_w = l2_evict_first(), pol_x = l2_evict_last();  // codes stream once; x serves every CTA
    const int npre = nunits < NS ? nunits : NS;
    auto issue_x = [&](int s, int ch) {
#pragma unroll
      for (int b = 0; b < L::XBOXES; ++b)
        tma_load_2d_hint(stage(s) + L::OFF_X + b * TP * 128, &tm_x, &full[s], ch * KC + b * 64, 0, pol_x);
    };
    Ring ring{0, 0};
    int tile = tile0, ch = ch0;
    int issued = 0;
    for (int cu = 0; cu < nunits; ++cu) {
      const int s = ring.slot;
      if (cu >= NS &&
          !__all_sync(0xffffffffu, !*abort_flag && mbar_wait(&empty[s], (uint32_t)(ring.phase ^ 1)))) {
        if (lane == 0) abort_now();
        break;
      }
      uint8_t* st = stage(s);
      if (elect_one()) {
        mbar_arrive_expect_tx(&full[s], L::TMA_BYTES);
#pragma unroll
        for (int b = 0; b < UB; ++b)
          tma_load_2d_hint(st + b * BOX_BYTES, &tm_codes, &full[s], (ch * UB + b) * 128, tile * 128, pol_w);
        if (Tr::PER_GROUP) tma_load_2d_hint(st + L::OFF_SC, &tm_sc, &full[s], (ch * L::GPC) & ~7, tile * 128, pol_w);
        if (cu >= npre) issue_x(s, ch);
      }
      __syncwarp();
      ++issued;
      if (cu == npre - 1) {
        asm volatile("griddepcontrol.wait;" ::: "memory");
        if (elect_one()) {
          int chx = ch0;
          for (int i = 0; i < npre; ++i) {
            issue_x(i, chx);
            if (++chx == cpt) chx = 0;
          }
        }
        __syncwarp();
      }
      ring.next(NS);
      if (++ch == cpt) {
        ch = 0;
        ++tile;
      }
    }
    // let every copy in flight land before the CTA can leave
    if (lane == 0)
      for (int cu = issued > NS ? issued - NS : 0; cu < issued; ++cu)
        mbar_wait(&full[cu % NS], (uint32_t)((cu / NS) & 1));
  } else if (warp >= FW_ISS0 && warp < FW_ISS0 + F_NISS) {
    // ---- MMA issue: issuer i takes chunks 2i and 2i + 1 of every unit into
    // its own accumulator.  The whole warp runs the loop; one elected lane
    // issues each tcgen05 instruction.
    const int i = warp - FW_ISS0;
    const uint32_t idesc = idesc_f16(128, TP);
    bool ok = true;
    Ring ring{0, 0};
    int ch = ch0, seg = 0;
    for (int cu = 0; cu < nunits && ok; ++cu) {
      const int s = ring.slot;
      const bool seg_first = cu == 0 || ch == 0;
      const bool seg_last = cu + 1 == nunits || ch == cpt - 1;
      const int b = NB == 2 ? (seg & 1) : 0;
      const uint32_t use_b = (uint32_t)(NB == 2 ? (seg >> 1) : seg);
      ok = __all_sync(0xffffffffu, !*abort_flag && mbar_wait(&full[s], (uint32_t)ring.phase));
      if (ok && seg_first) ok = __all_sync(0xffffffffu, mbar_wait(&acc_empty[b], (use_b & 1u) ^ 1u));
      if (!ok) break;
      tc_fence_after();
      const uint32_t d = tmem + (b * NACC + i) * TP;
      const uint32_t xs = smem_u32(stage(s) + L::OFF_X);
      const int slot = cu % NAW;
      const uint32_t use = (uint32_t)(cu / NAW);
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int g = 2 * i + q;  // the chunk's warpgroup
        const int j = g * NAW + slot;
        ok = __all_sync(0xffffffffu, mbar_wait(&a_full[j], use & 1u) && !*abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint32_t a = tmem + C::A0 + j * L::A_COLS;
        // the chunk's activation columns: boxes (g CK + 16 kk) / 64 of the stage
        const uint64_t xd = sdesc_k_sw128(xs + (g * CK / 64) * TP * 128);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < CK / 16; ++kk) {
            const uint32_t off = ((kk * 16) / 64) * TP * 128 + ((kk * 16) % 64) * 2;  // bytes
            mma_f16_ts(d, a + kk * 8, xd + (off >> 4), idesc, (seg_first && q == 0 && kk == 0) ? 0u : 1u);
          }
          tc_commit(&a_free[j]);  // the A slot may be rewritten once these complete
        }
        __syncwarp();
      }
      if (!ok) break;
      if (elect_one()) {
        tc_commit(&empty[s]);  // this issuer's reads of the stage are done
        if (seg_last) tc_commit(&acc_full[b]);
      }
      __syncwarp();
      if (seg_last) ++seg;
      ring.next(NS);
      if (++ch == cpt) ch = 0;
    }
    if (!ok && lane == 0) abort_now();
  } else if (warp >= FW_DQ0) {
    // ---- dequantize (warpgroup g takes chunk g, K columns [g CK, (g+1) CK),
    // of every unit: thread = weight row, FP16 (q * s) pairs written with
    // tcgen05.st into the warpgroup's A slots in turn) and, in rotation, the
    // epilogue of a finished segment (warpgroup seg % 4).
    const int g = (warp - FW_DQ0) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int et = r;  // epilogue thread = row of the tile
    const uint32_t lane_ofs = (uint32_t)(quarter * 32) << 16;
    bool dead = false;
    bool dep_done = false;  // griddepcontrol.wait passed (args.inv is written)
    Ring ring{0, 0};
    int tile = tile0, ch = ch0, seg = 0, seg_ch0 = ch0;
    for (int cu = 0; cu < nunits; ++cu) {
      const int s = ring.slot;
      const bool seg_last = cu + 1 == nunits || ch == cpt - 1;
      const int cur_tile = tile, cur_ch = ch;
      {
        const int slot = cu % NAW;
        const uint32_t use = (uint32_t)(cu / NAW);
        const int j = g * NAW + slot;
        if (!dead && !__all_sync(0xffffffffu, !*abort_flag && mbar_wait(&full[s], (uint32_t)ring.phase))) {
          dead = true;
          if (lane == 0) abort_now();
        }
        if (!dead) {
          const uint8_t* st = stage(s);
          const uint16_t* sc = (const uint16_t*)(st + L::OFF_SC) + r * 8 + ((ch * L::GPC) & 7);
          const uint32_t a_addr = tmem + lane_ofs + C::A0 + j * L::A_COLS;
          // each 64-column half in registers of its own: tcgen05.st reads its
          // source registers after issue
          uint32_t v[CK / 64][32];
#pragma unroll
          for (int h = 0; h < CK / 64; ++h) {  // 64-column halves of the chunk
            const int kb = g * CK + h * 64;  // K offset inside the unit
            if constexpr (FMT == QLIN_Q8_G32) {
              const int box = kb / 128, u = (kb % 128) / 16;
              dq_q8(st + box * BOX_BYTES, r, u, h2_bcast(sc[kb / 32]), h2_bcast(sc[kb / 32 + 1]), v[h]);
            } else {  // FP8_ROW
              const int box = kb / 128, u = (kb % 128) / 16;
              dq_fp8(st + box * BOX_BYTES, r, u, v[h]);
            }
            if (h == 0) {
              // the MMAs that last read this slot are complete
              if (!__all_sync(0xffffffffu, mbar_wait(&a_free[j], (use & 1u) ^ 1u))) {
                dead = true;
                if (lane == 0) abort_now();
                break;
              }
              tc_fence_after();
            }
            tmem_st_x32(a_addr + h * 32, v[h]);
          }
          if (!dead) {
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&a_full[j]);
          }
        }
      }
      ring.next(NS);
      if (++ch == cpt) {
        ch = 0;
        ++tile;
      }
      if (!seg_last) continue;
      // ---- the segment (units of tile cur_tile, K columns [seg_k0, seg_k1))
      // is complete in the accumulators; warpgroup seg % 4 writes it out
      const int b = NB == 2 ? (seg & 1) : 0;
      const uint32_t use_b = (uint32_t)(NB == 2 ? (seg >> 1) : seg);
      const int seg_k0 = seg_ch0 * KC, seg_k1 = (cur_ch + 1) * KC;
      const int my_seg = seg;
      seg_ch0 = ch;
      ++seg;
      if ((my_seg & 3) != g) continue;
      if (!dep_done) {
        asm volatile("griddepcontrol.wait;" ::: "memory");  // args.inv comes from the conversion
        dep_done = true;
      }
      const int64_t row = (int64_t)cur_tile * 128 + r;
      const bool exact_path = row < args.n && row_overflows<FMT>(args, row, seg_k0, seg_k1);
      float rs = 1.0f;
      if constexpr (FMT == QLIN_FP8_ROW) {
        if (row < args.n) rs = __bfloat162float(((const __nv_bfloat16*)args.scales)[row]);
      }
      dead = dead || __any_sync(0xffffffffu, *abort_flag != 0);
      if (!dead && !__all_sync(0xffffffffu, mbar_wait(&acc_full[b], use_b & 1u))) {
        dead = true;
        abort_now();
      }
      const int64_t tstart = (int64_t)cur_tile * cpt, tend = tstart + cpt;
      const bool whole = u0 <= tstart && u1 >= tend;
      const int pslot = (cur_tile == tile0) ? 0 : 1;
      float* mine = args.partials + ((int64_t)blockIdx.x * 2 + pslot) * T * 128;
      if (!dead) {
        tc_fence_after();
        const uint32_t d_addr = tmem + lane_ofs + b * NACC * TP;
#pragma unroll
        for (int c0 = 0; c0 < TP; c0 += 16) {
          if (c0 < T) {
            // the issuers' accumulators one after another into a running sum
            float sum[16];
#pragma unroll
            for (int a = 0; a < NACC; ++a) {
              uint32_t vr[16];
              tmem_ld_x16(d_addr + a * TP + c0, vr);
              tmem_ld_wait();
#pragma unroll
              for (int jj = 0; jj < 16; ++jj) asm volatile("" : "+r"(vr[jj]));
#pragma unroll
              for (int jj = 0; jj < 16; ++jj) sum[jj] = a == 0 ? __uint_as_float(vr[jj]) : sum[jj] + __uint_as_float(vr[jj]);
            }
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
              const int t = c0 + jj;
              if (t < T) {
                float v = sum[jj];
                if (args.inv) v *= __ldg(args.inv + t);
                if constexpr (Tr::PER_GROUP) {
                  if (exact_path) v = row_dot_exact<FMT>(args, row, seg_k0, seg_k1, t);
                }
                v *= rs;
                if (whole) {
                  if (row < args.n) {
                    if (args.y_dtype == QLIN_OUT_F32)
                      ((float*)args.y)[(int64_t)t * args.n + row] = v;
                    else
                      ((__nv_bfloat16*)args.y)[(int64_t)t * args.n + row] = __float2bfloat16_rn(v);
                  }
                } else {
                  mine[t * 128 + et] = v;
                }
              }
            }
          }
        }
        tc_fence_before();
      }
      __syncwarp();
      if (lane == 0 && !dead) mbar_arrive(&acc_empty[b]);
      if (whole) continue;
      // split tile: publish this part, the last contributor reduces
      __threadfence();
      named_barrier_sync(1 + g, 128);
      if (et == 0) fix_slot[g] = dead ? -1 : atomicAdd(&args.counters[cur_tile], 1);
      named_barrier_sync(1 + g, 128);
      const int old = fix_slot[g];
      const int64_t i_first = unit_owner(tstart, U, P), i_last = unit_owner(tend - 1, U, P);
      if (old == (int)(i_last - i_first)) {
        __threadfence();
        // the parts in CTA order, 16 tokens at a time with their loads in flight
        for (int c0 = 0; c0 < T; c0 += 16) {
          float acc[16];
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) acc[jj] = 0.0f;
          for (int64_t ip = i_first; ip <= i_last; ++ip) {
            const int si = (cur_tile == unit_start(ip, U, P) / cpt) ? 0 : 1;
            const float* part = args.partials + (ip * 2 + si) * T * 128 + et;
            float pv[16];
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) pv[jj] = c0 + jj < T ? __ldcg(part + (c0 + jj) * 128) : 0.0f;
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) acc[jj] += pv[jj];
          }
          if (row < args.n) {
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
              const int t = c0 + jj;
              if (t < T) {
                if (args.y_dtype == QLIN_OUT_F32)
                  ((float*)args.y)[(int64_t)t * args.n + row] = acc[jj];
                else
                  ((__nv_bfloat16*)args.y)[(int64_t)t * args.n + row] = __float2bfloat16_rn(acc[jj]);
              }
            }
          }
        }
        if (et == 0) args.counters[cur_tile] = 0;  // leave the counter ready for the next call
      }
    }
  }

  // Every accumulator's completion was observed by an epilogue before this
  // point, so no MMA is in flight -- unless a wait timed out; then give the
  // tensor core ample time (1 ms) before the tensor memory is released.
  tc_fence_before();
  __syncthreads();
  if (warp == FW_ISS0) {
    if (*abort_flag) {
      const unsigned long long t0 = global_ns();
      while (global_ns() - t0 < 1000000ull) {
      }
    }
    tc_fence_after();
    tmem_dealloc(tmem, F_TMEM_COLS);
  }
}

// ---- activation conversion: x BF16 [T][K] -> FP16 scaled by 2^e_t per token,
// e_t chosen so that the token's largest magnitude lies in [2^14, 2^15);
// inv[t] = 2^-e_t.  One block per token.
__global__ void __launch_bounds__(256) x_to_f16_kernel(const uint16_t* __restrict__ x, int64_t k,
                                                       uint16_t* __restrict__ x16, float* __restrict__ inv) {
  // the GEMV launched behind this kernel may start its prologue now
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ uint32_t red[8];
  const int64_t t = blockIdx.x;
  const uint4* row = (const uint4*)(x + t * k);
  uint4* orow = (uint4*)(x16 + t * k);
  const int64_t n16 = k / 8;
  uint32_t mx = 0;  // largest |x| as BF16 magnitude bits (ordered like the values)
  for (int64_t i = threadIdx.x; i < n16; i += blockDim.x) {
    const uint4 v = row[i];
    mx = max(mx, __vmaxu2(__vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu), __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu)));
  }
  mx = max(mx & 0xFFFFu, mx >> 16);
#pragma unroll
  for (int o = 16; o; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  mx = 0;
  for (int i = 0; i < (int)(blockDim.x >> 5); ++i) mx = max(mx, red[i]);
  int e = 0;  // e_t; 0 for an all-zero token or one holding Inf / NaN
  if (mx != 0 && mx < 0x7F80u) {
    const int ef = (int)(mx >> 7);
    const int lg = ef > 0 ? ef - 127 : (31 - __clz((int)(mx & 0x7Fu))) - 133;  // floor(log2 max|x|)
    e = 14 - lg;
    e = e > 126 ? 126 : (e < -126 ? -126 : e);
  }
  const float sc = __uint_as_float((uint32_t)(127 + e) << 23);
  for (int64_t i = threadIdx.x; i < n16; i += blockDim.x) {
    const uint4 v = row[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float lo = __uint_as_float(w[j] << 16) * sc, hi = __uint_as_float(w[j] & 0xFFFF0000u) * sc;
      const __half2 h = __floats2half2_rn(lo, hi);
      o[j] = *(const uint32_t*)&h;
    }
    orow[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
  if (threadIdx.x == 0) inv[t] = __uint_as_float((uint32_t)(127 - e) << 23);
}

int tpad_f(int64_t t) { return t <= 16 ? 16 : t <= 32 ? 32 : t <= 48 ? 48 : 64; }

template <int FMT>
int unit_k_f(int tp) {
  switch (tp) {
    case 16: return FCfg<FMT, 16>::L::KC;
    case 32: return FCfg<FMT, 32>::L::KC;
    case 48: return FCfg<FMT, 48>::L::KC;
    default: return FCfg<FMT, 64>::L::KC;
  }
}

int unit_k_of(int fmt, int tp) {
  return fmt == QLIN_Q8_G32 ? unit_k_f<QLIN_Q8_G32>(tp) : unit_k_f<QLIN_FP8_ROW>(tp);
}

struct WsLayout {
  size_t counters, partials, x16, inv, total;
};

size_t al256(size_t v) { return (v + 255) / 256 * 256; }

WsLayout ws_layout(const qlin_weights& w, int64_t t, int num_sms) {
  WsLayout L;
  const int64_t tiles = (w.n + 127) / 128;
  L.counters = 0;
  L.partials = al256((size_t)tiles * sizeof(int));
  L.x16 = L.partials + al256((size_t)num_sms * 2 * t * 128 * sizeof(float));
  L.inv = L.x16 + al256((size_t)t * w.k * 2);
  L.total = L.inv + al256((size_t)t * sizeof(float));
  return L;
}

template <int FMT, int TP>
int launch_tp_f(const CUtensorMap& mc, const CUtensorMap& mx, const CUtensorMap& ms, const FArgs& a,
                int grid, cudaStream_t st) {
  using C = FCfg<FMT, TP>;
  const cudaError_t e0 = set_smem_once<gemv_f16_kernel<FMT, TP>>((int)C::SMEM);
  if (e0 != cudaSuccess) return cuda_status(e0);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(F_THREADS);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_status(cudaLaunchKernelEx(&cfg, gemv_f16_kernel<FMT, TP>, mc, mx, ms, a));
}

template <int FMT>
int launch_fmt_f(int tp, const CUtensorMap& mc, const CUtensorMap& mx, const CUtensorMap& ms,
                 const FArgs& a, int grid, cudaStream_t st) {
  switch (tp) {
    case 16: return launch_tp_f<FMT, 16>(mc, mx, ms, a, grid, st);
    case 32: return launch_tp_f<FMT, 32>(mc, mx, ms, a, grid, st);
    case 48: return launch_tp_f<FMT, 48>(mc, mx, ms, a, grid, st);
    default: return launch_tp_f<FMT, 64>(mc, mx, ms, a, grid, st);
  }
}

}  // namespace

// FP8-row and Q8 group-32 weights whose rows are whole units (K a multiple of
// the unit's 256 columns), 1 <= T <= 64.
bool gemv_f16_supported(const qlin_weights& w, int64_t t) {
  if (t < 1 || t > 64) return false;
  if (w.fmt != QLIN_FP8_ROW && w.fmt != QLIN_Q8_G32) return false;
  return w.k % unit_k_of(w.fmt, tpad_f(t)) == 0;
}

size_t gemv_f16_workspace_bytes(const qlin_weights& w, int64_t t, int num_sms) {
  return ws_layout(w, t, num_sms).total;
}

int launch_gemv_f16(const qlin_weights& w, const uint16_t* x, int64_t t, void* y, int y_dtype,
                    const Exec& ex) {
  const int tp = tpad_f(t);
  const int64_t tiles = (w.n + 127) / 128;
  const int64_t kc = unit_k_of(w.fmt, tp);
  const int64_t cpt = w.k / kc;
  const int64_t units = tiles * cpt;
  const int grid = (int)std::min<int64_t>(ex.num_sms, units);
  const WsLayout wl = ws_layout(w, t, ex.num_sms);
  uint8_t* ws = (uint8_t*)ex.workspace;
  uint16_t* x16 = (uint16_t*)(ws + wl.x16);
  float* inv = (float*)(ws + wl.inv);
  x_to_f16_kernel<<<(unsigned)t, 256, 0, ex.stream>>>(x, w.k, x16, inv);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_status(e);
  CUtensorMap mc, mx, ms;
  int rc = encode_tmap_2d(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, w.codes, (uint64_t)w.k, (uint64_t)w.n,
                          (uint64_t)w.k, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return rc;
  rc = encode_tmap_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, x16, (uint64_t)w.k, (uint64_t)t,
                      (uint64_t)w.k * 2, 64, (uint32_t)tp, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return rc;
  ms = mc;
  if (w.fmt == QLIN_Q8_G32) {
    // the group scales: one box of 8 FP16 scales (16 bytes) x 128 rows per unit
    const int64_t ng = w.k / 32;
    rc = encode_tmap_2d(&ms, CU_TENSOR_MAP_DATA_TYPE_UINT16, w.scales, (uint64_t)ng, (uint64_t)w.n,
                        (uint64_t)ng * 2, 8, 128, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (rc) return rc;
  }
  FArgs a;
  a.scales = w.scales;
  a.codes = (const uint8_t*)w.codes;
  a.x = x;
  a.inv = inv;
  a.y = y;
  a.counters = (int*)(ws + wl.counters);
  a.partials = (float*)(ws + wl.partials);
  a.dev_status = ex.dev_status;
  a.n = w.n;
  a.k = w.k;
  a.t = t;
  a.cpt = cpt;
  a.units = units;
  a.y_dtype = y_dtype;
  if (w.fmt == QLIN_Q8_G32) return launch_fmt_f<QLIN_Q8_G32>(tp, mc, mx, ms, a, grid, ex.stream);
  return launch_fmt_f<QLIN_FP8_ROW>(tp, mc, mx, ms, a, grid, ex.stream);
}

}  // namespace qlin
