// BF16-route projection on the 5th-generation tensor cores (decode / MTP /
// verify steps, T <= 64): y[T][N] = x[T][K] * W^T with the packed weights
// dequantized on the fly ("Qwen3.8-27B, NInfer int8-prefill artifact for the
// RTX 4090", "What changes": decode keeps the BF16 route; "...NVFP4-
// NInferV3", "How it was created": the FP8 head op over T = 1..33).
//
// Why tensor cores for a bandwidth-bound GEMV: at T >= 2 the CUDA cores cannot
// both unpack the codes and do T FMAs per weight at HBM speed.  Here the CUDA
// cores only unpack; tcgen05 MMAs do the dot products.
//
// One persistent CTA per SM walks a contiguous range of units (a unit is one
// 128-row tile x 256 bytes of packed codes per row, or 128 bytes when the
// activation tile would not leave room for three stages), so every SM streams
// the same number of weight bytes (stream-K):
//   warp 0      TMA: the unit's packed codes (two 128-byte-wide boxes: wide
//               row segments keep HBM efficient), the Q5 high-bit plane and the
//               matching activation columns into a ring of shared-memory
//               stages; its 32 lanes cp.async the group scales;
//   warpgroups 1-2  take turns on batches of quantization groups: every thread
//               owns one weight row, expands the batch's codes to exact BF16
//               integers (exponent-bias tricks, no conversions) and writes them
//               with tcgen05.st as the MMA's A operand straight into tensor
//               memory, then each warp arrives on the warpgroup's barrier and
//               goes on to its next batch;
//   warps 1-2   issuer w waits for warpgroup w's batch and one elected thread
//               issues its tcgen05.mma.kind::f16 (A in tensor memory, B = the
//               activations in shared memory, M = 128, N = T padded to 16), one
//               FP32 accumulator per group, and commits once (the expanding
//               warps no longer stop to issue MMAs themselves);
//   warpgroup 3 the epilogue reads a batch's 128 x T sums with tcgen05.ld,
//               applies each group's FP16 scale in FP32 registers and re-zeroes
//               the accumulators (every MMA accumulates: one that overwrites its
//               accumulator costs about four that accumulate).
// Tiles split between two CTAs meet in a workspace; the last CTA to arrive
// sums the parts in a fixed order (deterministic) and writes y.
#include "qlin_gemv_common.cuh"

namespace qlin {
namespace {
using namespace gemv;

constexpr uint32_t TMEM_COLS = 512;
constexpr int SMEM_BUDGET = 212992;
constexpr int NWG = 2;                // dequantizing / MMA-issuing warpgroups
constexpr int THREADS = 16 * 32;      // control, 2 x dequant, epilogue warpgroups
constexpr int W_DQ0 = 4, W_EPI0 = 12;

template <int FMT, int TP, int UB>
struct Layout {
  using Tr = TcT<FMT>;
  static constexpr int GPC = Tr::GPB * UB;            // groups per unit
  static constexpr int KC = Tr::GK * GPC;             // K columns per unit
  static constexpr int XBOXES = KC / 64;              // activation boxes (64 columns each)
  static constexpr int X_BYTES = XBOXES * TP * 128;
  static constexpr int HIB_BYTES = Tr::HIB ? UB * 128 * Tr::HROW : 0;
  static constexpr int SC_ROW = Tr::PER_GROUP ? GPC * 2 : 0;  // scale bytes per row per unit
  static constexpr int SC_BYTES = 128 * SC_ROW;
  static constexpr int TMA_BYTES = UB * BOX_BYTES + X_BYTES + HIB_BYTES;
  static constexpr int STAGE = TMA_BYTES + SC_BYTES;
  static constexpr int NS = (SMEM_BUDGET / STAGE) > 8 ? 8 : (SMEM_BUDGET / STAGE);
};

template <int FMT, int TP>
struct Cfg {
  using Tr = TcT<FMT>;
  // two 128-byte boxes per unit when three stages still fit, else one
  static constexpr int UB = Layout<FMT, TP, 2>::NS >= 3 ? 2 : 1;
  using L = Layout<FMT, TP, UB>;
  static constexpr int GPC = L::GPC, KC = L::KC, NS = L::NS;
  static constexpr int ACOLS = Tr::GK / 2;            // tensor-memory columns of one group's A
  static constexpr bool fits(int gb, int nd) { return NWG * (gb * ACOLS + nd * gb * TP) <= (int)TMEM_COLS; }
  static constexpr int gb_for(int nd) {
    return (GPC % 4 == 0 && fits(4, nd)) ? 4 : (GPC % 2 == 0 && fits(2, nd)) ? 2 : 1;
  }
  // groups per batch: one barrier, one commit and one epilogue wait per batch.
  // Fixed costs per batch (tensor-memory round trips, the barrier, the MMA
  // issue) favour large batches: one accumulator slot per warpgroup when that
  // allows more groups per batch than two slots do.
  static constexpr int NDW = gb_for(1) > gb_for(2) ? 1 : 2;  // accumulator slots per warpgroup
  static constexpr int GB = gb_for(NDW);
  static constexpr int BPU = GPC / GB;                // batches per unit
  static constexpr int A_COLS = GB * ACOLS;           // a warpgroup's A slot
  static constexpr int D_COLS = GB * TP;              // one accumulator slot (a batch)
  static constexpr int WG_COLS = A_COLS + NDW * D_COLS; // per warpgroup: A slot + accumulator slots
  static_assert(NS >= 2, "pipeline needs two stages");
  static_assert(NWG * WG_COLS <= (int)TMEM_COLS, "tensor memory budget");
  static constexpr size_t SMEM = (size_t)NS * L::STAGE + 1024 + 512;
  static constexpr int RND = TP <= 32 ? TP : 32;      // accumulator columns per epilogue read
};

// Keeps uses of r after the preceding tcgen05.wait::ld (volatile asm statements
// keep their order; plain arithmetic on r would not be tied to the wait).
template <int W>
__device__ __forceinline__ void after_wait(uint32_t* r) {
#pragma unroll
  for (int i = 0; i < W; ++i) asm volatile("" : "+r"(r[i]));
}

struct TcArgs {
  const void* scales;
  void* y;
  float* partials;  // [P][2][T][128]
  int* counters;    // [tiles]
  int32_t* dev_status;
  int64_t n, k, t;
  int64_t cpt;      // units per tile
  int64_t units;    // tiles * cpt
  int y_dtype;
};

template <int FMT, int TP>
__global__ void __launch_bounds__(THREADS, 1)
    gemv_tc_kernel(const __grid_constant__ CUtensorMap tm_codes,
                   const __grid_constant__ CUtensorMap tm_hib,
                   const __grid_constant__ CUtensorMap tm_x, TcArgs args) {
  using Tr = TcT<FMT>;
  using C = Cfg<FMT, TP>;
  using L = typename C::L;
  constexpr int NS = C::NS, UB = C::UB, GPC = C::GPC, GB = C::GB, BPU = C::BPU;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* codes_s = base;                                  // NS x UB boxes
  uint8_t* x_s = codes_s + NS * UB * BOX_BYTES;             // NS x X_BYTES
  uint8_t* hib_s = x_s + NS * L::X_BYTES;                   // NS x HIB_BYTES
  uint8_t* sc_s = hib_s + NS * L::HIB_BYTES;                // NS x SC_BYTES
  uint64_t* full = (uint64_t*)(sc_s + NS * L::SC_BYTES);
  uint64_t* empty = full + NS;
  uint64_t* d_full = empty + NS;        // [NWG][2], slots 0..NDW-1 used
  uint64_t* d_empty = d_full + 2 * NWG; // [NWG][2]
  uint64_t* a_full = d_empty + 2 * NWG;  // [NWG]: a batch's A operand is written
  uint32_t* tmem_slot = (uint32_t*)(a_full + NWG);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  volatile int* fix_slot = (volatile int*)(tmem_slot + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t P = gridDim.x;
  const int64_t U = args.units;
  const int64_t u0 = unit_start(blockIdx.x, U, P), u1 = unit_start(blockIdx.x + 1, U, P);
  const int64_t ng = args.k / Tr::GK;  // groups per row
  const int T = (int)args.t;
  const int cpt = (int)args.cpt;
  const int nunits = (int)(u1 - u0);
  const int tile0 = (int)(u0 / cpt), ch0 = (int)(u0 % cpt);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1 + 32);  // TMA issue + 32 scale-copy arrivals
      mbar_init(&empty[s], 128);    // every epilogue thread, once done with the unit's scales
    }
    for (int i = 0; i < 2 * NWG; ++i) {
      mbar_init(&d_full[i], 1);  // the issuer's tcgen05.commit
      mbar_init(&d_empty[i], 128);
    }
    for (int i = 0; i < NWG; ++i) mbar_init(&a_full[i], 4);  // the warpgroup's four warps
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_codes);
    tma_prefetch_desc(&tm_x);
    if (Tr::HIB) tma_prefetch_desc(&tm_hib);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // warpgroup w: A slot at w * WG_COLS, accumulator slots j at + A_COLS + j * D_COLS
  if (warp >= W_EPI0) {  // accumulators start at zero; the epilogue re-zeroes each after use
    const uint32_t lo = (uint32_t)((warp & 3) * 32) << 16;
#pragma unroll 1
    for (int w = 0; w < NWG; ++w)
#pragma unroll 1
      for (int c = 0; c < C::NDW * C::D_COLS; c += 16)
        tmem_fill_x16(tmem + lo + w * C::WG_COLS + C::A_COLS + c, 0u);
    tmem_st_wait();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // the next kernel on the stream may be scheduled as this one's CTAs leave;
  // it waits (griddepcontrol.wait) before it touches anything this one writes
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  auto abort_now = [&]() {
    *abort_flag = 1;
    report_timeout(args.dev_status);
  };

  if (warp == 0) {
    // lane 0 issues the TMA copies; all 32 lanes copy the unit's group scales
    // (SC_ROW bytes per row) with cp.async, tracked by the same barrier.  The
    // weights of the first NS units (codes, planes, scales: never written by
    // the kernels of a decode step) go out before the wait for the kernel
    // launched ahead of this one; x, which that kernel may produce, after it.
    const uint64_t pol_w = l2_evict_first(), pol_x = l2_evict_last();  // codes stream once; x serves every CTA
    const int npre = nunits < NS ? nunits : NS;
    int issued = 0;
    Ring ring{0, 0};
    int tile = tile0, ch = ch0;
    for (int cu = 0; cu < nunits; ++cu) {
      const int s = ring.slot;
      if (!__all_sync(0xffffffffu, !*abort_flag && mbar_wait(&empty[s], (uint32_t)(ring.phase ^ 1)))) {
        if (lane == 0) abort_now();
        break;
      }
      if (lane == 0) {
        mbar_arrive_expect_tx(&full[s], L::TMA_BYTES);
#pragma unroll
        for (int b = 0; b < UB; ++b)
          tma_load_2d_hint(codes_s + (s * UB + b) * BOX_BYTES, &tm_codes, &full[s], (ch * UB + b) * 128, tile * 128,
                           pol_w);
        if (Tr::HIB)
          tma_load_2d_hint(hib_s + s * L::HIB_BYTES, &tm_hib, &full[s], ch * UB * Tr::HROW, tile * 128, pol_w);
        if (cu >= npre) {
#pragma unroll
          for (int b = 0; b < L::XBOXES; ++b)
            tma_load_2d_hint(x_s + s * L::X_BYTES + b * TP * 128, &tm_x, &full[s], ch * C::KC + b * 64, 0, pol_x);
        }
      }
      if constexpr (Tr::PER_GROUP) {
        const __half* src = (const __half*)args.scales + ch * GPC;
        uint8_t* dst = sc_s + s * L::SC_BYTES;
#pragma unroll
        for (int rr = lane; rr < 128; rr += 32) {
          const int64_t row = (int64_t)tile * 128 + rr;
          if (row < args.n) {
#pragma unroll
            for (int q8 = 0; q8 < L::SC_ROW / 8; ++q8)  // four scales per 8-byte copy
              cp_async_8(dst + rr * L::SC_ROW + 8 * q8, src + row * ng + 4 * q8);
          }
        }
      }
      cp_async_arrive_noinc(&full[s]);
      ++issued;
      ring.next(NS);
      if (++ch == cpt) {
        ch = 0;
        ++tile;
      }
      if (cu == npre - 1) {
        asm volatile("griddepcontrol.wait;" ::: "memory");
        if (lane == 0) {
          // the activation boxes of the first npre units (stages 0..npre-1)
          for (int c = 0; c < npre; ++c) {
            const int chc = (int)((ch0 + c) % cpt);
#pragma unroll
            for (int b = 0; b < L::XBOXES; ++b)
              tma_load_2d_hint(x_s + c * L::X_BYTES + b * TP * 128, &tm_x, &full[c], chc * C::KC + b * 64, 0,
                               pol_x);
          }
        }
      }
    }
    if (lane == 0)
      for (int cu = issued > NS ? issued - NS : 0; cu < issued; ++cu)
        mbar_wait(&full[cu % NS], (uint32_t)((cu / NS) & 1));
  } else if (warp >= 1 && warp <= NWG) {
    // ---- MMA issue for warpgroup wg = warp - 1: once the warpgroup's four
    // warps have written a batch's A operand, one elected thread issues the
    // batch's MMAs (every group into its own accumulator) and commits once.
    const int wg = warp - 1;
    const uint32_t idesc = idesc_bf16(128, TP);
    const uint32_t a_base = tmem + wg * C::WG_COLS;
    const uint32_t d_base = a_base + C::A_COLS;
    bool ok = true;
    Ring ring{0, 0};
    Ring dr{0, 0};
    uint32_t nb = 0;  // batches of this warpgroup so far
    int bw = 0;       // owner of the next batch
    for (int cu = 0; cu < nunits && ok; ++cu) {
      const int s = ring.slot;
      bool mine = false;
      {
        int w = bw;
        for (int bi = 0; bi < BPU; ++bi) {
          mine |= w == wg;
          w = (w + 1 == NWG) ? 0 : w + 1;
        }
      }
      // the stage's activations have landed
      if (mine) ok = __all_sync(0xffffffffu, !*abort_flag && mbar_wait(&full[s], (uint32_t)ring.phase));
      const uint32_t xs_base = smem_u32(x_s + s * L::X_BYTES);
      for (int bi = 0; bi < BPU && ok; ++bi, bw = (bw + 1 == NWG) ? 0 : bw + 1) {
        if (bw != wg) continue;
        const int ds = dr.slot;
        // the batch's A operand is written; the accumulator slot was read and
        // re-zeroed by the epilogue
        ok = __all_sync(0xffffffffu, !*abort_flag && mbar_wait(&a_full[wg], nb & 1u) &&
                                         mbar_wait(&d_empty[wg * 2 + ds], (uint32_t)(dr.phase ^ 1)));
        if (!ok) break;
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int g = 0; g < GB; ++g) {
            const int kofs = (bi * GB + g) * Tr::GK;  // K offset of the group inside the unit
            const uint32_t xaddr = xs_base + (kofs / 64) * TP * 128 + (kofs % 64) * 2;
#pragma unroll
            for (int kk = 0; kk < Tr::GK / 16; ++kk)
              mma_f16_ts(d_base + ds * C::D_COLS + g * TP, a_base + g * C::ACOLS + kk * 8,
                         sdesc_k_sw128(xaddr + kk * 32), idesc, 1u);
          }
          tc_commit(&d_full[wg * 2 + ds]);
        }
        __syncwarp();
        ++nb;
        dr.next(C::NDW);
      }
      ring.next(NS);
    }
    if (!ok && lane == 0) abort_now();
  } else if (warp >= W_DQ0 && warp < W_EPI0) {
    // ---- dequantize: warpgroup wg takes the batches b with b % NWG == wg
    const int wg = (warp - W_DQ0) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_ofs = (uint32_t)(quarter * 32) << 16;
    const uint32_t a_base = tmem + wg * C::WG_COLS;
    bool dead = false;  // after a timed-out wait: skip work, keep the barrier sequence
    Ring ring{0, 0};
    Ring dr{0, 0};       // this warpgroup's accumulator slot
    int prev_slot = -1, prev_phase = 0;
    int bw = 0;          // owner of the next batch
    for (int cu = 0; cu < nunits; ++cu) {
      const int s = ring.slot;
      bool mine = false;
      {
        int w = bw;
        for (int bi = 0; bi < BPU; ++bi) {
          mine |= w == wg;
          w = (w + 1 == NWG) ? 0 : w + 1;
        }
      }
      if (mine && !dead &&
          !__all_sync(0xffffffffu, !*abort_flag && mbar_wait(&full[s], (uint32_t)ring.phase))) {
        dead = true;
        abort_now();
      }
      const uint8_t* cs = codes_s + s * UB * BOX_BYTES;
      const uint8_t* hs = hib_s + s * L::HIB_BYTES;
      for (int bi = 0; bi < BPU; ++bi, bw = (bw + 1 == NWG) ? 0 : bw + 1) {
        if (bw != wg) continue;
        const int ds = dr.slot;
        if (!dead) {
          // the previous batch's MMAs (which read the A slot) are complete; the
          // accumulator slot is waited for only by the issuing threads, so that
          // the expansion overlaps the epilogue's draining of it
          bool ok = true;
          if (prev_slot >= 0) ok = mbar_wait(&d_full[wg * 2 + prev_slot], (uint32_t)prev_phase);
          if (!__all_sync(0xffffffffu, ok)) {
            dead = true;
            abort_now();
          }
        }
        if (!dead) {
          tc_fence_after();
#pragma unroll 2
          for (int g = 0; g < GB; ++g) {
            const int gi = bi * GB + g;  // group within the unit
            uint32_t v[C::ACOLS];
            dequant_group<FMT>(cs + (gi / Tr::GPB) * BOX_BYTES, hs + r * Tr::HROW * UB + (gi / Tr::GPB) * Tr::HROW,
                               r, gi % Tr::GPB, v);
            if constexpr (C::ACOLS == 32)
              tmem_st_x32(a_base + lane_ofs + g * C::ACOLS, v);
            else
              tmem_st_x16(a_base + lane_ofs + g * C::ACOLS, v);
          }
          tmem_st_wait();
        }
        // hand the batch to the warpgroup's issuing warp; the four warps never
        // wait for one another or for the MMA issue
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&a_full[wg]);
        prev_slot = ds;
        prev_phase = dr.phase;
        dr.next(C::NDW);
      }
      ring.next(NS);
    }
  } else if (warp >= W_EPI0) {
    // y and the split-tile workspace may still be in use by the kernel ahead
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int et = threadIdx.x - W_EPI0 * 32;  // 0..127
    const uint32_t lane_ofs = (uint32_t)(quarter * 32) << 16;
    float acc[TP];
#pragma unroll
    for (int t = 0; t < TP; ++t) acc[t] = 0.0f;
    bool dead = false;  // after a timed-out wait: skip waits and work, keep the barrier sequence
    Ring ring{0, 0};
    Ring dr[NWG] = {{0, 0}, {0, 0}};
    int bw = 0;
    int tile = tile0, ch = ch0;
    for (int cu = 0; cu < nunits; ++cu) {
      const int s = ring.slot;
      const int64_t row = (int64_t)tile * 128 + r;
      const bool seg_first = cu == 0 || ch == 0;
      const bool seg_last = cu + 1 == nunits || ch == cpt - 1;
      if (seg_first) {
#pragma unroll
        for (int t = 0; t < TP; ++t) acc[t] = 0.0f;
      }
      dead = dead || __any_sync(0xffffffffu, *abort_flag != 0);
      // the stage's scales have landed once its barrier completed (acquire)
      if (!dead && !__all_sync(0xffffffffu, mbar_wait(&full[s], (uint32_t)ring.phase))) {
        dead = true;
        abort_now();
      }
      const __half* sc_row = (const __half*)(sc_s + s * L::SC_BYTES) + r * GPC;
      for (int bi = 0; bi < BPU; ++bi, bw = (bw + 1 == NWG) ? 0 : bw + 1) {
        const int ds = dr[bw].slot;
        const uint32_t dph = (uint32_t)dr[bw].phase;
        dr[bw].next(C::NDW);
        if (dead) continue;
        if (!__all_sync(0xffffffffu, mbar_wait(&d_full[bw * 2 + ds], dph))) {
          dead = true;
          abort_now();
          continue;
        }
        tc_fence_after();
        const uint32_t d_addr = tmem + bw * C::WG_COLS + C::A_COLS + ds * C::D_COLS + lane_ofs;
#pragma unroll
        for (int g = 0; g < GB; ++g) {
          float sc = 1.0f;
          if constexpr (Tr::PER_GROUP) sc = __half2float(sc_row[bi * GB + g]);
#pragma unroll
          for (int c0 = 0; c0 < TP; c0 += C::RND) {
            if (c0 < T) {
              // one round trip for up to RND columns, in 16-column loads (the
              // last may run past T: those columns stay zero).  Narrower loads
              // chosen at run time (x1..x8) measured twice as slow overall.
              uint32_t vr[C::RND];
#pragma unroll
              for (int c = 0; c < C::RND; c += 16)
                if (c0 + c < T) tmem_ld_x16(d_addr + g * TP + c0 + c, vr + c);
              tmem_ld_wait();
              after_wait<C::RND>(vr);
#pragma unroll
              for (int c = 0; c < C::RND; c += 16) {
                if (c0 + c < T) {
                  tmem_fill_x16(d_addr + g * TP + c0 + c, 0u);  // ready for a later batch
#pragma unroll
                  for (int j = 0; j < 16; ++j)
                    acc[c0 + c + j] = fmaf(sc, __uint_as_float(vr[c + j]), acc[c0 + c + j]);
                }
              }
            }
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&d_empty[bw * 2 + ds]);
      }
      // every batch of the unit is done: the TMA stage (codes, activations,
      // scales) can be refilled once all four epilogue warps have read its scales
      if (!dead) mbar_arrive(&empty[s]);
      ring.next(NS);
      const int cur_tile = tile;
      if (++ch == cpt) {
        ch = 0;
        ++tile;
      }
      if (!seg_last) continue;
      // ---- the CTA's part of this tile is complete
      float rs = 1.0f;
      if constexpr (FMT == QLIN_FP8_ROW) {
        if (row < args.n) rs = __bfloat162float(((const __nv_bfloat16*)args.scales)[row]);
      }
      const int64_t tstart = (int64_t)cur_tile * cpt, tend = tstart + cpt;
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
      const int slot = (cur_tile == tile0) ? 0 : 1;
      float* mine = args.partials + ((int64_t)blockIdx.x * 2 + slot) * T * 128;
      if (!dead) {
#pragma unroll
        for (int t = 0; t < TP; ++t)
          if (t < T) mine[t * 128 + et] = acc[t];
      }
      __threadfence();
      named_barrier_sync(15, 128);
      if (et == 0) *fix_slot = dead ? -1 : atomicAdd(&args.counters[cur_tile], 1);
      named_barrier_sync(15, 128);
      const int old = *fix_slot;
      const int64_t i_first = unit_owner(tstart, U, P), i_last = unit_owner(tend - 1, U, P);
      if (old == (int)(i_last - i_first)) {
        __threadfence();
#pragma unroll
        for (int t = 0; t < TP; ++t) acc[t] = 0.0f;
        for (int64_t i = i_first; i <= i_last; ++i) {
          const int si = (cur_tile == unit_start(i, U, P) / cpt) ? 0 : 1;
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
        if (et == 0) args.counters[cur_tile] = 0;  // leave the counter ready for the next call
      }
    }
  }

  // Every accumulator's completion was observed by the epilogue before this
  // point -- unless a wait timed out; then give the tensor core ample time
  // (1 ms) before the tensor memory is released.
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (*abort_flag) {
      const unsigned long long t0 = global_ns();
      while (global_ns() - t0 < 1000000ull) {
      }
    }
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

int tpad_of(int64_t t) { return t <= 16 ? 16 : t <= 32 ? 32 : t <= 48 ? 48 : 64; }

template <int FMT>
int unit_k_fmt(int tp) {
  switch (tp) {
    case 16: return Cfg<FMT, 16>::KC;
    case 32: return Cfg<FMT, 32>::KC;
    case 48: return Cfg<FMT, 48>::KC;
    default: return Cfg<FMT, 64>::KC;
  }
}

int unit_k(int fmt, int tp) {
  switch (fmt) {
    case QLIN_Q4_G64: return unit_k_fmt<QLIN_Q4_G64>(tp);
    case QLIN_Q5_G64: return unit_k_fmt<QLIN_Q5_G64>(tp);
    case QLIN_Q3_G64: return unit_k_fmt<QLIN_Q3_G64>(tp);
    case QLIN_Q6_G64: return unit_k_fmt<QLIN_Q6_G64>(tp);
    case QLIN_Q8_G32: return unit_k_fmt<QLIN_Q8_G32>(tp);
    case QLIN_FP8_ROW: return unit_k_fmt<QLIN_FP8_ROW>(tp);
    default: return unit_k_fmt<QLIN_BF16>(tp);
  }
}

template <int FMT, int TP>
int launch_tp(const CUtensorMap& mc, const CUtensorMap& mh, const CUtensorMap& mx, const TcArgs& a,
              int grid, cudaStream_t st) {
  using C = Cfg<FMT, TP>;
  auto kern = gemv_tc_kernel<FMT, TP>;
  const cudaError_t e = set_smem_once<gemv_tc_kernel<FMT, TP>>((int)C::SMEM);
  if (e != cudaSuccess) return cuda_status(e);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_status(cudaLaunchKernelEx(&cfg, kern, mc, mh, mx, a));
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

// Rows must be whole units (K a multiple of the unit's K columns: 512 for
// Q4/Q5 at T <= 16, etc.); other shapes take the CUDA-core kernel.
bool gemv_tc_supported(const qlin_weights& w, int64_t t) {
  if (t < 1 || t > 64) return false;
  return w.k % unit_k(w.fmt, tpad_of(t)) == 0;
}

size_t gemv_tc_workspace_bytes(const qlin_weights& w, int64_t t, int num_sms) {
  const int64_t tiles = (w.n + 127) / 128;
  const size_t counters = ((size_t)tiles * sizeof(int) + 255) / 256 * 256;
  return counters + (size_t)num_sms * 2 * t * 128 * sizeof(float);
}

int launch_gemv_tc(const qlin_weights& w, const uint16_t* x, int64_t t, void* y, int y_dtype,
                   const Exec& ex) {
  const int tp = tpad_of(t);
  const int64_t tiles = (w.n + 127) / 128;
  const int64_t kc = unit_k(w.fmt, tp);
  const int64_t cpt = w.k / kc;
  const int64_t units = tiles * cpt;
  const int grid = (int)std::min<int64_t>(ex.num_sms, units);
  const int64_t row_bytes = code_row_bytes(w.fmt, w.k);
  CUtensorMap mc, mh, mx;
  int rc = encode_tmap_2d(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, w.codes, (uint64_t)row_bytes,
                          (uint64_t)w.n, (uint64_t)row_bytes, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return rc;
  rc = encode_tmap_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, (uint64_t)w.k, (uint64_t)t,
                      (uint64_t)w.k * 2, 64, (uint32_t)tp, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return rc;
  if (hrow_of(w.fmt) != 0) {
    // second plane: its bytes for the unit's K columns per row
    const uint32_t hib_box = (uint32_t)hib_row_bytes(w.fmt, kc);
    const uint64_t hib_row = (uint64_t)hib_row_bytes(w.fmt, w.k);
    rc = encode_tmap_2d(&mh, CU_TENSOR_MAP_DATA_TYPE_UINT8, w.hibits, hib_row, (uint64_t)w.n, hib_row,
                        hib_box, 128, CU_TENSOR_MAP_SWIZZLE_NONE);
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
    case QLIN_Q3_G64: return launch_fmt<QLIN_Q3_G64>(tp, mc, mh, mx, a, grid, ex.stream);
    case QLIN_Q6_G64: return launch_fmt<QLIN_Q6_G64>(tp, mc, mh, mx, a, grid, ex.stream);
    case QLIN_Q8_G32: return launch_fmt<QLIN_Q8_G32>(tp, mc, mh, mx, a, grid, ex.stream);
    case QLIN_FP8_ROW: return launch_fmt<QLIN_FP8_ROW>(tp, mc, mh, mx, a, grid, ex.stream);
    default: return launch_fmt<QLIN_BF16>(tp, mc, mh, mx, a, grid, ex.stream);
  }
}

}  // namespace qlin
