// BF16-route projection for a single token (T = 1) on the CUDA cores:
// y[T][N] = x[T][K] * W^T with the packed weights dequantized on the fly
// ("Qwen3.8-27B, NInfer int8-prefill artifact for the RTX 4090", "What
// changes": decode keeps the BF16 route and is bandwidth bound).
//
// At T = 1 a tensor-core MMA (M = 128, N >= 16) wastes 15/16 of its work and
// one thread issues an MMA only every ~45-80 cycles; the CUDA cores do the
// dot products with the mixed-precision FMA of sm_100 (BF16 x BF16 + FP32,
// exact products, FP32 accumulation).  The kernel is written for T tokens,
// but from T = 2 on the tensor-core kernel measured faster, so only T = 1 is
// instantiated.
//
// One persistent CTA per SM walks a contiguous range of units (128-row tile x
// 256 bytes of packed codes per row), so every SM streams the same bytes:
//   warp 0      TMA: the unit's packed codes (two 128-byte-wide boxes), the Q5
//               high-bit plane and the matching activation columns into a ring
//               of shared-memory stages; its lanes cp.async the group scales;
//   warps 1-16  thread = (weight row, quarter of the unit's groups; 8 rows per
//               warp): expand each group to exact BF16 pairs (the same
//               exponent-bias tricks as the tensor-core kernel), FMA against x
//               from shared memory into one FP32 sum per group, apply the group's
//               FP16 scale; the parts of a row meet by shuffles at the end of the
//               CTA's part of a tile.  (BF16 weights, two groups per unit: halves,
//               16 rows per warp, warps 1-8.)
// Tiles split between two CTAs meet in the workspace exactly as in the
// tensor-core kernel (same layout, same deterministic reduction order).
#include "qlin_gemv_common.cuh"

namespace qlin {
namespace {
using namespace gemv;

constexpr int SM_SMEM_BUDGET = 212992;
constexpr int UBS = 2;                   // 128-byte code boxes per unit

template <int FMT, int T>
struct SmCfg {
  using Tr = TcT<FMT>;
  static constexpr int GPC = Tr::GPB * UBS;           // groups per unit
  static constexpr int KC = Tr::GK * GPC;             // K columns per unit
  static constexpr int XBOXES = KC / 64;              // activation boxes (64 columns x T rows)
  static constexpr int X_BYTES = XBOXES * T * 128;
  static constexpr int HIB_BYTES = Tr::HIB ? UBS * 128 * Tr::HROW : 0;
  static constexpr int SC_ROW = Tr::PER_GROUP ? GPC * 2 : 0;
  static constexpr int SC_BYTES = 128 * SC_ROW;
  static constexpr int TMA_BYTES = UBS * BOX_BYTES + X_BYTES + HIB_BYTES;
  // stage = codes | x | high bits | scales, each part 1024-byte aligned
  static constexpr int up(int v) { return (v + 1023) / 1024 * 1024; }
  static constexpr int OFF_X = UBS * BOX_BYTES;
  static constexpr int OFF_HIB = OFF_X + up(X_BYTES);
  static constexpr int OFF_SC = OFF_HIB + up(HIB_BYTES);
  static constexpr int STAGE = OFF_SC + up(SC_BYTES);
  static constexpr int NS = (SM_SMEM_BUDGET / STAGE) > 8 ? 8 : (SM_SMEM_BUDGET / STAGE);
  static_assert(NS >= 2, "pipeline needs two stages");
  static constexpr size_t SMEM = (size_t)NS * STAGE + 1024 + 256;
  static constexpr int ACOLS = Tr::GK / 2;            // BF16 pairs per group
  // a row's groups are split over PARTS lanes of one warp (RPW rows per warp);
  // 128 rows then take NCW compute warps: 16 warps (4 per scheduler) keep the
  // shared-memory and FMA latencies hidden
  static constexpr int PARTS = GPC >= 4 ? 4 : GPC;
  static constexpr int RPW = 32 / PARTS;
  static constexpr int NCW = 128 / RPW;
  static constexpr int THREADS = 32 * (1 + NCW);
  static constexpr int GPP = GPC / PARTS;             // groups per part
};

struct SmArgs {
  const void* scales;
  void* y;
  float* partials;  // [P][2][T][128]
  int* counters;    // [tiles]
  int32_t* dev_status;
  int64_t n, k;
  int64_t cpt;      // units per tile
  int64_t units;    // tiles * cpt
  int y_dtype;
};

__device__ __forceinline__ float fma_bf16(uint16_t a, uint16_t b, float c) {
  float d;
  asm("fma.rn.f32.bf16 %0, %1, %2, %3;" : "=f"(d) : "h"(a), "h"(b), "f"(c));
  return d;
}
__device__ __forceinline__ void halves(uint32_t v, uint16_t& lo, uint16_t& hi) {
  asm("mov.b32 {%0, %1}, %2;" : "=h"(lo), "=h"(hi) : "r"(v));
}

template <int FMT, int T>
__global__ void __launch_bounds__(SmCfg<FMT, T>::THREADS, 1)
    gemv_sm_kernel(const __grid_constant__ CUtensorMap tm_codes,
                   const __grid_constant__ CUtensorMap tm_hib,
                   const __grid_constant__ CUtensorMap tm_x, SmArgs args) {
  using Tr = TcT<FMT>;
  using C = SmCfg<FMT, T>;
  constexpr int NS = C::NS, GPC = C::GPC, NCW = C::NCW, RPW = C::RPW, GPP = C::GPP;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* full = (uint64_t*)(base + NS * C::STAGE);
  uint64_t* empty = full + NS;
  volatile int* abort_flag = (volatile int*)(empty + NS);
  volatile int* fix_slot = abort_flag + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t P = gridDim.x;
  const int64_t U = args.units;
  const int64_t u0 = unit_start(blockIdx.x, U, P), u1 = unit_start(blockIdx.x + 1, U, P);
  const int64_t ng = args.k / Tr::GK;  // groups per row
  const int cpt = (int)args.cpt;
  const int nunits = (int)(u1 - u0);
  const int tile0 = (int)(u0 / cpt), ch0 = (int)(u0 % cpt);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1 + 32);  // TMA issue + 32 scale-copy arrivals
      mbar_init(&empty[s], NCW);    // one arrival per compute warp
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_codes);
    tma_prefetch_desc(&tm_x);
    if (Tr::HIB) tma_prefetch_desc(&tm_hib);
  }
  __syncthreads();
  // the next kernel on the stream may be scheduled as this one's CTAs leave;
  // it waits (griddepcontrol.wait) before it touches anything this one writes
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  auto abort_now = [&]() {
    *abort_flag = 1;
    report_timeout(args.dev_status);
  };

  if (warp == 0) {
    // the weights of the first NS units (codes, planes, scales: never written
    // by the kernels of a decode step) go out before the wait for the kernel
    // launched ahead of this one; x, which that kernel may produce, after it
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
      uint8_t* st = base + s * C::STAGE;
      if (lane == 0) {
        mbar_arrive_expect_tx(&full[s], C::TMA_BYTES);
#pragma unroll
        for (int b = 0; b < UBS; ++b)
          tma_load_2d_hint(st + b * BOX_BYTES, &tm_codes, &full[s], (ch * UBS + b) * 128, tile * 128, pol_w);
        if (Tr::HIB) tma_load_2d_hint(st + C::OFF_HIB, &tm_hib, &full[s], ch * UBS * Tr::HROW, tile * 128, pol_w);
        if (cu >= npre) {
#pragma unroll
          for (int b = 0; b < C::XBOXES; ++b)
            tma_load_2d_hint(st + C::OFF_X + b * T * 128, &tm_x, &full[s], ch * C::KC + b * 64, 0, pol_x);
        }
      }
      if constexpr (Tr::PER_GROUP) {
        const __half* src = (const __half*)args.scales + ch * GPC;
        uint8_t* dst = st + C::OFF_SC;
#pragma unroll
        for (int rr = lane; rr < 128; rr += 32) {
          const int64_t row = (int64_t)tile * 128 + rr;
          if (row < args.n) {
#pragma unroll
            for (int q8 = 0; q8 < C::SC_ROW / 8; ++q8)  // four scales per 8-byte copy
              cp_async_8(dst + rr * C::SC_ROW + 8 * q8, src + row * ng + 4 * q8);
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
            uint8_t* stc = base + c * C::STAGE;
#pragma unroll
            for (int b = 0; b < C::XBOXES; ++b)
              tma_load_2d_hint(stc + C::OFF_X + b * T * 128, &tm_x, &full[c], chc * C::KC + b * 64, 0, pol_x);
          }
        }
      }
    }
    if (lane == 0) {
      Ring r2{0, 0};
      for (int i = 0; i < issued; ++i) {
        if (i + NS >= issued) mbar_wait(&full[r2.slot], (uint32_t)r2.phase);
        r2.next(NS);
      }
    }
  } else {
    // ---- compute warps: row r of the tile, part h of the unit's groups
    // (y and the split-tile workspace may still be in use by the kernel ahead)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int cw = warp - 1;
    const int r = cw * RPW + (lane % RPW);
    const int h = lane / RPW;
    const int et = r;  // index of the row within the tile
    float acc[T];
#pragma unroll
    for (int t = 0; t < T; ++t) acc[t] = 0.0f;
    bool dead = false;
    Ring ring{0, 0};
    int tile = tile0, ch = ch0;
    for (int cu = 0; cu < nunits; ++cu) {
      const int s = ring.slot;
      const int64_t row = (int64_t)tile * 128 + r;
      const bool seg_first = cu == 0 || ch == 0;
      const bool seg_last = cu + 1 == nunits || ch == cpt - 1;
      if (seg_first) {
#pragma unroll
        for (int t = 0; t < T; ++t) acc[t] = 0.0f;
      }
      dead = dead || __any_sync(0xffffffffu, *abort_flag != 0);
      if (!dead && !__all_sync(0xffffffffu, mbar_wait(&full[s], (uint32_t)ring.phase))) {
        dead = true;
        abort_now();
      }
      if (!dead) {
        const uint8_t* st = base + s * C::STAGE;
        const uint8_t* xs = st + C::OFF_X;
        const __half* sc_row = (const __half*)(st + C::OFF_SC) + r * GPC;
#pragma unroll 2
        for (int gg = 0; gg < GPP; ++gg) {
          const int gi = h * GPP + gg;  // group within the unit
          uint32_t v[C::ACOLS];
          // second-plane rows are UBS * HROW bytes
          dequant_group<FMT>(st + (gi / Tr::GPB) * BOX_BYTES,
                             st + C::OFF_HIB + r * Tr::HROW * UBS + (gi / Tr::GPB) * Tr::HROW, r,
                             gi % Tr::GPB, v);
          float g0[T], g1[T];  // two FMA chains per token
#pragma unroll
          for (int t = 0; t < T; ++t) g0[t] = g1[t] = 0.0f;
          const int kofs = gi * Tr::GK;  // K offset of the group inside the unit
#pragma unroll
          for (int c4 = 0; c4 < C::ACOLS / 4; ++c4) {
            const int kk = kofs + 8 * c4;  // 8 consecutive elements: one 16-byte unit of x
#pragma unroll
            for (int t = 0; t < T; ++t) {
              // x boxes are plain row-major [T][64] (all lanes read the same address)
              const uint4 xv = *(const uint4*)(xs + (kk / 64) * T * 128 + t * 128 + (kk % 64) * 2);
              const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                uint16_t ql, qh, xl, xh;
                halves(v[4 * c4 + e], ql, qh);
                halves(xw[e], xl, xh);
                g0[t] = fma_bf16(ql, xl, g0[t]);
                g1[t] = fma_bf16(qh, xh, g1[t]);
              }
            }
          }
          float sc = 1.0f;
          if constexpr (Tr::PER_GROUP) sc = __half2float(sc_row[gi]);
#pragma unroll
          for (int t = 0; t < T; ++t) acc[t] = fmaf(sc, g0[t] + g1[t], acc[t]);
        }
      }
      // the stage can be refilled once every compute warp is done with it
      __syncwarp();
      if (!dead && lane == 0) mbar_arrive(&empty[s]);
      ring.next(NS);
      const int cur_tile = tile;
      if (++ch == cpt) {
        ch = 0;
        ++tile;
      }
      if (!seg_last) continue;
      // ---- the CTA's part of this tile is complete: the parts of each row meet
#pragma unroll
      for (int o = RPW; o < 32; o <<= 1)
#pragma unroll
        for (int t = 0; t < T; ++t) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], o);
      float rs = 1.0f;
      if constexpr (FMT == QLIN_FP8_ROW) {
        if (row < args.n) rs = __bfloat162float(((const __nv_bfloat16*)args.scales)[row]);
      }
      const int64_t tstart = (int64_t)cur_tile * cpt, tend = tstart + cpt;
      const bool whole = u0 <= tstart && u1 >= tend;
      if (whole) {
        if (!dead && h == 0 && row < args.n) {
#pragma unroll
          for (int t = 0; t < T; ++t) {
            if (args.y_dtype == QLIN_OUT_F32)
              ((float*)args.y)[(int64_t)t * args.n + row] = acc[t] * rs;
            else
              ((__nv_bfloat16*)args.y)[(int64_t)t * args.n + row] = __float2bfloat16_rn(acc[t] * rs);
          }
        }
        continue;
      }
      // split tile: publish this part, the last contributor reduces
      const int slot = (cur_tile == tile0) ? 0 : 1;
      float* mine = args.partials + ((int64_t)blockIdx.x * 2 + slot) * T * 128;
      if (!dead && h == 0) {
#pragma unroll
        for (int t = 0; t < T; ++t) mine[t * 128 + et] = acc[t];
      }
      __threadfence();
      named_barrier_sync(1, NCW * 32);
      if (cw == 0 && lane == 0) *fix_slot = dead ? -1 : atomicAdd(&args.counters[cur_tile], 1);
      named_barrier_sync(1, NCW * 32);
      const int old = *fix_slot;
      const int64_t i_first = unit_owner(tstart, U, P), i_last = unit_owner(tend - 1, U, P);
      if (old == (int)(i_last - i_first)) {
        __threadfence();
        if (h == 0) {
#pragma unroll
          for (int t = 0; t < T; ++t) acc[t] = 0.0f;
          for (int64_t i = i_first; i <= i_last; ++i) {
            const int si = (cur_tile == unit_start(i, U, P) / cpt) ? 0 : 1;
            const float* part = args.partials + (i * 2 + si) * T * 128;
#pragma unroll
            for (int t = 0; t < T; ++t) acc[t] += __ldcg(part + t * 128 + et);
          }
          if (row < args.n) {
#pragma unroll
            for (int t = 0; t < T; ++t) {
              if (args.y_dtype == QLIN_OUT_F32)
                ((float*)args.y)[(int64_t)t * args.n + row] = acc[t] * rs;
              else
                ((__nv_bfloat16*)args.y)[(int64_t)t * args.n + row] = __float2bfloat16_rn(acc[t] * rs);
            }
          }
        }
        if (cw == 0 && lane == 0) args.counters[cur_tile] = 0;  // ready for the next call
      }
    }
  }
  __syncthreads();
}

template <int FMT>
int sm_unit_k() {
  return SmCfg<FMT, 1>::KC;
}
int unit_k_sm(int fmt) {
  switch (fmt) {
    case QLIN_Q4_G64: return sm_unit_k<QLIN_Q4_G64>();
    case QLIN_Q5_G64: return sm_unit_k<QLIN_Q5_G64>();
    case QLIN_Q3_G64: return sm_unit_k<QLIN_Q3_G64>();
    case QLIN_Q6_G64: return sm_unit_k<QLIN_Q6_G64>();
    case QLIN_Q8_G32: return sm_unit_k<QLIN_Q8_G32>();
    case QLIN_FP8_ROW: return sm_unit_k<QLIN_FP8_ROW>();
    default: return sm_unit_k<QLIN_BF16>();
  }
}

template <int FMT, int T>
int launch_t(const CUtensorMap& mc, const CUtensorMap& mh, const CUtensorMap& mx, const SmArgs& a,
             int grid, cudaStream_t st) {
  using C = SmCfg<FMT, T>;
  auto kern = gemv_sm_kernel<FMT, T>;
  const cudaError_t e = set_smem_once<gemv_sm_kernel<FMT, T>>((int)C::SMEM);
  if (e != cudaSuccess) return cuda_status(e);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(C::THREADS);
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
int launch_fmt_sm(int64_t t, const CUtensorMap& mc, const CUtensorMap& mh, const CUtensorMap& mx,
                  const SmArgs& a, int grid, cudaStream_t st) {
  (void)t;  // T == 1 (gemv_sm_supported)
  return launch_t<FMT, 1>(mc, mh, mx, a, grid, st);
}

}  // namespace

// T = 1 with rows of whole units (K a multiple of 512 for Q4/Q5 and of 256
// for Q8/FP8, 128 for BF16).  (Measured on B200: from T = 2 on, the
// tensor-core kernel is faster.)
bool gemv_sm_supported(const qlin_weights& w, int64_t t) {
  if (t != 1) return false;
  return w.k % unit_k_sm(w.fmt) == 0;
}

size_t gemv_sm_workspace_bytes(const qlin_weights& w, int64_t t, int num_sms) {
  const int64_t tiles = (w.n + 127) / 128;
  const size_t counters = ((size_t)tiles * sizeof(int) + 255) / 256 * 256;
  return counters + (size_t)num_sms * 2 * t * 128 * sizeof(float);
}

int launch_gemv_sm(const qlin_weights& w, const uint16_t* x, int64_t t, void* y, int y_dtype,
                   const Exec& ex) {
  const int64_t tiles = (w.n + 127) / 128;
  const int64_t kc = unit_k_sm(w.fmt);
  const int64_t cpt = w.k / kc;
  const int64_t units = tiles * cpt;
  const int grid = (int)std::min<int64_t>(ex.num_sms, units);
  const int64_t row_bytes = code_row_bytes(w.fmt, w.k);
  CUtensorMap mc, mh, mx;
  int rc = encode_tmap_2d(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, w.codes, (uint64_t)row_bytes,
                          (uint64_t)w.n, (uint64_t)row_bytes, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return rc;
  rc = encode_tmap_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, (uint64_t)w.k, (uint64_t)t,
                      (uint64_t)w.k * 2, 64, (uint32_t)t, CU_TENSOR_MAP_SWIZZLE_NONE);
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
  SmArgs a;
  a.scales = w.scales;
  a.y = y;
  const size_t counters = ((size_t)tiles * sizeof(int) + 255) / 256 * 256;
  a.counters = (int*)ex.workspace;
  a.partials = (float*)((uint8_t*)ex.workspace + counters);
  a.dev_status = ex.dev_status;
  a.n = w.n;
  a.k = w.k;
  a.cpt = cpt;
  a.units = units;
  a.y_dtype = y_dtype;
  switch (w.fmt) {
    case QLIN_Q4_G64: return launch_fmt_sm<QLIN_Q4_G64>(t, mc, mh, mx, a, grid, ex.stream);
    case QLIN_Q5_G64: return launch_fmt_sm<QLIN_Q5_G64>(t, mc, mh, mx, a, grid, ex.stream);
    case QLIN_Q3_G64: return launch_fmt_sm<QLIN_Q3_G64>(t, mc, mh, mx, a, grid, ex.stream);
    case QLIN_Q6_G64: return launch_fmt_sm<QLIN_Q6_G64>(t, mc, mh, mx, a, grid, ex.stream);
    case QLIN_Q8_G32: return launch_fmt_sm<QLIN_Q8_G32>(t, mc, mh, mx, a, grid, ex.stream);
    case QLIN_FP8_ROW: return launch_fmt_sm<QLIN_FP8_ROW>(t, mc, mh, mx, a, grid, ex.stream);
    default: return launch_fmt_sm<QLIN_BF16>(t, mc, mh, mx, a, grid, ex.stream);
  }
}

}  // namespace qlin
