// C ABI entry points (include/qlin.h): argument validation on the host, then
// dispatch to the kernel launchers.  Nothing here allocates device memory.
#include <cudaTypedefs.h>

#include <atomic>
#include <mutex>

#include "qlin_internal.cuh"

namespace qlin {

size_t gemv_cc_workspace_bytes(const qlin_weights& w, int64_t t);
int launch_gemv_cc(const qlin_weights& w, const uint16_t* x, int64_t t, void* y, int y_dtype,
                   const Exec& ex, float* acc_ws);
bool gemv_tc_supported(const qlin_weights& w, int64_t t);
bool gemv_sm_supported(const qlin_weights& w, int64_t t);
size_t gemv_sm_workspace_bytes(const qlin_weights& w, int64_t t, int num_sms);
int launch_gemv_sm(const qlin_weights& w, const uint16_t* x, int64_t t, void* y, int y_dtype,
                   const Exec& ex);
size_t gemv_tc_workspace_bytes(const qlin_weights& w, int64_t t, int num_sms);
int launch_gemv_tc(const qlin_weights& w, const uint16_t* x, int64_t t, void* y, int y_dtype,
                   const Exec& ex);
bool gemm_bf16_tok_supported(const qlin_weights& w, int64_t t);
size_t gemm_bf16_tok_workspace_bytes(const qlin_weights& w, int64_t t, int num_sms);
int launch_gemm_bf16_tok(const qlin_weights& w, const uint16_t* x, int64_t t, void* y, int y_dtype,
                         const Exec& ex);
bool gemv_f16_supported(const qlin_weights& w, int64_t t);
size_t gemv_f16_workspace_bytes(const qlin_weights& w, int64_t t, int num_sms);
int launch_gemv_f16(const qlin_weights& w, const uint16_t* x, int64_t t, void* y, int y_dtype,
                    const Exec& ex);

namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// SM count per device, queried once (0 = not yet known).
std::atomic<int> g_num_sms[64];

int make_exec(const qlin_exec* e, Exec* out) {
  out->stream = e ? (cudaStream_t)e->stream : (cudaStream_t)0;
  out->dev_status = e ? e->dev_status : nullptr;
  out->workspace = e ? e->workspace : nullptr;
  out->workspace_bytes = e ? e->workspace_bytes : 0;
  if (out->workspace && !aligned16(out->workspace)) return QLIN_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QLIN_ERR_CUDA;
  const bool cacheable = dev >= 0 && dev < 64;
  int sms = cacheable ? g_num_sms[dev].load(std::memory_order_relaxed) : 0;
  if (sms <= 0) {
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return QLIN_ERR_CUDA;
    if (cacheable) g_num_sms[dev].store(sms, std::memory_order_relaxed);
  }
  out->num_sms = sms;
  return QLIN_OK;
}

// Encoded tensor maps of recent calls, per host thread: a decode loop calls
// the same few projections over and over, and an encode costs about a
// microsecond of driver time.  The key is every argument of the encode; a
// cached map is only reused for the identical request.
struct TmapKey {
  const void* base;
  uint64_t inner, outer, stride;
  uint32_t box_inner, box_outer;
  int dtype, swizzle;
  bool operator==(const TmapKey& o) const {
    return base == o.base && inner == o.inner && outer == o.outer && stride == o.stride &&
           box_inner == o.box_inner && box_outer == o.box_outer && dtype == o.dtype &&
           swizzle == o.swizzle;
  }
};
constexpr int kTmapCache = 32;
struct TmapCache {
  TmapKey key[kTmapCache];
  CUtensorMap map[kTmapCache];
  bool used[kTmapCache] = {};
  int next = 0;
};
thread_local TmapCache t_tmaps;

int group_of(int fmt) {
  switch (fmt) {
    case QLIN_Q3_G64:
    case QLIN_Q4_G64:
    case QLIN_Q5_G64:
    case QLIN_Q6_G64:
    case QLIN_FP8_ROW:
    case QLIN_BF16:
      return 64;
    case QLIN_Q8_G32:
      return 32;
    default:
      return 0;
  }
}

int sizes_of(int fmt, int64_t n, int64_t k, size_t* c, size_t* h, size_t* s) {
  int g = group_of(fmt);
  if (g == 0 || n <= 0 || k <= 0 || k % g != 0) return QLIN_ERR_INVALID_ARG;
  size_t cb = 0, hb = 0, sb = 0;
  switch (fmt) {
    case QLIN_Q4_G64: cb = (size_t)n * (k / 2); sb = (size_t)n * (k / 64) * 2; break;
    case QLIN_Q5_G64: cb = (size_t)n * (k / 2); hb = (size_t)n * (k / 8); sb = (size_t)n * (k / 64) * 2; break;
    case QLIN_Q3_G64: cb = (size_t)n * (k / 4); hb = (size_t)n * (k / 8); sb = (size_t)n * (k / 64) * 2; break;
    case QLIN_Q6_G64: cb = (size_t)n * (k / 2); hb = (size_t)n * (k / 4); sb = (size_t)n * (k / 64) * 2; break;
    case QLIN_Q8_G32: cb = (size_t)n * k; sb = (size_t)n * (k / 32) * 2; break;
    case QLIN_FP8_ROW: cb = (size_t)n * k; sb = (size_t)n * 2; break;
    case QLIN_BF16: cb = (size_t)n * k * 2; break;
  }
  if (c) *c = cb;
  if (h) *h = hb;
  if (s) *s = sb;
  return QLIN_OK;
}

int check_weights(const qlin_weights* w) {
  if (!w) return QLIN_ERR_INVALID_ARG;
  size_t c, h, s;
  int rc = sizes_of(w->fmt, w->n, w->k, &c, &h, &s);
  if (rc) return rc;
  if (!w->codes || !aligned16(w->codes)) return QLIN_ERR_INVALID_ARG;
  if (h && (!w->hibits || !aligned16(w->hibits))) return QLIN_ERR_INVALID_ARG;
  if (s && (!w->scales || !aligned16(w->scales))) return QLIN_ERR_INVALID_ARG;
  return QLIN_OK;
}

}  // namespace

int encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner,
                   uint64_t outer, uint64_t row_stride_bytes, uint32_t box_inner,
                   uint32_t box_outer, CUtensorMapSwizzle swizzle) {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = (PFN_cuTensorMapEncodeTiled_v12000)fn;
  });
  if (!g_encode) return QLIN_ERR_CUDA;
  const TmapKey key{base, inner, outer, row_stride_bytes, box_inner, box_outer, (int)dtype, (int)swizzle};
  TmapCache& c = t_tmaps;
  for (int i = 0; i < kTmapCache; ++i)
    if (c.used[i] && c.key[i] == key) {
      *map = c.map[i];
      return QLIN_OK;
    }
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return QLIN_ERR_CUDA;
  const int slot = c.next;
  c.next = (c.next + 1) % kTmapCache;
  c.key[slot] = key;
  c.map[slot] = *map;
  c.used[slot] = true;
  return QLIN_OK;
}

// Kernel choice (measured on B200, calls queued, L2 flushed):
//  - FP8-row weights, and Q8 group-32 matrices of at least 2^27 weights (the
//    output head): gemv_f16 (group scale folded into an FP16 A operand, one
//    accumulator per tile segment): E4M3 and Q8 expand in few instructions,
//    and the fixed per-call costs are spread over many units;
//  - Q4 / Q5 and the smaller Q8 matrices: T = 1 on the CUDA cores (gemv_sm),
//    2 <= T <= 64 on gemv_tc (exact BF16 integer codes, one FP32 sum per
//    group scaled in the epilogue): the nibble expansion of gemv_f16 costs
//    about 13 instructions per 32-bit word, which made it slower there;
//  - BF16 weights: gemv_tc up to 64 tokens; above that, with N <= 256 (the
//    GDN a/b projection at prefill), gemm_bf16_tok: tokens on the MMA's M
//    side, K split over CTAs until every SM streams a share of x; larger N in
//    64-token gemv_tc chunks;
//  - rows that are not whole units: the CUDA-core kernel.
constexpr int64_t kTcMaxT = 64;
static bool bf16_chunked(const qlin_weights& w, int64_t t) {
  return w.fmt == QLIN_BF16 && t > kTcMaxT && gemv_tc_supported(w, kTcMaxT);
}
static bool use_f16(const qlin_weights& w, int64_t t) {
  const bool wanted = w.fmt == QLIN_FP8_ROW || (w.fmt == QLIN_Q8_G32 && w.n * w.k >= ((int64_t)1 << 27));
  return wanted && gemv_f16_supported(w, t);
}

size_t gemv_workspace_bytes(const qlin_weights& w, int64_t t, int num_sms) {
  if (gemm_bf16_tok_supported(w, t)) return gemm_bf16_tok_workspace_bytes(w, t, num_sms);
  if (use_f16(w, t)) return gemv_f16_workspace_bytes(w, t, num_sms);
  if (gemv_sm_supported(w, t)) return gemv_sm_workspace_bytes(w, t, num_sms);
  if (bf16_chunked(w, t)) return gemv_tc_workspace_bytes(w, kTcMaxT, num_sms);
  if (gemv_tc_supported(w, t)) return gemv_tc_workspace_bytes(w, t, num_sms);
  return gemv_cc_workspace_bytes(w, t);
}

int launch_gemv(const qlin_weights& w, const uint16_t* x, int64_t t, void* y, int y_dtype,
                const Exec& ex) {
  if (gemm_bf16_tok_supported(w, t)) return launch_gemm_bf16_tok(w, x, t, y, y_dtype, ex);
  if (use_f16(w, t)) return launch_gemv_f16(w, x, t, y, y_dtype, ex);
  if (gemv_sm_supported(w, t)) return launch_gemv_sm(w, x, t, y, y_dtype, ex);
  if (bf16_chunked(w, t)) {
    const size_t ysz = y_dtype == QLIN_OUT_F32 ? 4 : 2;
    for (int64_t t0 = 0; t0 < t; t0 += kTcMaxT) {
      const int64_t tc = t - t0 < kTcMaxT ? t - t0 : kTcMaxT;
      const int rc = launch_gemv_tc(w, x + t0 * w.k, tc, (uint8_t*)y + (size_t)t0 * w.n * ysz, y_dtype, ex);
      if (rc != QLIN_OK) return rc;
    }
    return QLIN_OK;
  }
  if (gemv_tc_supported(w, t)) return launch_gemv_tc(w, x, t, y, y_dtype, ex);
  return launch_gemv_cc(w, x, t, y, y_dtype, ex, (float*)ex.workspace);
}

// Host checks of qlin_gemv's arguments (shared with qlin_gemv_noalloc, which
// must reject a call before it enqueues anything).
int check_gemv_args(const qlin_weights* w, const uint16_t* x_bf16, int64_t t, const void* y,
                    int y_dtype) {
  int rc = check_weights(w);
  if (rc) return rc;
  if (!x_bf16 || !y || t <= 0 || !aligned16(x_bf16) || !aligned16(y)) return QLIN_ERR_INVALID_ARG;
  if (y_dtype != QLIN_OUT_BF16 && y_dtype != QLIN_OUT_F32) return QLIN_ERR_INVALID_ARG;
  if (w->fmt != QLIN_BF16 && t > 64) return QLIN_ERR_UNSUPPORTED;
  return QLIN_OK;
}

}  // namespace qlin

using namespace qlin;

extern "C" {

const char* qlin_status_string(int status) {
  switch (status) {
    case QLIN_OK: return "ok";
    case QLIN_ERR_INVALID_ARG: return "invalid argument";
    case QLIN_ERR_UNSUPPORTED: return "unsupported request";
    case QLIN_ERR_NOT_PERMITTED: return "int8 route not permitted for these weights";
    case QLIN_ERR_CUDA: return "CUDA error";
    case QLIN_ERR_TIMEOUT: return "a bounded device wait timed out";
    case QLIN_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

int qlin_packed_bytes(int fmt, int64_t n, int64_t k, size_t* codes_bytes, size_t* hibits_bytes,
                      size_t* scales_bytes) {
  return sizes_of(fmt, n, k, codes_bytes, hibits_bytes, scales_bytes);
}

int qlin_pack_weights(int src_kind, const void* src, const void* src_aux0, const void* src_aux1,
                      const qlin_weights* dst, const qlin_exec* ex) {
  int rc = check_weights(dst);
  if (rc) return rc;
  if (!src || !aligned16(src)) return QLIN_ERR_INVALID_ARG;
  switch (src_kind) {
    case QLIN_SRC_F32:
    case QLIN_SRC_BF16:
      break;
    case QLIN_SRC_MXFP8:
      if (dst->k % 32 || !src_aux0 || !aligned16(src_aux0)) return QLIN_ERR_INVALID_ARG;
      break;
    case QLIN_SRC_MLX_AFFINE8:
      if (dst->k % 128 || !src_aux0 || !src_aux1 || !aligned16(src_aux0) || !aligned16(src_aux1))
        return QLIN_ERR_INVALID_ARG;
      break;
    case QLIN_SRC_FP8_BLOCK128:
      if (!src_aux0 || !aligned16(src_aux0)) return QLIN_ERR_INVALID_ARG;
      break;
    default:
      return QLIN_ERR_INVALID_ARG;
  }
  Exec e;
  if ((rc = make_exec(ex, &e))) return rc;
  return launch_pack(src_kind, src, src_aux0, src_aux1, *dst, e);
}

int qlin_decode_mxfp8(const uint32_t* words, const uint8_t* scales, int64_t rows, int64_t cols,
                      uint16_t* out_bf16, const qlin_exec* ex) {
  if (!words || !scales || !out_bf16 || rows <= 0 || cols <= 0 || cols % 32) return QLIN_ERR_INVALID_ARG;
  if (!aligned16(words) || !aligned16(out_bf16)) return QLIN_ERR_INVALID_ARG;
  Exec e;
  int rc = make_exec(ex, &e);
  if (rc) return rc;
  return launch_decode_mxfp8(words, scales, rows, cols, out_bf16, e);
}

int qlin_quantize_act(const uint16_t* x_bf16, int64_t t, int64_t k, int8_t* xq, float* xs,
                      const qlin_exec* ex) {
  if (!x_bf16 || !xq || !xs || t <= 0 || k <= 0 || k % 64) return QLIN_ERR_INVALID_ARG;
  if (!aligned16(x_bf16) || !aligned16(xq) || !aligned16(xs)) return QLIN_ERR_INVALID_ARG;
  Exec e;
  int rc = make_exec(ex, &e);
  if (rc) return rc;
  return launch_quantize_act(x_bf16, t, k, xq, xs, e);
}

int qlin_gemv_workspace_bytes(const qlin_weights* w, int64_t t, size_t* bytes) {
  int rc = check_weights(w);
  if (rc) return rc;
  if (!bytes || t <= 0) return QLIN_ERR_INVALID_ARG;
  Exec e;
  if ((rc = make_exec(nullptr, &e))) return rc;
  *bytes = gemv_workspace_bytes(*w, t, e.num_sms);
  return QLIN_OK;
}

int qlin_gemv(const qlin_weights* w, const uint16_t* x_bf16, int64_t t, void* y, int y_dtype,
              const qlin_exec* ex) {
  int rc = qlin::check_gemv_args(w, x_bf16, t, y, y_dtype);
  if (rc) return rc;
  Exec e;
  if ((rc = make_exec(ex, &e))) return rc;
  size_t need = gemv_workspace_bytes(*w, t, e.num_sms);
  if (need > e.workspace_bytes || (need && !e.workspace)) return QLIN_ERR_WORKSPACE;
  return launch_gemv(*w, x_bf16, t, y, y_dtype, e);
}

int qlin_gemm_a8_workspace_bytes(int64_t t, int64_t n, int64_t k, size_t* bytes) {
  if (!bytes || t <= 0 || n <= 0 || k <= 0 || k % 64) return QLIN_ERR_INVALID_ARG;
  // the stream-K partials are sized for the current device's SMs (256 when no
  // device is visible, which covers any current part)
  Exec e;
  const int sms = make_exec(nullptr, &e) == QLIN_OK ? e.num_sms : 256;
  (void)cudaGetLastError();
  *bytes = gemm_a8_workspace_bytes(t, n, k, sms);
  return QLIN_OK;
}

int qlin_gemm_a8(const qlin_weights* w, const uint16_t* x_bf16, const int8_t* xq, const float* xs,
                 int64_t t, void* y, int y_dtype, uint32_t flags, int32_t* group_sums_dbg,
                 const qlin_exec* ex) {
  int rc = check_weights(w);
  if (rc) return rc;
  if (w->fmt != QLIN_Q4_G64 && w->fmt != QLIN_Q5_G64 && w->fmt != QLIN_Q3_G64 && w->fmt != QLIN_Q6_G64)
    return QLIN_ERR_UNSUPPORTED;
  if (!(w->flags & QLIN_ALLOW_A8)) return QLIN_ERR_NOT_PERMITTED;
  if (w->k % 128) return QLIN_ERR_UNSUPPORTED;
  if (t <= 0 || !y || !aligned16(y)) return QLIN_ERR_INVALID_ARG;
  if (y_dtype != QLIN_OUT_BF16 && y_dtype != QLIN_OUT_F32) return QLIN_ERR_INVALID_ARG;
  const bool fused = x_bf16 != nullptr;
  if (fused == (xq != nullptr || xs != nullptr)) return QLIN_ERR_INVALID_ARG;
  if (fused && !aligned16(x_bf16)) return QLIN_ERR_INVALID_ARG;
  if (!fused && (!xq || !xs || !aligned16(xq) || !aligned16(xs))) return QLIN_ERR_INVALID_ARG;
  if ((flags & QLIN_DEBUG_GROUP_SUMS) && !group_sums_dbg) return QLIN_ERR_INVALID_ARG;
  if (t > (int64_t)INT32_MAX || w->n > (int64_t)INT32_MAX || w->k > (int64_t)INT32_MAX)
    return QLIN_ERR_UNSUPPORTED;
  Exec e;
  if ((rc = make_exec(ex, &e))) return rc;
  if (fused) {
    // at least the activation codes; the recommended size also holds the
    // weights expanded to int8 (the faster kernel)
    size_t need = gemm_a8_act_workspace_bytes(t, w->k);
    if (need > e.workspace_bytes || !e.workspace) return QLIN_ERR_WORKSPACE;
  }
  return launch_gemm_a8(*w, x_bf16, xq, xs, t, y, y_dtype, flags, group_sums_dbg, e);
}

int qlin_quantize_act_fp8(const uint16_t* x_bf16, int64_t t, int64_t k, uint8_t* xq, float* xs,
                          const qlin_exec* ex) {
  if (!x_bf16 || !xq || !xs || t <= 0 || k <= 0 || k % 16) return QLIN_ERR_INVALID_ARG;
  if (!aligned16(x_bf16) || !aligned16(xq) || !aligned16(xs)) return QLIN_ERR_INVALID_ARG;
  if (t > (int64_t)INT32_MAX) return QLIN_ERR_UNSUPPORTED;
  Exec e;
  int rc = make_exec(ex, &e);
  if (rc) return rc;
  return launch_quantize_act_fp8(x_bf16, t, k, xq, xs, e);
}

int qlin_gemm_fp8_workspace_bytes(int64_t t, int64_t k, size_t* bytes) {
  if (!bytes || t <= 0 || k <= 0 || k % 16) return QLIN_ERR_INVALID_ARG;
  *bytes = gemm_fp8_workspace_bytes(t, k);
  return QLIN_OK;
}

int qlin_gemm_fp8(const qlin_weights* w, const uint16_t* x_bf16, const uint8_t* xq, const float* xs,
                  int64_t t, void* y, int y_dtype, const qlin_exec* ex) {
  int rc = check_weights(w);
  if (rc) return rc;
  if (w->fmt != QLIN_FP8_ROW) return QLIN_ERR_UNSUPPORTED;
  if (t <= 0 || !y || !aligned16(y)) return QLIN_ERR_INVALID_ARG;
  if (y_dtype != QLIN_OUT_BF16 && y_dtype != QLIN_OUT_F32) return QLIN_ERR_INVALID_ARG;
  const bool fused = x_bf16 != nullptr;
  if (fused == (xq != nullptr || xs != nullptr)) return QLIN_ERR_INVALID_ARG;
  if (fused && !aligned16(x_bf16)) return QLIN_ERR_INVALID_ARG;
  if (!fused && (!xq || !xs || !aligned16(xq) || !aligned16(xs))) return QLIN_ERR_INVALID_ARG;
  if (t > (int64_t)INT32_MAX || w->n > (int64_t)INT32_MAX || w->k > (int64_t)INT32_MAX)
    return QLIN_ERR_UNSUPPORTED;
  Exec e;
  if ((rc = make_exec(ex, &e))) return rc;
  if (fused) {
    const size_t need = gemm_fp8_workspace_bytes(t, w->k);
    if (need > e.workspace_bytes || !e.workspace) return QLIN_ERR_WORKSPACE;
  }
  return launch_gemm_fp8(*w, x_bf16, xq, xs, t, y, y_dtype, e);
}

}  // extern "C"
