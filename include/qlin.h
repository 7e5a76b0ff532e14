/*
 * qlin.h -- C ABI of the quantized-linear library for one NVIDIA B200 (sm_100a).
 *
 * The library computes the linear projections of a 27B-class decoder whose
 * weights are stored quantized, as the NInfer artifact pages describe them:
 *   - groupwise Q4 / Q5 codes with one FP16 scale per 64 columns
 *     ["Qwen3.8-27B for NInfer -- RTX 5080 16 GB", "Quantization profile":
 *      Q4G64_F16S, Q5G64_F16S; "Qwen3.8-27B-NVIDIA-NVFP4-NInferV3",
 *      "What is in the file": grouped Q4/Q5/Q8 with FP16 scales];
 *   - Q8 codes with one FP16 scale per 32 columns
 *     ["Qwen3.8-27B EfficientThink-Uncensored FP8 for NInfer", intro: Q8 group-32];
 *   - E4M3 codes with one BF16 scale per output row, fp8_row_maxabs
 *     [same page, "Conversion and verification"];
 *   - plain BF16 weights (the GDN a/b projections kept unquantized)
 *     [same page, "Conversion and verification"; "...NVFP4-NInferV3",
 *      "How it was created"].
 * Decode, MTP and verify steps (T = 1..33 tokens) run the BF16 route:
 * weights are dequantized on the fly and multiplied with BF16 activations
 * ["NInfer int8-prefill artifact for the RTX 4090", "What changes":
 * decode keeps the BF16 route].  Prefill steps may run the int8 route:
 * activations are quantized per token and per 64 channels with scale =
 * amax / 127, integer MMAs give one int32 sum per group and each sum is
 * scaled by weight_scale x activation_scale in FP32 [same page, "What changes"].
 *
 * Conventions (all entry points):
 *   - Every call returns an int status (QLIN_OK or a QLIN_ERR_* code) and
 *     never aborts or throws.  qlin_status_string() gives the text.
 *   - Every array argument is a DEVICE pointer, allocated and owned by the
 *     caller; the library never allocates.  Scratch memory is the caller's
 *     `qlin_exec.workspace`, sized by the *_workspace_bytes queries.
 *   - Work is enqueued asynchronously on `qlin_exec.stream` (NULL = the
 *     legacy default stream).  Argument checks happen on the host before
 *     anything is enqueued; a rejected call enqueues nothing.
 *   - Every device array must start on a 16-byte boundary (TMA rule), and
 *     K must be a multiple of the format's group (64 for Q3/Q4/Q5/Q6, 32 for Q8,
 *     32 for MXFP8 sources, 128 for MLX affine sources, 64 for BF16/FP8 rows).
 *   - Kernels that wait on on-chip barriers bound every wait.  A wait that
 *     runs out stores QLIN_ERR_TIMEOUT into `*qlin_exec.dev_status` (when the
 *     pointer is non-NULL) and the kernel returns early; the host sees it
 *     after synchronizing the stream.  The output is then undefined.
 *
 * Layouts of the packed formats (this library's own; the pages fix code
 * widths, group sizes and scale types only):
 *   Q4_G64  codes  uint8[N][K/2].  Each row is read as K/8 little-endian
 *           32-bit words.  Word j holds elements 8j..8j+7: element 8j+2s
 *           (s = 0..3) in bits [4s, 4s+4) and element 8j+2s+1 in bits
 *           [16+4s, 16+4s+4), as the offset code u = q + 8, q in [-8, 7].
 *           scales binary16[N][K/64].
 *   Q5_G64  codes as Q4 holding the low 4 bits of u = q + 16, q in [-16, 15];
 *           hibits uint8[N][K/8], read as K/32 little-endian words; in word h
 *           element 32h + 8jj + 2s + o (jj, s in 0..3, o in 0..1) keeps bit 4
 *           of its u at bit 16*o + 4*jj + s.  scales binary16[N][K/64].
 *   Q8_G32  codes int8[N][K] (two's complement, q in [-128, 127]);
 *           scales binary16[N][K/32].
 *   FP8_ROW codes E4M3 bytes [N][K]; scales bfloat16[N] (one per row).
 *   BF16    codes bfloat16[N][K]; no scales.
 *   Q3_G64  u = q + 4, q in [-4, 3] (scale amax / 3).  codes uint8[N][K/4],
 *           the crumb plane of bits 0..1 of u: read as K/16 little-endian
 *           words, word c holds element 16c + 2s + o (s in 0..7, o in 0..1)
 *           in bits [16o + 2s, 16o + 2s + 2); hibits uint8[N][K/8], bit 2 of
 *           u laid out as Q5's high-bit plane.  scales binary16[N][K/64].
 *   Q6_G64  u = q + 32, q in [-32, 31] (scale amax / 31).  codes as Q4
 *           holding bits 0..3 of u; hibits uint8[N][K/4], bits 4..5 of u in
 *           the crumb layout of Q3's codes.  scales binary16[N][K/64].
 *           ["Qwen3.8-27B for NInfer -- RTX 5080 16 GB", "Quantization
 *           profile": Q3G64_F16S; "Qwen3.8-27B MXFP8-CRACK -- NInfer
 *           artifact", "Caveats": Q6 groupwise.  The code widths and group
 *           size are the pages'; Qmax = 2^(bits-1) - 1 and the planes are this
 *           library's reading.]
 * Activations x are bfloat16[T][K] row-major; outputs y are [T][N] row-major
 * in bfloat16 or float32 (y[t][n] = sum_k w[n][k] * x[t][k]).
 */
#ifndef QLIN_H
#define QLIN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QLIN_API __attribute__((visibility("default")))
#else
#define QLIN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------- */
#define QLIN_OK 0
#define QLIN_ERR_INVALID_ARG 1   /* null / misaligned pointer, bad size or enum   */
#define QLIN_ERR_UNSUPPORTED 2   /* valid request this library does not serve     */
#define QLIN_ERR_NOT_PERMITTED 3 /* int8 route on weights without QLIN_ALLOW_A8   */
#define QLIN_ERR_CUDA 4          /* a CUDA runtime / driver call failed           */
#define QLIN_ERR_TIMEOUT 5       /* (device status) a bounded on-chip wait ran out */
#define QLIN_ERR_WORKSPACE 6     /* workspace missing or smaller than required    */

/* ---- weight formats ----------------------------------------------------- */
#define QLIN_Q4_G64 0
#define QLIN_Q5_G64 1
#define QLIN_Q8_G32 2
#define QLIN_FP8_ROW 3
#define QLIN_BF16 4
#define QLIN_Q3_G64 5
#define QLIN_Q6_G64 6

/* ---- weight sources for qlin_pack_weights ------------------------------- */
#define QLIN_SRC_F32 0         /* float32[N][K]                                 */
#define QLIN_SRC_BF16 1        /* bfloat16[N][K]                                */
#define QLIN_SRC_MXFP8 2       /* uint32 words[N][K/4] + uint8 UE8M0 [N][K/32]  */
#define QLIN_SRC_MLX_AFFINE8 3 /* uint8 q[N][K] + f16 scale, f16 bias [N][K/128]*/
#define QLIN_SRC_FP8_BLOCK128 4 /* E4M3 uint8[N][K] + float32 [ceil(N/128)][ceil(K/128)] */

/* ---- output dtypes ------------------------------------------------------ */
#define QLIN_OUT_BF16 0
#define QLIN_OUT_F32 1

/* ---- flags -------------------------------------------------------------- */
#define QLIN_ALLOW_A8 0x1u         /* qlin_weights.flags: object may take the int8 route */
#define QLIN_DEBUG_GROUP_SUMS 0x1u /* qlin_gemm_a8 flags: also dump int32 group sums   */

/* Execution context of one call.  All members are optional except as noted. */
typedef struct {
  void* stream;             /* cudaStream_t to enqueue on; NULL = legacy default */
  int32_t* dev_status;      /* device int32; receives QLIN_ERR_TIMEOUT on a timed-out
                               on-chip wait; never cleared by the library            */
  void* workspace;          /* device scratch owned by the caller                    */
  size_t workspace_bytes;   /* its size                                              */
} qlin_exec;

/* A packed weight matrix W[N][K] (caller-owned device buffers). */
typedef struct {
  int32_t fmt;     /* QLIN_Q4_G64 .. QLIN_BF16                                  */
  uint32_t flags;  /* QLIN_ALLOW_A8: activation permission (A16Only when clear)  */
  int64_t n, k;    /* output rows, input columns                                */
  void* codes;     /* see the layouts above                                     */
  void* hibits;    /* Q5_G64 only, else NULL                                    */
  void* scales;    /* NULL for BF16                                             */
} qlin_weights;

/* Text for a status code; never NULL. */
QLIN_API const char* qlin_status_string(int status);

/* Sizes in bytes of the three buffers of a packed matrix (0 when unused).
 * Returns QLIN_ERR_INVALID_ARG for an unknown format, n <= 0, or K not a
 * multiple of the format's group. */
QLIN_API int qlin_packed_bytes(int fmt, int64_t n, int64_t k, size_t* codes_bytes, size_t* hibits_bytes,
                      size_t* scales_bytes);

/* Quantize (or re-encode) a source matrix into dst->fmt, on the device.
 * Source values are first taken to numbers exactly as the pages describe:
 *   F32   used as is; BF16 widened exactly;
 *   MXFP8 4 x E4M3 per U32 word (element 4i+j = byte j of word i), value =
 *         E4M3 * 2^(b-127) rounded once to BF16 ["MXFP8-CRACK NInfer
 *         artifact", "How it was built", step 1]; `src_aux0` = UE8M0 scales;
 *   MLX_AFFINE8  w = q * scale + bias as one FP32 fused multiply-add, rounded
 *         to BF16 [same page, step 2]; `src_aux0` = f16 scales, `src_aux1` =
 *         f16 biases, one per 128 columns.
 *   FP8_BLOCK128  E4M3 codes uint8[N][K] with one float32 scale per 128 x 128
 *         block (`src_aux0` = the weight_scale_inv grid, row-major
 *         [ceil(N/128)][ceil(K/128)]): value = E4M3 * scale as one FP32
 *         multiplication (exact when the scale has at most 20 significant
 *         bits, e.g. a BF16 scale), rounded to BF16; an E4M3 NaN code gives
 *         0x7FC0 with its sign ["...EfficientThink-Uncensored FP8 for NInfer",
 *         "Conversion and verification": block-wise to per-row].  With
 *         dst->fmt = FP8_ROW this is the page's re-encode to one BF16 scale
 *         per row.
 * Then quantized: Q4/Q5/Q8: per (row, group) s = FP16_rne(amax / Qmax) with
 * Qmax = 7 / 15 / 127 and q = clamp(rint(w / s)) against the stored scale
 * (0 when s == 0).  FP8_ROW: sc = BF16_rne(rowmax|w| / 448), code =
 * E4M3_rne_satfinite(w / sc) (0 when sc == 0) ["...FP8 for NInfer",
 * "Conversion and verification", fp8_row_maxabs].  BF16: BF16_rne(w).
 * dst must describe preallocated buffers of qlin_packed_bytes() sizes.
 * Bit-exact with the library's CPU oracle. */
QLIN_API int qlin_pack_weights(int src_kind, const void* src, const void* src_aux0, const void* src_aux1,
                      const qlin_weights* dst, const qlin_exec* ex);

/* MXFP8 -> BF16 decode of a [rows][cols] matrix (cols % 32 == 0).
 * words uint32[rows][cols/4], scales uint8[rows][cols/32], out bfloat16[rows][cols].
 * b == 255 or an E4M3 NaN gives 0x7FC0 with the element's sign bit.
 * ["MXFP8-CRACK NInfer artifact", "How it was built", step 1.]  Bit-exact. */
QLIN_API int qlin_decode_mxfp8(const uint32_t* words, const uint8_t* scales, int64_t rows, int64_t cols,
                      uint16_t* out_bf16, const qlin_exec* ex);

/* Per-token, per-64-channel activation quantization of x bfloat16[T][K]:
 * xs[t][g] = amax / 127 (FP32) and xq[t][k] = clamp(rint(x / xs), -127, 127)
 * (0 when xs == 0).  xq int8[T][K], xs float32[T][K/64].  K % 64 == 0.
 * ["NInfer int8-prefill artifact for the RTX 4090", "What changes".]  Bit-exact. */
QLIN_API int qlin_quantize_act(const uint16_t* x_bf16, int64_t t, int64_t k, int8_t* xq, float* xs,
                      const qlin_exec* ex);

/* Workspace bytes qlin_gemv needs for these weights and T (may be 0). */
QLIN_API int qlin_gemv_workspace_bytes(const qlin_weights* w, int64_t t, size_t* bytes);

/* BF16-route projection y[T][N] = x[T][K] * W^T with on-the-fly dequantization
 * (decode / MTP / verify steps).  Q4/Q5/Q8/FP8_ROW: 1 <= T <= 64
 * (QLIN_ERR_UNSUPPORTED above); BF16 weights: any T >= 1.  FP32 accumulation;
 * y_dtype QLIN_OUT_BF16 (RNE) or QLIN_OUT_F32.  The workspace must hold
 * qlin_gemv_workspace_bytes() and be zero-filled before its first use with
 * this library; every call that completes leaves its counters at zero again.
 * After a call that reported QLIN_ERR_TIMEOUT its split-tile counters may be
 * left non-zero: zero-fill the workspace again before its next use
 * (qlin_gemv_noalloc clears its own counters on every call).
 * Ordering: the kernels are launched with programmatic dependent launch, so
 * they may start, and read the packed weights, while the kernel ahead of them
 * on `stream` is still finishing (when that kernel allows it); x, y and the
 * workspace are touched only once it has completed.  The weights must not be
 * written by a kernel that is still running.
 * Accuracy: |y - y_ref| <= 1e-3 * sum_k |w||x| per element (plus the BF16
 * output rounding).  ["NInfer int8-prefill artifact for the RTX 4090",
 * "What changes": decode keeps the BF16 route; "...NVFP4-NInferV3", "How it
 * was created": the FP8 head op over T = 1..33.] */
QLIN_API int qlin_gemv(const qlin_weights* w, const uint16_t* x_bf16, int64_t t, void* y, int y_dtype,
              const qlin_exec* ex);

/* Workspace bytes qlin_gemm_a8 should get for T tokens against an N x K
 * matrix: the activation codes and scales (T*K + T*K/64*4 bytes, 256-byte
 * aligned; the least a call with x_bf16 accepts) plus the weights expanded to
 * int8 once per call (N*K bytes) and the split-tile counters and FP32 partial
 * tiles of its stream-K schedule (64 bytes per 128x128 tile and 128 KB per SM
 * of the current device; sized for 256 SMs when no device is visible).  With
 * the full size the GEMM reads int8 weights through TMA (the faster kernel);
 * with less, or none when the activations come pre-quantized, it expands the
 * codes on chip.  No part of it needs to be zero-filled. */
QLIN_API int qlin_gemm_a8_workspace_bytes(int64_t t, int64_t n, int64_t k, size_t* bytes);

/* Int8-route projection (prefill).  Weights must be Q3_G64, Q4_G64, Q5_G64 or Q6_G64
 * (QLIN_ERR_UNSUPPORTED otherwise) carrying QLIN_ALLOW_A8
 * (QLIN_ERR_NOT_PERMITTED otherwise) and K % 128 == 0 (QLIN_ERR_UNSUPPORTED
 * otherwise).  Activations either as x_bf16 (the
 * per-token per-64 quantizer runs inside the call, xq/xs must be NULL) or
 * pre-quantized as xq int8[T][K] + xs float32[T][K/64] (x_bf16 NULL).
 * S[t][n][g] = sum over the group of xq * q (int32, exact);
 * y[t][n] = sum_g (FP32(ws[n][g] * xs[t][g])) * S accumulated in FP32.
 * With flags & QLIN_DEBUG_GROUP_SUMS, S is also written to group_sums_dbg
 * int32[T][N][K/64].  The routing policy (T >= 129) is the caller's.  The
 * workspace (see qlin_gemm_a8_workspace_bytes) is read and written; it must
 * hold the activation part when x_bf16 is given (QLIN_ERR_WORKSPACE otherwise).
 * Accuracy: |y - y_ref| <= 5e-6 * sum_k |q ws||qa as| per element before the
 * BF16 output rounding.  ["NInfer int8-prefill artifact for the RTX 4090",
 * "What changes".] */
QLIN_API int qlin_gemm_a8(const qlin_weights* w, const uint16_t* x_bf16, const int8_t* xq, const float* xs,
                 int64_t t, void* y, int y_dtype, uint32_t flags, int32_t* group_sums_dbg,
                 const qlin_exec* ex);

/* Per-token FP8 activation quantization of x bfloat16[T][K] for the
 * FP8-activation route: xs[t] = max_k |x[t][k]| / 448 (FP32, IEEE division)
 * and xq[t][k] = E4M3(x / xs) rounded to nearest even with saturation to
 * +-448 (all zero when xs == 0).  xq uint8[T][K] (E4M3 bytes), xs
 * float32[T].  K % 16 == 0.  ["Qwen3.8-27B EfficientThink-Uncensored FP8 for
 * NInfer", "Conversion and verification" and "Hardware fit": row-scaled FP8
 * weights run on FP8-activation tensor-core routes; the page fixes no
 * activation scheme, and one FP32 scale per token mirrors fp8_row_maxabs on
 * the activation side.]  Bit-exact. */
QLIN_API int qlin_quantize_act_fp8(const uint16_t* x_bf16, int64_t t, int64_t k, uint8_t* xq, float* xs,
                                   const qlin_exec* ex);

/* Workspace bytes qlin_gemm_fp8 needs when it quantizes T x K activations itself. */
QLIN_API int qlin_gemm_fp8_workspace_bytes(int64_t t, int64_t k, size_t* bytes);

/* FP8-activation projection (prefill and decode) for FP8_ROW weights
 * (QLIN_ERR_UNSUPPORTED for any other format), any T >= 1.  Activations
 * either as x_bf16 (qlin_quantize_act_fp8 runs inside the call into the
 * workspace, xq/xs must be NULL) or pre-quantized as xq uint8[T][K] +
 * xs float32[T] (x_bf16 NULL; no workspace needed).
 * y[t][n] = FP32(ws[n] * xs[t]) * sum_k E4M3(w[n][k]) * E4M3(xq[t][k]),
 * the products exact and the sum accumulated in FP32 on the tensor cores.
 * Accuracy: |y - y_ref| <= 1e-5 * |ws xs| sum_k |w||xq| per element before
 * the BF16 output rounding, y_ref the exact product of the same codes.
 * [Same page, "Hardware fit".] */
QLIN_API int qlin_gemm_fp8(const qlin_weights* w, const uint16_t* x_bf16, const uint8_t* xq, const float* xs,
                           int64_t t, void* y, int y_dtype, const qlin_exec* ex);

/* qlin_gemv without a caller workspace.  The pages have no counterpart: this
 * entry point exists for callers that cannot allocate device memory when they
 * call (memory planned once at start-up; plain C code owning only w, x and y).
 * Same arguments, results, limits and errors as qlin_gemv (stream is a
 * cudaStream_t or NULL, dev_status as qlin_exec.dev_status, may be NULL); the
 * scratch qlin_gemv would take from qlin_exec.workspace comes instead from a
 * fixed 16 MiB device array inside the library, one per device.
 * Argument errors are reported exactly as qlin_gemv reports them, before
 * anything is enqueued (quantized weights with T > 64: QLIN_ERR_UNSUPPORTED).
 * Requests whose qlin_gemv_workspace_bytes() exceeds 16 MiB return
 * QLIN_ERR_WORKSPACE.  The tensor-core kernels need at most a few MiB at
 * T <= 64; a matrix whose K is not a whole number of the kernels' column
 * units (and is above 2048) runs on the CUDA-core kernel, which needs
 * T * N * 4 bytes: e.g. Q4 152064 x 5184 at T = 64 needs 39 MB and is refused.
 * The first call on a device resolves the array's address and zero-fills it
 * (synchronously); make that first call before any stream capture.  Each call
 * clears the array's split-tile counters on `stream` before its kernels.
 * The array is shared by all calls on a device: calls that may overlap in time
 * (other streams or host threads) race on it and must be serialized by the
 * caller.  Allocates nothing. */
QLIN_API int qlin_gemv_noalloc(const qlin_weights* w, const uint16_t* x_bf16, int64_t t, void* y,
                               int y_dtype, void* stream, int32_t* dev_status);

#ifdef __cplusplus
}
#endif
#endif /* QLIN_H */
