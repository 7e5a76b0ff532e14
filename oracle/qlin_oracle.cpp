// qlin oracle -- TEST INFRASTRUCTURE ONLY.
//
// A plain, slow, scalar C++ restatement of what the quantized linear path
// computes.  Only the tests, the smoke check and the bench's CPU-baseline leg
// may load it.  It shares no code, header, table or helper with the CUDA
// library: every number format below is decoded and encoded from its written
// definition (IEEE 754 binary16, bfloat16 = the top half of binary32, OCP FP8
// E4M3 "fn"), with exact double arithmetic plus one explicit rounding.
//
// Build: g++ -O2 -ffp-contract=off -fno-fast-math -shared -fPIC (see build.py).
// No FMA contraction, no fast-math: every float operation is the IEEE one.
//
// Sources (page title, section):
//   [MXFP8] "Qwen3.8-27B MXFP8-CRACK -- NInfer artifact", "How it was built",
//           step 1 (MXFP8) and step 2 (MLX affine int8).
//   [ROWFP8] "Qwen3.8-27B EfficientThink-Uncensored FP8 for NInfer",
//           "Conversion and verification" (fp8_row_maxabs, its error bound).
//   [NVFP4] "Qwen3.8-27B-NVIDIA-NVFP4-NInferV3", "What is in the file" and
//           "How it was created" (grouped Q4/Q5/Q8 with FP16 scales; head op).
//   [RTX5080] "Qwen3.8-27B for NInfer -- RTX 5080 16 GB", "Quantization
//           profile" (Q3G64_F16S, Q4G64_F16S, Q5G64_F16S).
//   [MXFP8] "Caveats" also names Q6 among the groupwise formats.
//   [A8]    "Qwen3.8-27B, NInfer int8-prefill artifact for the RTX 4090",
//           "What changes" (the int8 prefill route).
//
// Parity status per function is stated next to it ("pinned by ...").

#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <thread>
#include <vector>

namespace {

// ---------------------------------------------------------------------------
// Number formats, from their definitions.
// ---------------------------------------------------------------------------

// A binary floating-point format with `p` significant bits (implicit bit
// included), minimum normal exponent `emin`, exponent bias `bias`, `mbits`
// explicit mantissa bits and largest finite value `maxf`.
struct Fmt {
  int p, emin, bias, mbits;
  double maxf;
};
const Fmt kF16 = {11, -14, 15, 10, 65504.0};
const Fmt kBF16 = {8, -126, 127, 7, 3.3895313892515355e38};  // (2 - 2^-7) * 2^127
const Fmt kE4M3 = {4, -6, 7, 3, 448.0};

// Round the exact (double) value |v| to the format's grid, ties to even.
// Returns the rounded magnitude (may exceed maxf: the caller decides overflow).
double round_to_grid(double av, const Fmt& f) {
  if (av == 0.0) return 0.0;
  int e;
  std::frexp(av, &e);  // av = m * 2^e, m in [0.5, 1)  ->  floor(log2 av) = e - 1
  int ex = e - 1;
  if (ex < f.emin) ex = f.emin;  // subnormal range shares the min-normal quantum
  double quantum = std::ldexp(1.0, ex - (f.p - 1));
  double r = std::nearbyint(av / quantum);  // exact division by a power of two; RNE
  return r * quantum;
}

// Bits of a finite, representable magnitude `m` (already on the grid).
uint32_t grid_to_bits(double m, const Fmt& f) {
  if (m == 0.0) return 0;
  double min_normal = std::ldexp(1.0, f.emin);
  if (m < min_normal) {
    double sub_quantum = std::ldexp(1.0, f.emin - (f.p - 1));
    return (uint32_t)(m / sub_quantum);  // exponent field 0
  }
  int e;
  std::frexp(m, &e);
  int ex = e - 1;
  double frac = m / std::ldexp(1.0, ex) - 1.0;  // in [0, 1)
  uint32_t mant = (uint32_t)(frac * (double)(1u << f.mbits));
  return ((uint32_t)(ex + f.bias) << f.mbits) | mant;
}

double bits_to_value(uint32_t bits, const Fmt& f, bool has_inf) {
  int ebits = f.mbits == 10 ? 5 : (f.mbits == 7 ? 8 : 4);
  uint32_t sign = (bits >> (f.mbits + ebits)) & 1u;
  uint32_t ef = (bits >> f.mbits) & ((1u << ebits) - 1u);
  uint32_t mf = bits & ((1u << f.mbits) - 1u);
  double v;
  uint32_t emax_field = (1u << ebits) - 1u;
  if (has_inf && ef == emax_field) {
    v = mf ? std::numeric_limits<double>::quiet_NaN() : std::numeric_limits<double>::infinity();
  } else if (!has_inf && ef == emax_field && mf == (1u << f.mbits) - 1u) {
    v = std::numeric_limits<double>::quiet_NaN();  // E4M3 "fn": S.1111.111 is NaN
  } else if (ef == 0) {
    v = std::ldexp((double)mf, f.emin - f.mbits);
  } else {
    v = std::ldexp((double)(mf | (1u << f.mbits)), (int)ef - f.bias - f.mbits);
  }
  return sign ? -v : v;
}

// IEEE 754 binary16.
double f16_value(uint16_t h) { return bits_to_value(h, kF16, true); }
uint16_t f16_rne(double v) {
  uint16_t s = std::signbit(v) ? 0x8000 : 0;
  if (std::isnan(v)) return 0x7E00;
  double m = round_to_grid(std::fabs(v), kF16);
  if (std::isinf(v) || m > kF16.maxf) return s | 0x7C00;
  return s | (uint16_t)grid_to_bits(m, kF16);
}

// bfloat16: sign, 8 exponent bits (bias 127), 7 mantissa bits.
double bf16_value(uint16_t h) { return bits_to_value(h, kBF16, true); }
uint16_t bf16_rne(double v) {
  uint16_t s = std::signbit(v) ? 0x8000 : 0;
  if (std::isnan(v)) return s | 0x7FC0;
  double m = round_to_grid(std::fabs(v), kBF16);
  if (std::isinf(v) || m > kBF16.maxf) return s | 0x7F80;
  return s | (uint16_t)grid_to_bits(m, kBF16);
}

// OCP FP8 E4M3 ("fn"): bias 7, max 448, no infinities, S.1111.111 = NaN.
double e4m3_value(uint8_t c) { return bits_to_value(c, kE4M3, false); }
// Round to nearest even; magnitudes beyond 448 saturate to 448 (satfinite).
uint8_t e4m3_rne_satfinite(double v) {
  uint8_t s = std::signbit(v) ? 0x80 : 0;
  if (std::isnan(v)) return 0x7F | s;
  double m = std::isinf(v) ? kE4M3.maxf : round_to_grid(std::fabs(v), kE4M3);
  if (m > kE4M3.maxf) m = kE4M3.maxf;
  return s | (uint8_t)grid_to_bits(m, kE4M3);
}

float clampf(float v, float lo, float hi) { return std::fmin(std::fmax(v, lo), hi); }

// ---------------------------------------------------------------------------
// Packed layouts (this library's own; the pages fix only code widths, group
// sizes and scale types).
//
// Q4_G64 / Q5_G64 nibble plane, per row K/2 bytes read as K/8 little-endian
// 32-bit words.  Word j holds elements 8j..8j+7: element 8j+2s (s = 0..3) in
// bits [4s, 4s+4), element 8j+2s+1 in bits [16+4s, 16+4s+4).  The value stored
// is the offset code u = q + 8 (Q4) or the low 4 bits of u = q + 16 (Q5).
// Q5 high-bit plane, per row K/8 bytes read as K/32 little-endian words.  In
// word h, element 32h + 8jj + 2s + o (jj, s in 0..3; o in 0..1) keeps bit 4 of
// its u at bit 16*o + 4*jj + s.
// Q8_G32: int8 two's complement codes, row-major.  FP8_ROW: E4M3 bytes,
// row-major, one bfloat16 scale per row.  Scales of Q4/Q5 are binary16
// [N][K/64]; of Q8 binary16 [N][K/32].
// Two-bit ("crumb") plane, per row K/4 bytes read as K/16 little-endian
// words.  Word c holds elements 16c..16c+15: element 16c+2s+o (s = 0..7,
// o = 0..1) in bits [16o+2s, 16o+2s+2).
// Q3_G64: u = q + 4 in [0, 7]; the crumb plane holds bits 0..1 of u (codes,
// K/4 bytes per row) and a bit plane laid out as Q5's holds bit 2 (K/8 bytes
// per row).  Q6_G64: u = q + 32 in [0, 63]; a nibble plane laid out as Q4's
// holds bits 0..3 (codes, K/2 bytes per row) and a crumb plane holds bits
// 4..5 (K/4 bytes per row).  Scales binary16 [N][K/64].
// ---------------------------------------------------------------------------

enum { FMT_Q4_G64 = 0, FMT_Q5_G64 = 1, FMT_Q8_G32 = 2, FMT_FP8_ROW = 3, FMT_BF16 = 4,
       FMT_Q3_G64 = 5, FMT_Q6_G64 = 6 };

inline bool is_groupwise64(int fmt) {
  return fmt == FMT_Q4_G64 || fmt == FMT_Q5_G64 || fmt == FMT_Q3_G64 || fmt == FMT_Q6_G64;
}

inline uint32_t load_u32_le(const uint8_t* p) {
  return (uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16) | ((uint32_t)p[3] << 24);
}
inline void store_u32_le(uint8_t* p, uint32_t w) {
  p[0] = (uint8_t)w;
  p[1] = (uint8_t)(w >> 8);
  p[2] = (uint8_t)(w >> 16);
  p[3] = (uint8_t)(w >> 24);
}

inline int nibble_bit(int64_t e) {  // bit position of element e inside its word
  int i = (int)(e & 7);
  return 16 * (i & 1) + 4 * (i >> 1);
}
inline int hibit_bit(int64_t e) {  // bit position of element e's high bit
  int ee = (int)(e & 31);
  int jj = ee >> 3, i = ee & 7;
  return 16 * (i & 1) + 4 * jj + (i >> 1);
}

inline int crumb_bit(int64_t e) {  // bit position of element e inside its crumb word
  int i = (int)(e & 15);
  return 16 * (i & 1) + 2 * (i >> 1);
}

// Field readers of the planes (row r of a K-column matrix, element e).
int nibble_at(const uint8_t* plane, int64_t k, int64_t r, int64_t e) {
  uint32_t w = load_u32_le(plane + r * (k / 2) + (e / 8) * 4);
  return (int)((w >> nibble_bit(e)) & 0xF);
}
int crumb_at(const uint8_t* plane, int64_t k, int64_t r, int64_t e) {
  uint32_t w = load_u32_le(plane + r * (k / 4) + (e / 16) * 4);
  return (int)((w >> crumb_bit(e)) & 0x3);
}
int bit_at(const uint8_t* plane, int64_t k, int64_t r, int64_t e) {
  uint32_t h = load_u32_le(plane + r * (k / 8) + (e / 32) * 4);
  return (int)((h >> hibit_bit(e)) & 1u);
}

// Offset code u of element (row r, col e) of a Q3/Q4/Q5/Q6 matrix.
int read_u(int fmt, const uint8_t* codes, const uint8_t* hibits, int64_t k, int64_t r, int64_t e) {
  switch (fmt) {
    case FMT_Q4_G64: return nibble_at(codes, k, r, e);
    case FMT_Q5_G64: return nibble_at(codes, k, r, e) | (bit_at(hibits, k, r, e) << 4);
    case FMT_Q3_G64: return crumb_at(codes, k, r, e) | (bit_at(hibits, k, r, e) << 2);
    default: return nibble_at(codes, k, r, e) | (crumb_at(hibits, k, r, e) << 4);  // Q6
  }
}

// Offset of u: 2^(bits - 1).
int code_offset(int fmt) {
  return fmt == FMT_Q4_G64 ? 8 : fmt == FMT_Q5_G64 ? 16 : fmt == FMT_Q3_G64 ? 4 : 32;
}

// Integer weight code q of any integer format.
int weight_code(int fmt, const void* codes, const void* hibits, int64_t k, int64_t r, int64_t e) {
  if (is_groupwise64(fmt))
    return read_u(fmt, (const uint8_t*)codes, (const uint8_t*)hibits, k, r, e) - code_offset(fmt);
  return (int)((const int8_t*)codes)[r * k + e];  // Q8_G32
}

int group_size(int fmt) { return fmt == FMT_Q8_G32 ? 32 : 64; }

// Dequantized weight w[r][e] as an exact double.
double weight_value(int fmt, const void* codes, const void* hibits, const void* scales, int64_t k,
                    int64_t r, int64_t e) {
  if (fmt == FMT_BF16) return bf16_value(((const uint16_t*)codes)[r * k + e]);
  if (fmt == FMT_FP8_ROW) {
    double c = e4m3_value(((const uint8_t*)codes)[r * k + e]);
    return c * bf16_value(((const uint16_t*)scales)[r]);
  }
  int gs = group_size(fmt);
  double s = f16_value(((const uint16_t*)scales)[r * (k / gs) + e / gs]);
  return (double)weight_code(fmt, codes, hibits, k, r, e) * s;
}

template <class F>
void parallel_rows(int64_t n, int nthreads, F&& body) {
  if (nthreads <= 1 || n < 2) {
    body((int64_t)0, n);
    return;
  }
  std::vector<std::thread> th;
  int64_t per = (n + nthreads - 1) / nthreads;
  for (int i = 0; i < nthreads; ++i) {
    int64_t a = i * per, b = std::min(n, a + per);
    if (a >= b) break;
    th.emplace_back([&body, a, b] { body(a, b); });
  }
  for (auto& t : th) t.join();
}

}  // namespace

extern "C" {

// ---- format codecs, exported so the tests can pin them -------------------
double oracle_f16_value(uint16_t h) { return f16_value(h); }
uint16_t oracle_f16_rne(double v) { return f16_rne(v); }
double oracle_bf16_value(uint16_t h) { return bf16_value(h); }
uint16_t oracle_bf16_rne(double v) { return bf16_rne(v); }
double oracle_e4m3_value(uint8_t c) { return e4m3_value(c); }
uint8_t oracle_e4m3_rne_satfinite(double v) { return e4m3_rne_satfinite(v); }

// BF16 re-encode of float32 values (the QLIN_BF16 target format).
int oracle_to_bf16(const float* v, int64_t count, uint16_t* out) {
  for (int64_t i = 0; i < count; ++i) out[i] = bf16_rne((double)v[i]);
  return 0;
}

// ---- groupwise integer packing --------------------------------------------
// [NVFP4] "What is in the file": Q4/Q5/Q8 grouped, FP16 scales.
// [RTX5080] "Quantization profile": Q3G64_F16S, Q4G64_F16S, Q5G64_F16S
// (group 64); [MXFP8] "Caveats": Q4/Q5/Q6 groupwise.
// Per row r and group g: a = max |w| over the group (FP32); the stored scale
// is s16 = binary16_rne(a / Qmax) with the FP32 quotient; s = value(s16);
// q = (s == 0) ? 0 : clamp(rint(w / s), -(Qmax+1), Qmax), w / s in FP32.
// Qmax = 2^(bits-1) - 1: 3 (Q3), 7 (Q4), 15 (Q5), 31 (Q6), 127 (Q8, group 32)
// -- the signed range of the code width, as the pages' Q4/Q5 scale amax/7,
// amax/15 read.
// Pinned by: codes in range, |q*s - w| <= s/2, pack(dequant(pack)) == pack,
// hand-derived groups (ties included), and the exhaustive codec tests.
int oracle_pack_groupwise(int fmt, const float* w, int64_t n, int64_t k, void* codes, void* hibits,
                          uint16_t* scales) {
  if (!is_groupwise64(fmt) && fmt != FMT_Q8_G32) return 1;
  int gs = group_size(fmt);
  if (k % gs != 0 || (fmt != FMT_Q8_G32 && k % 64 != 0)) return 1;
  int qmax = fmt == FMT_Q8_G32 ? 127 : code_offset(fmt) - 1;
  int64_t ng = k / gs;
  if (fmt == FMT_Q4_G64 || fmt == FMT_Q5_G64 || fmt == FMT_Q6_G64) std::memset(codes, 0, (size_t)(n * (k / 2)));
  if (fmt == FMT_Q3_G64) std::memset(codes, 0, (size_t)(n * (k / 4)));
  if (fmt == FMT_Q5_G64 || fmt == FMT_Q3_G64) std::memset(hibits, 0, (size_t)(n * (k / 8)));
  if (fmt == FMT_Q6_G64) std::memset(hibits, 0, (size_t)(n * (k / 4)));
  for (int64_t r = 0; r < n; ++r) {
    for (int64_t g = 0; g < ng; ++g) {
      const float* wg = w + r * k + g * gs;
      float a = 0.0f;
      for (int i = 0; i < gs; ++i) {
        float m = std::fabs(wg[i]);
        if (m > a) a = m;
      }
      float quot = a / (float)qmax;
      uint16_t s16 = f16_rne((double)quot);
      scales[r * ng + g] = s16;
      float s = (float)f16_value(s16);
      for (int i = 0; i < gs; ++i) {
        int q = 0;
        if (s != 0.0f) {
          float v = std::nearbyint(wg[i] / s);
          q = (int)clampf(v, (float)(-(qmax + 1)), (float)qmax);
        }
        int64_t e = g * gs + i;
        if (fmt == FMT_Q8_G32) {
          ((int8_t*)codes)[r * k + e] = (int8_t)q;
        } else {
          const uint32_t u = (uint32_t)(q + code_offset(fmt));
          // OR a field into a plane word (planes start zeroed)
          auto put = [](uint8_t* wp, uint32_t field, int bit) {
            store_u32_le(wp, load_u32_le(wp) | (field << bit));
          };
          uint8_t* cp = (uint8_t*)codes;
          uint8_t* hp = (uint8_t*)hibits;
          if (fmt == FMT_Q3_G64) {
            put(cp + r * (k / 4) + (e / 16) * 4, u & 0x3, crumb_bit(e));
            put(hp + r * (k / 8) + (e / 32) * 4, (u >> 2) & 1, hibit_bit(e));
          } else {
            put(cp + r * (k / 2) + (e / 8) * 4, u & 0xF, nibble_bit(e));
            if (fmt == FMT_Q5_G64) put(hp + r * (k / 8) + (e / 32) * 4, (u >> 4) & 1, hibit_bit(e));
            if (fmt == FMT_Q6_G64) put(hp + r * (k / 4) + (e / 16) * 4, (u >> 4) & 0x3, crumb_bit(e));
          }
        }
      }
    }
  }
  return 0;
}

// ---- row-scaled FP8 packing (fp8_row_maxabs) ------------------------------
// [ROWFP8] "Conversion and verification": one BF16 scale per output row.
// a = max_k |w[r,k]| (FP32); sc16 = bf16_rne(a / 448) (FP32 quotient);
// code = (sc == 0) ? 0x00 : e4m3_rne_satfinite(w / sc) (FP32 quotient).
// Pinned by: the element-wise half-ulp bound the page states, re-encode
// idempotence ("re-encodes bit-exact"), and the exhaustive E4M3 codec tests.
int oracle_pack_fp8_row(const float* w, int64_t n, int64_t k, uint8_t* codes, uint16_t* scales) {
  for (int64_t r = 0; r < n; ++r) {
    const float* wr = w + r * k;
    float a = 0.0f;
    for (int64_t i = 0; i < k; ++i) {
      float m = std::fabs(wr[i]);
      if (m > a) a = m;
    }
    float quot = a / 448.0f;
    uint16_t sc16 = bf16_rne((double)quot);
    scales[r] = sc16;
    float sc = (float)bf16_value(sc16);
    for (int64_t i = 0; i < k; ++i) {
      codes[r * k + i] = sc == 0.0f ? (uint8_t)0 : e4m3_rne_satfinite((double)(wr[i] / sc));
    }
  }
  return 0;
}

// ---- MXFP8 decode ----------------------------------------------------------
// [MXFP8] step 1: four E4M3 values per U32 word, one U8 UE8M0 scale 2^(b-127)
// per 32-element group, decoded to BF16.  Element 4i+j of a row is byte j
// (bits 8j..8j+7) of word i.  value = e4m3(byte) * 2^(b-127) computed exactly
// and rounded once to BF16 (RNE).  b = 255 or an E4M3 NaN gives the BF16 NaN
// 0x7FC0 carrying the element's sign bit.
// Pinned by: exhaustive 256 codes x 256 exponents against the closed form.
int oracle_decode_mxfp8(const uint32_t* words, const uint8_t* scales, int64_t rows, int64_t cols,
                        uint16_t* out) {
  if (cols % 32 != 0) return 1;
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t c = 0; c < cols; ++c) {
      uint32_t wv = words[r * (cols / 4) + c / 4];
      uint8_t byte = (uint8_t)(wv >> (8 * (c % 4)));
      uint8_t b = scales[r * (cols / 32) + c / 32];
      uint16_t sign = (byte & 0x80) ? 0x8000 : 0;
      double v = e4m3_value(byte);
      if (b == 255 || std::isnan(v)) {
        out[r * cols + c] = sign | 0x7FC0;
        continue;
      }
      out[r * cols + c] = bf16_rne(std::ldexp(v, (int)b - 127));
    }
  }
  return 0;
}

// ---- FP8 block-128 source decode -------------------------------------------
// [ROWFP8] "Conversion and verification": the checkpoint stores a projection
// as E4M3 codes with a weight_scale_inv value per 128x128 weight block; each
// code is decoded in FP32 (E4M3 value times the block's scale) and the decoded
// values are re-encoded (per row, fp8_row_maxabs, or into any other target).
// Reading: the block grid is float32 [ceil(rows/128)][ceil(cols/128)]
// row-major; value = float32(e4m3(code) * scale) with one IEEE rounding (exact
// whenever the scale has at most 20 significant bits, e.g. a BF16 scale: the
// page's "fits exactly"); the value is then taken to BF16 (RNE) like every
// non-F32 source of this library, which is the page's "source value's own
// BF16 rounding" in its error bound.  E4M3 NaN codes decode to the BF16 NaN
// with their sign.
// Pinned by: the exact product for BF16-representable scales (numpy float64),
// a hand example, and the page's element bound after the row re-encode.
int oracle_decode_fp8_block128(const uint8_t* codes, const float* scale_inv, int64_t rows,
                               int64_t cols, uint16_t* out) {
  int64_t gcols = (cols + 127) / 128;
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t c = 0; c < cols; ++c) {
      uint8_t code = codes[r * cols + c];
      double e = e4m3_value(code);
      if (std::isnan(e)) {
        out[r * cols + c] = (uint16_t)(((code & 0x80) ? 0x8000 : 0) | 0x7FC0);
        continue;
      }
      float v = (float)e * scale_inv[(r / 128) * gcols + c / 128];  // one FP32 rounding
      out[r * cols + c] = bf16_rne((double)v);
    }
  }
  return 0;
}

// ---- MLX affine int8 decode -------------------------------------------------
// [MXFP8] step 2: uint8 codes, per-128-group F16 scale and F16 bias,
// w = q * scale + bias, decoded to BF16.  Reading: one FP32 fused
// multiply-add (single rounding), then BF16 RNE.
// Pinned by: hand values and the exact-in-double identity of the fma.
int oracle_decode_mlx_affine(const uint8_t* q, const uint16_t* scales, const uint16_t* biases,
                             int64_t rows, int64_t cols, uint16_t* out) {
  if (cols % 128 != 0) return 1;
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t c = 0; c < cols; ++c) {
      int64_t gi = r * (cols / 128) + c / 128;
      float s = (float)f16_value(scales[gi]);
      float bsum = (float)f16_value(biases[gi]);
      float v = std::fmaf((float)q[r * cols + c], s, bsum);
      out[r * cols + c] = bf16_rne((double)v);
    }
  }
  return 0;
}

// ---- dequantized weights ----------------------------------------------------
int oracle_dequant(int fmt, const void* codes, const void* hibits, const void* scales, int64_t n,
                   int64_t k, double* wdq) {
  for (int64_t r = 0; r < n; ++r)
    for (int64_t e = 0; e < k; ++e) wdq[r * k + e] = weight_value(fmt, codes, hibits, scales, k, r, e);
  return 0;
}

// ---- BF16-route projection (decode GEMV / skinny GEMM, and BF16 weights) ----
// [A8] "What changes": decode (MTP, DFlash2, n-gram verification) keeps the
// BF16 route.  [NVFP4] "How it was created": the head op over T = 1..33.
// y[t][r] = sum_e wdq[r][e] * x[t][e], accumulated in double; bound[t][r] =
// sum_e |wdq[r][e]| * |x[t][e]| (the per-element tolerance scale).
// Pinned by: integer inputs with unit scales equal an exact integer product.
int oracle_gemv(int fmt, const void* codes, const void* hibits, const void* scales, int64_t n,
                int64_t k, const uint16_t* x, int64_t t, double* y, double* bound, int nthreads) {
  std::vector<double> xv((size_t)(t * k));
  for (int64_t i = 0; i < t * k; ++i) xv[i] = bf16_value(x[i]);
  parallel_rows(n, nthreads, [&](int64_t r0, int64_t r1) {
    std::vector<double> wr((size_t)k);
    for (int64_t r = r0; r < r1; ++r) {
      for (int64_t e = 0; e < k; ++e) wr[e] = weight_value(fmt, codes, hibits, scales, k, r, e);
      for (int64_t tt = 0; tt < t; ++tt) {
        double acc = 0.0, ab = 0.0;
        const double* xr = xv.data() + tt * k;
        for (int64_t e = 0; e < k; ++e) {
          acc += wr[e] * xr[e];
          ab += std::fabs(wr[e]) * std::fabs(xr[e]);
        }
        y[tt * n + r] = acc;
        if (bound) bound[tt * n + r] = ab;
      }
    }
  });
  return 0;
}

// ---- activation quantization (int8 prefill route) -------------------------
// [A8] "What changes": activations are quantized per token and per 64
// channels, scale = amax / 127, in the same groups as the weight scales.
// Per (t, g): a = max |x| over the 64 BF16 values (exact in FP32);
// as = a / 127 (FP32, kept FP32); qa = (as == 0) ? 0 :
// clamp(rint(x / as), -127, 127) with the FP32 quotient.
// Pinned by: |qa*as - x| <= as/2, the amax element maps to +-127, zero groups.
int oracle_quantize_act(const uint16_t* x, int64_t t, int64_t k, int8_t* qa, float* as) {
  if (k % 64 != 0) return 1;
  for (int64_t tt = 0; tt < t; ++tt) {
    for (int64_t g = 0; g < k / 64; ++g) {
      const uint16_t* xg = x + tt * k + g * 64;
      float a = 0.0f;
      for (int i = 0; i < 64; ++i) {
        float m = std::fabs((float)bf16_value(xg[i]));
        if (m > a) a = m;
      }
      float s = a / 127.0f;
      as[tt * (k / 64) + g] = s;
      for (int i = 0; i < 64; ++i) {
        int q = 0;
        if (s != 0.0f) {
          float v = std::nearbyint((float)bf16_value(xg[i]) / s);
          q = (int)clampf(v, -127.0f, 127.0f);
        }
        qa[tt * k + g * 64 + i] = (int8_t)q;
      }
    }
  }
  return 0;
}

// ---- int8 route: per-group integer sums ------------------------------------
// [A8] "What changes": the weight codes feed integer MMAs exactly; one int32
// sum per 64-group.  S[t][r][g] = sum over the group of qa[t][e] * q[r][e],
// computed in int64 and checked to fit int32.
// Pinned by: numpy integer matmul per group on tiny shapes; |S| at all-max codes.
int oracle_group_sums(int fmt, const void* codes, const void* hibits, const int8_t* qa, int64_t t,
                      int64_t n, int64_t k, int32_t* S) {
  if (!is_groupwise64(fmt)) return 1;
  int64_t ng = k / 64;
  for (int64_t tt = 0; tt < t; ++tt)
    for (int64_t r = 0; r < n; ++r)
      for (int64_t g = 0; g < ng; ++g) {
        int64_t s = 0;
        for (int i = 0; i < 64; ++i) {
          int64_t e = g * 64 + i;
          s += (int64_t)qa[tt * k + e] * (int64_t)weight_code(fmt, codes, hibits, k, r, e);
        }
        if (s > INT32_MAX || s < INT32_MIN) return 2;
        S[(tt * n + r) * ng + g] = (int32_t)s;
      }
  return 0;
}

// ---- int8 route: FP32 rescale of each group sum ----------------------------
// [A8] "What changes": each group's int32 sum is scaled by
// weight_scale x activation_scale in FP32.  Reading: c = float(ws) * as is
// the FP32 product; y[t][r] = sum_g c * S accumulated in double.
// bound[t][r] = sum_e |q*ws| * |qa*as| (the per-element tolerance scale).
// Pinned by: unit scales reduce it to an exact integer product.
int oracle_gemm_a8(int fmt, const void* codes, const void* hibits, const uint16_t* wscales,
                   const int8_t* qa, const float* as, int64_t t, int64_t n, int64_t k, double* y,
                   double* bound, int nthreads) {
  if (!is_groupwise64(fmt)) return 1;
  int64_t ng = k / 64;
  parallel_rows(n, nthreads, [&](int64_t r0, int64_t r1) {
    std::vector<int> qr((size_t)k);
    for (int64_t r = r0; r < r1; ++r) {
      for (int64_t e = 0; e < k; ++e) qr[e] = weight_code(fmt, codes, hibits, k, r, e);
      for (int64_t tt = 0; tt < t; ++tt) {
        double acc = 0.0, ab = 0.0;
        for (int64_t g = 0; g < ng; ++g) {
          int64_t s = 0, sa = 0;
          for (int i = 0; i < 64; ++i) {
            int64_t e = g * 64 + i;
            int64_t a = qa[tt * k + e], w = qr[e];
            s += a * w;
            sa += (a < 0 ? -a : a) * (w < 0 ? -w : w);
          }
          float ws = (float)f16_value(wscales[r * ng + g]);
          float c = ws * as[tt * ng + g];
          acc += (double)c * (double)s;
          ab += std::fabs((double)ws * (double)as[tt * ng + g]) * (double)sa;
        }
        y[tt * n + r] = acc;
        if (bound) bound[tt * n + r] = ab;
      }
    }
  });
  return 0;
}

// ---- FP8-activation route: per-token E4M3 activations --------------------
// [ROWFP8] "Conversion and verification", "Hardware fit": the row-scaled FP8
// weights run on FP8-activation tensor-core routes.  The page fixes no
// activation scheme; reading, mirroring fp8_row_maxabs on the activation side:
// per token t, a = max_k |x[t][k]| (exact in FP32), xs = a / 448 (FP32, kept
// FP32), xq = (xs == 0) ? 0x00 : E4M3_rne_satfinite(x / xs) (FP32 quotient).
// Pinned by: hand examples (incl. a tie), the amax element at +-448, zero
// tokens, and the E4M3 half-ulp bound of every element.
int oracle_quantize_act_fp8(const uint16_t* x, int64_t t, int64_t k, uint8_t* xq, float* xs) {
  for (int64_t tt = 0; tt < t; ++tt) {
    const uint16_t* xr = x + tt * k;
    float a = 0.0f;
    for (int64_t i = 0; i < k; ++i) {
      float m = std::fabs((float)bf16_value(xr[i]));
      if (m > a) a = m;
    }
    float s = a / 448.0f;
    xs[tt] = s;
    for (int64_t i = 0; i < k; ++i)
      xq[tt * k + i] = s == 0.0f ? (uint8_t)0 : e4m3_rne_satfinite((double)((float)bf16_value(xr[i]) / s));
  }
  return 0;
}

// ---- FP8-activation route: row-FP8 weights x per-token FP8 activations ------
// y[t][n] = c * S with S = sum_k e4m3(wq[n][k]) * e4m3(xq[t][k]) (exact, in
// double) and c = FP32(ws[n] * xs[t]), ws the BF16 row scale; reported in
// double.  bound[t][n] = sum_k |e4m3(wq) ws| * |e4m3(xq) xs| (tolerance scale).
// Pinned by: integer-valued E4M3 codes with unit scales equal an exact integer
// matrix product.
int oracle_gemm_fp8(const uint8_t* wq, const uint16_t* ws, const uint8_t* xq, const float* xs,
                    int64_t t, int64_t n, int64_t k, double* y, double* bound, int nthreads) {
  std::vector<double> xv((size_t)(t * k));
  for (int64_t i = 0; i < t * k; ++i) xv[i] = e4m3_value(xq[i]);
  parallel_rows(n, nthreads, [&](int64_t r0, int64_t r1) {
    std::vector<double> wr((size_t)k);
    for (int64_t r = r0; r < r1; ++r) {
      for (int64_t e = 0; e < k; ++e) wr[e] = e4m3_value(wq[r * k + e]);
      float wsr = (float)bf16_value(ws[r]);
      for (int64_t tt = 0; tt < t; ++tt) {
        double S = 0.0, A = 0.0;
        const double* xr = xv.data() + tt * k;
        for (int64_t e = 0; e < k; ++e) {
          S += wr[e] * xr[e];
          A += std::fabs(wr[e]) * std::fabs(xr[e]);
        }
        float c = wsr * xs[tt];
        y[tt * n + r] = (double)c * S;
        if (bound) bound[tt * n + r] = std::fabs((double)wsr * (double)xs[tt]) * A;
      }
    }
  });
  return 0;
}

}  // extern "C"
