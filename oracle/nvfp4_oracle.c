/*
 * nvfp4_oracle.c -- plain, slow CPU oracle for NVFP4 / MXFP8 block-scaled
 * quantization (TEST INFRASTRUCTURE ONLY).
 *
 * Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may
 * load this library.  It shares no code, header, table or constant with the
 * CUDA path; the two meet only through the seeded input generators.
 *
 * Arithmetic rules: every step that the method performs in fp32 is done here
 * with C `float` under strict IEEE semantics (built with -ffp-contract=off,
 * no fast-math; x86-64 SSE evaluates float expressions in single precision),
 * so each rounding happens exactly where the method rounds.  Contractions are
 * not done here: the Python side (oracle.py) feeds exact float64 operands to
 * a float64 matmul.
 *
 * Sources (page title, then file / section):
 *  [P1] "mlx 0.30.7.2 -> 0.30.7.6" diff, page 8: ops.cpp fp_quantize /
 *       fp_dequantize fallbacks, QQMatmul::vjp.
 *  [P2] "mlx 0.30.7.2 -> 0.30.7.6" diff, page 7: fp_quantize.cu kernels
 *       fp_quantize_dequantize, fp_quantize_rowwise, fp_dequantize;
 *       qqmm_utils.cu compute_qqmm_pointers.
 *  [P3] "[Metal] global scale for qmm" (ml-explore/mlx pull 4458): the worked
 *       example; the pasted mlxcel pull 1772 note on MXFP8 E8M0 round-up.
 *  [P4] osaurus-ai/mlx pull 31 (CPU qqmm global scales): "What fails",
 *       "The test", "The fix".
 *  [P5] "mlx 0.30.7" diff, page 71: qqmm_utils.cu swizzle_scales and its
 *       128x4 tile layout comment.
 *
 * Parity status: every exported function is pinned by tests under
 * tests/test_oracle_*.py (format brute force, worked example, cases A-D,
 * MXFP8 round-up case, swizzle index table, closed-form invariants).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* Input / output element types (oracle-local tags). */
enum { ORC_F32 = 0, ORC_F16 = 1, ORC_BF16 = 2 };

/* ------------------------------------------------------------------------ */
/* 1. Format definitions (decoders)                                          */
/* ------------------------------------------------------------------------ */

/* e2m1: 1 sign bit (bit 3), 2 exponent bits (bias 1), 1 mantissa bit.
 * Exponent field 0 is subnormal: value = m * 0.5. */
double orc_e2m1_value(int code) {
  int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
  double mag = (e == 0) ? m * 0.5 : (1.0 + m / 2.0) * ldexp(1.0, e - 1);
  return s ? -mag : mag;
}

/* e4m3 ("fn" variant): 1 sign, 4 exponent bits (bias 7), 3 mantissa bits;
 * no infinities; exponent 15 with mantissa 7 is NaN; exponent 0 subnormal. */
double orc_e4m3_value(int byte) {
  int s = (byte >> 7) & 1, e = (byte >> 3) & 15, m = byte & 7;
  double mag;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) mag = (m / 8.0) * ldexp(1.0, -6);
  else mag = (1.0 + m / 8.0) * ldexp(1.0, e - 7);
  return s ? -mag : mag;
}

/* e8m0: unsigned power of two 2^(b-127); 0xFF is NaN. */
double orc_e8m0_value(int byte) {
  if (byte == 255) return NAN;
  return ldexp(1.0, byte - 127);
}

/* ------------------------------------------------------------------------ */
/* 2. Encoders by exhaustive nearest search                                  */
/* ------------------------------------------------------------------------ */

/* Nearest non-negative code of a magnitude among `ncodes` candidates whose
 * values come from `dec`; ties go to the even code (mantissa LSB 0);
 * magnitudes above the largest finite value saturate to it ("satfinite"). */
static int nearest_code(double mag, int ncodes, double (*dec)(int)) {
  int best = 0;
  double bestd = INFINITY;
  /* saturation first: at or beyond the largest finite value (infinity
   * included) the answer is that value's code */
  int top = 0;
  for (int c = 0; c < ncodes; ++c)
    if (!isnan(dec(c)) && dec(c) > dec(top)) top = c;
  if (mag >= dec(top)) return top;
  /* below it, distances to the two neighbouring candidates are exact in
   * double (Sterbenz), so the search is exact */
  for (int c = 0; c < ncodes; ++c) {
    double v = dec(c);
    if (isnan(v)) continue;
    double d = fabs(mag - v);
    if (d < bestd || (d == bestd && (c & 1) == 0 && (best & 1) == 1)) {
      best = c;
      bestd = d;
    }
  }
  return best;
}

/* e2m1, round to nearest even, saturate to +-6; the sign of the input is
 * kept, so a negative value that rounds to zero gives -0 (code 0x8). */
int orc_e2m1_rne_satfinite(float v) {
  double mag = fabs((double)v);
  int c = nearest_code(mag, 8, orc_e2m1_value);
  return signbit(v) ? (c | 8) : c;
}

/* e4m3, round to nearest even, saturate to +-448. */
int orc_e4m3_rne_satfinite(float v) {
  double mag = fabs((double)v);
  int c = nearest_code(mag, 127, orc_e4m3_value);
  return signbit(v) ? (c | 0x80) : c;
}

/* e8m0, rounded up: smallest power of two 2^k >= v, byte k+127, clamped to
 * [0, 254].  "CUDA rounds up" ([P3], mlxcel note): the block scale is never
 * below amax/448, so no element saturates.  v == 0 gives byte 0 (2^-127). */
int orc_e8m0_ceil(float v) {
  if (!(v > 0.0f)) return 0;
  if (isinf(v)) return 254;
  int e;
  double f = frexp((double)v, &e); /* v = f * 2^e, f in [0.5, 1) */
  int k = (f == 0.5) ? e - 1 : e;  /* ceil(log2 v), exact */
  int b = k + 127;
  if (b < 0) b = 0;
  if (b > 254) b = 254;
  return b;
}

/* ------------------------------------------------------------------------ */
/* 3. Element types: read as float, round a real to the type                */
/* ------------------------------------------------------------------------ */

/* Round a real number to a binary floating-point format with p significand
 * bits, minimum normal exponent emin and largest finite value maxv, round to
 * nearest with ties to even, overflow to infinity (IEEE conversion rules).
 * The quantum is 2^(exponent - p + 1), floored at the subnormal quantum. */
double orc_round_to_format(double v, int p, int emin, double maxv) {
  if (v == 0.0 || !isfinite(v)) return v;
  int e;
  frexp(fabs(v), &e);
  int lead = e - 1;
  if (lead < emin) lead = emin;
  double q = ldexp(1.0, lead - (p - 1));
  double r = rint(v / q) * q; /* v / q is exact: q is a power of two */
  if (fabs(r) > maxv) return v > 0 ? INFINITY : -INFINITY;
  return r;
}

static const double BF16_MAX = 3.38953138925153547590470800371487866880e+38;
static const double F16_MAX = 65504.0;

double orc_round_to_type(double v, int dt) {
  switch (dt) {
    case ORC_F32: return (double)(float)v; /* IEEE double->float conversion */
    case ORC_F16: return orc_round_to_format(v, 11, -14, F16_MAX);
    default: return orc_round_to_format(v, 8, -126, BF16_MAX);
  }
}

/* bf16 bit pattern of a real already representable in bf16. */
static uint16_t bf16_bits(double v) {
  float f = (float)v;
  uint32_t u;
  memcpy(&u, &f, 4);
  return (uint16_t)(u >> 16);
}

/* fp16 bit pattern of a real already representable in fp16. */
static uint16_t f16_bits(double v) {
  uint16_t s = signbit(v) ? 0x8000 : 0;
  double a = fabs(v);
  if (isinf(a)) return s | 0x7C00;
  if (a == 0.0) return s;
  int e;
  double f = frexp(a, &e); /* a = f 2^e, f in [0.5,1); leading exponent e-1 */
  int lead = e - 1;
  if (lead < -14) { /* subnormal: a = m * 2^-24 */
    return s | (uint16_t)(a * ldexp(1.0, 24));
  }
  uint16_t m = (uint16_t)((f * 2.0 - 1.0) * 1024.0);
  return s | (uint16_t)((lead + 15) << 10) | m;
}

/* Value of element i of a raw array of type dt (exact in double). */
double orc_load(const void* x, int dt, int64_t i) {
  if (dt == ORC_F32) return ((const float*)x)[i];
  uint16_t h = ((const uint16_t*)x)[i];
  if (dt == ORC_BF16) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
  }
  /* fp16: 1 sign, 5 exponent bits (bias 15), 10 mantissa bits */
  int s = h >> 15, e = (h >> 10) & 31, m = h & 1023;
  double mag;
  if (e == 31) mag = m ? NAN : INFINITY;
  else if (e == 0) mag = m * ldexp(1.0, -24);
  else mag = (1.0 + m / 1024.0) * ldexp(1.0, e - 15);
  return s ? -mag : mag;
}

/* Store v (rounded to type dt) as element i of a raw array of type dt. */
void orc_store(void* out, int dt, int64_t i, double v) {
  double r = orc_round_to_type(v, dt);
  if (dt == ORC_F32) ((float*)out)[i] = (float)r;
  else if (dt == ORC_BF16) ((uint16_t*)out)[i] = bf16_bits(r);
  else ((uint16_t*)out)[i] = f16_bits(r);
}

/* ------------------------------------------------------------------------ */
/* 4. Tensor amax: g = max |x| as fp32 ([P1] QQMatmul::vjp takes             */
/*    astype(max(abs(cotan)), float32); [P2] names alpha's inputs            */
/*    tensor_amax_x / tensor_amax_w).                                        */
/* ------------------------------------------------------------------------ */
float orc_amax(const void* x, int dt, int64_t n) {
  double m = 0.0;
  for (int64_t i = 0; i < n; ++i) {
    double a = fabs(orc_load(x, dt, i));
    if (a > m) m = a;
  }
  return (float)m; /* exact: m is an element of x */
}

/* ------------------------------------------------------------------------ */
/* 5. NVFP4 two-level quantize ([P2] fp_quantize_rowwise with global scale,  */
/*    comment "Global encode scale ... Per-block decode scale ...").         */
/*    Per row, per 16-element block along K:                                 */
/*      E   = 2688 / g            (1 without a global scale)                 */
/*      a   = max |x_i|                                                      */
/*      t   = (a / 6) * E         fp32, in that order                        */
/*      s   = e4m3_rne_satfinite(t)            -> scale byte                 */
/*      k   = E / f8(s)           fp32 division                              */
/*      q_i = e2m1_rne_satfinite(x_i * k)      -> 4-bit code                 */
/*    A block whose scale byte decodes to 0 stores all-zero codes (k would   */
/*    be infinite; [P4] "The fix": x_hat is 0 when s is 0).                  */
/*    Codes: element 8w+i of a row in bits 4i..4i+3 of word w.               */
/*    Scales: LINEAR layout [rows, K/16].                                    */
/* ------------------------------------------------------------------------ */
static float encode_factor(const float* g) {
  return g ? (448.0f * 6.0f) / *g : 1.0f;
}

/* Scale byte of one block from its amax a: t = a / 6 first, then t * E,
 * each rounded to fp32 ([P2] fp_quantize_rowwise computes the block maximum
 * over 6 and multiplies by the encode factor). */
static int nvfp4_scale_byte(float a, float E) {
  float t = a / 6.0f;
  t = t * E;
  return orc_e4m3_rne_satfinite(t);
}

/* Value handed to the e2m1 encoder: the factor k = E / f8(s) first, then
 * x * k, each rounded to fp32 ([P2] fp_quantize_rowwise divides the encode
 * factor by the block scale once and multiplies every element by it). */
static float nvfp4_scaled_value(float x, float E, float fs) {
  float k = E / fs;
  return x * k;
}

void orc_nvfp4_quantize(const void* x, int dt, int64_t rows, int64_t K,
                        const float* g, uint32_t* codes, uint8_t* scales) {
  const float E = encode_factor(g);
  const int64_t nb = K / 16;
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t b = 0; b < nb; ++b) {
      float xv[16];
      float a = 0.0f;
      for (int i = 0; i < 16; ++i) {
        xv[i] = (float)orc_load(x, dt, r * K + b * 16 + i);
        if (fabsf(xv[i]) > a) a = fabsf(xv[i]);
      }
      int s = nvfp4_scale_byte(a, E);
      scales[r * nb + b] = (uint8_t)s;
      float fs = (float)orc_e4m3_value(s);
      uint32_t w[2] = {0, 0};
      if (fs != 0.0f) {
        for (int i = 0; i < 16; ++i) {
          uint32_t q = (uint32_t)orc_e2m1_rne_satfinite(nvfp4_scaled_value(xv[i], E, fs));
          w[i / 8] |= q << (4 * (i % 8));
        }
      }
      codes[(r * K + b * 16) / 8] = w[0];
      codes[(r * K + b * 16) / 8 + 1] = w[1];
    }
  }
}

/* Decode factor d(g) = g / 2688 in fp32 ([P2] fp_dequantize:
 * inv_scale_enc = global_scale / (448 * 6)); 1 without a global scale. */
static float decode_factor(const float* g) {
  return g ? *g / (448.0f * 6.0f) : 1.0f;
}

/* Per-block decoded scale f8(s) * d(g), rounded to fp32 as the dequantize
 * kernel does ([P2] fp_dequantize: float(scale) * inv_scale_enc). */
float orc_nvfp4_block_scale(uint8_t s, const float* g) {
  return (float)orc_e4m3_value(s) * decode_factor(g);
}

/* ------------------------------------------------------------------------ */
/* 6. NVFP4 dequantize ([P2] fp_dequantize; [P1] fp_dequantize fallback):    */
/*    w_hat = T( e2m1(q) * (f8(s) * d(g)) ), products in fp32, then rounded  */
/*    to the output type T.                                                  */
/* ------------------------------------------------------------------------ */
void orc_nvfp4_dequantize(const uint32_t* codes, const uint8_t* scales,
                          int64_t rows, int64_t K, const float* g, void* out,
                          int out_dt) {
  const int64_t nb = K / 16;
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t k = 0; k < K; ++k) {
      int64_t idx = r * K + k;
      int q = (codes[idx / 8] >> (4 * (idx % 8))) & 15;
      float sd = orc_nvfp4_block_scale(scales[r * nb + k / 16], g);
      float v = (float)orc_e2m1_value(q) * sd;
      orc_store(out, out_dt, idx, v);
    }
  }
}

/* Exact real value of each quantized element, e2m1(q) * f8(s) * d(g), in
 * float64 (at most 2 + 4 + 24 significant bits, so exact).  Operand of the
 * dense block-scaled GEMM oracle, where no operand is rounded to T. */
void orc_nvfp4_decode_exact(const uint32_t* codes, const uint8_t* scales,
                            int64_t rows, int64_t K, const float* g,
                            double* out) {
  const int64_t nb = K / 16;
  const double d = (double)decode_factor(g);
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t k = 0; k < K; ++k) {
      int64_t idx = r * K + k;
      int q = (codes[idx / 8] >> (4 * (idx % 8))) & 15;
      out[idx] = orc_e2m1_value(q) * orc_e4m3_value(scales[r * nb + k / 16]) * d;
    }
  }
}

/* Weight values of the qmv route: e2m1(q) times the per-block decoded scale
 * as the dequantize kernel forms it in fp32 (f8(s) * d(g), one rounding),
 * the product exact in float64.  The weight is not rounded to an output
 * type on that route ([P4] "The fix": the global scale goes on each block
 * scale; the sum is not rescaled). */
void orc_nvfp4_decode_blockscale(const uint32_t* codes, const uint8_t* scales,
                                 int64_t rows, int64_t K, const float* g,
                                 double* out) {
  const int64_t nb = K / 16;
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t k = 0; k < K; ++k) {
      int64_t idx = r * K + k;
      int q = (codes[idx / 8] >> (4 * (idx % 8))) & 15;
      out[idx] = orc_e2m1_value(q) * (double)orc_nvfp4_block_scale(scales[r * nb + k / 16], g);
    }
  }
}

/* ------------------------------------------------------------------------ */
/* 7. Quantize-dequantize x_hat ([P2] fp_quantize_dequantize; used by the    */
/*    M=1 qqmm route before fp_qmv): quantize as in 5, decode as in 6.       */
/* ------------------------------------------------------------------------ */
void orc_nvfp4_quantize_dequantize(const void* x, int dt, int64_t rows,
                                   int64_t K, const float* g, void* out) {
  const int64_t nb = K / 16;
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t b = 0; b < nb; ++b) {
      uint32_t c[2];
      uint8_t s;
      /* one block is a 1 x 16 tensor: reuse the quantizer on it */
      float xv[16];
      for (int i = 0; i < 16; ++i) xv[i] = (float)orc_load(x, dt, r * K + b * 16 + i);
      orc_nvfp4_quantize(xv, ORC_F32, 1, 16, g, c, &s);
      orc_nvfp4_dequantize(c, &s, 1, 16, g, xv, ORC_F32);
      for (int i = 0; i < 16; ++i) orc_store(out, dt, r * K + b * 16 + i, xv[i]);
    }
  }
}

/* ------------------------------------------------------------------------ */
/* 8. MXFP8 quantize ([P2] fp_quantize_rowwise with bits 8 and the e8m0      */
/*    scale type; [P1] fp_quantize: group size 32 and 8 bits for mxfp8;      */
/*    [P3] mlxcel note: the E8M0 scale is rounded up).                       */
/*    Per row, per 32-element block:                                         */
/*      v   = a / 448             fp32                                       */
/*      s   = e8m0_ceil(v)                     -> scale byte                 */
/*      k   = 1 / 2^(s-127)       fp32 (exact power of two)                  */
/*      q_i = e4m3_rne_satfinite(x_i * k)      -> code byte                  */
/*    Codes: element 4w+i of a row in byte i of word w.                      */
/* ------------------------------------------------------------------------ */
void orc_mxfp8_quantize(const void* x, int dt, int64_t rows, int64_t K,
                        uint32_t* codes, uint8_t* scales) {
  const int64_t nb = K / 32;
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t b = 0; b < nb; ++b) {
      float xv[32];
      float a = 0.0f;
      for (int i = 0; i < 32; ++i) {
        xv[i] = (float)orc_load(x, dt, r * K + b * 32 + i);
        if (fabsf(xv[i]) > a) a = fabsf(xv[i]);
      }
      float v = a / 448.0f;
      int s = orc_e8m0_ceil(v);
      scales[r * nb + b] = (uint8_t)s;
      float k = 1.0f / (float)orc_e8m0_value(s);
      for (int i = 0; i < 32; ++i) {
        uint32_t q = (uint32_t)orc_e4m3_rne_satfinite(xv[i] * k);
        int64_t idx = r * K + b * 32 + i;
        codes[idx / 4] = (codes[idx / 4] & ~(0xFFu << (8 * (idx % 4)))) |
                         (q << (8 * (idx % 4)));
      }
    }
  }
}

/* MXFP8 dequantize ([P1] fp_dequantize fallback, e8m0 branch):
 * w_hat = T( e4m3(q) * 2^(s-127) ), product in fp32. */
void orc_mxfp8_dequantize(const uint32_t* codes, const uint8_t* scales,
                          int64_t rows, int64_t K, void* out, int out_dt) {
  const int64_t nb = K / 32;
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t k = 0; k < K; ++k) {
      int64_t idx = r * K + k;
      int q = (codes[idx / 4] >> (8 * (idx % 4))) & 255;
      float v = (float)orc_e4m3_value(q) * (float)orc_e8m0_value(scales[r * nb + k / 32]);
      orc_store(out, out_dt, idx, v);
    }
  }
}

/* Exact real value of each MXFP8 element, e4m3(q) * 2^(s-127), float64. */
void orc_mxfp8_decode_exact(const uint32_t* codes, const uint8_t* scales,
                            int64_t rows, int64_t K, double* out) {
  const int64_t nb = K / 32;
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t k = 0; k < K; ++k) {
      int64_t idx = r * K + k;
      int q = (codes[idx / 4] >> (8 * (idx % 4))) & 255;
      out[idx] = orc_e4m3_value(q) * orc_e8m0_value(scales[r * nb + k / 32]);
    }
  }
}

/* ------------------------------------------------------------------------ */
/* 8b. MXFP4 quantize ([P2] fp_quantize_rowwise / fp_quantize_dequantize     */
/*    with bits = 4 and the mx scale: the e8m0 scale type, no global scale). */
/*    Per 32-block (the MX block size; the pages' mx scale is the e8m0 one): */
/*      v   = max|x| / 6.0f                     fp32                          */
/*      s   = e8m0 of v, rounded up (the conversion that the MXFP8 path uses; */
/*            [P3] mlxcel note: CUDA rounds the E8M0 scale up)                */
/*      k   = 1 / 2^(s-127)       fp32 (exact power of two)                  */
/*      q_i = e2m1_rne_satfinite(x_i * k)      -> 4-bit code                 */
/*    Codes: element 8w+i of a row in bits 4i..4i+3 of word w (as NVFP4).    */
/*    Scales: LINEAR layout [rows, K/32].                                    */
/* ------------------------------------------------------------------------ */
void orc_mxfp4_quantize(const void* x, int dt, int64_t rows, int64_t K,
                        uint32_t* codes, uint8_t* scales) {
  const int64_t nb = K / 32;
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t b = 0; b < nb; ++b) {
      float xv[32];
      float a = 0.0f;
      for (int i = 0; i < 32; ++i) {
        xv[i] = (float)orc_load(x, dt, r * K + b * 32 + i);
        if (fabsf(xv[i]) > a) a = fabsf(xv[i]);
      }
      float v = a / 6.0f;
      int s = orc_e8m0_ceil(v);
      scales[r * nb + b] = (uint8_t)s;
      float k = 1.0f / (float)orc_e8m0_value(s);
      uint32_t w[4] = {0, 0, 0, 0};
      for (int i = 0; i < 32; ++i) {
        uint32_t q = (uint32_t)orc_e2m1_rne_satfinite(xv[i] * k);
        w[i / 8] |= q << (4 * (i % 8));
      }
      for (int j = 0; j < 4; ++j) codes[(r * K + b * 32) / 8 + j] = w[j];
    }
  }
}

/* MXFP4 dequantize ([P1] fp_dequantize fallback, e8m0 branch with 4-bit
 * codes): w_hat = T( e2m1(q) * 2^(s-127) ), product in fp32. */
void orc_mxfp4_dequantize(const uint32_t* codes, const uint8_t* scales,
                          int64_t rows, int64_t K, void* out, int out_dt) {
  const int64_t nb = K / 32;
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t k = 0; k < K; ++k) {
      int64_t idx = r * K + k;
      int q = (codes[idx / 8] >> (4 * (idx % 8))) & 15;
      float v = (float)orc_e2m1_value(q) * (float)orc_e8m0_value(scales[r * nb + k / 32]);
      orc_store(out, out_dt, idx, v);
    }
  }
}

/* Exact real value of each MXFP4 element, e2m1(q) * 2^(s-127), float64. */
void orc_mxfp4_decode_exact(const uint32_t* codes, const uint8_t* scales,
                            int64_t rows, int64_t K, double* out) {
  const int64_t nb = K / 32;
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t k = 0; k < K; ++k) {
      int64_t idx = r * K + k;
      int q = (codes[idx / 8] >> (4 * (idx % 8))) & 15;
      out[idx] = orc_e2m1_value(q) * orc_e8m0_value(scales[r * nb + k / 32]);
    }
  }
}

/* ------------------------------------------------------------------------ */
/* 8c. Stochastic rounding of the codes (the pages reserve it: [P2]           */
/*    fp_quantize_rowwise<..., USE_SR> with `rbits` "reserved for future     */
/*    use"; the reading taken here is the plain one):                        */
/*    the block scale s is computed exactly as in section 5; each scaled     */
/*    value t = x * k (fp32) goes to one of the two e2m1 magnitudes lo <= |t| */
/*    <= hi around it, up with probability (|t| - lo) / (hi - lo), decided by */
/*    8 random bits b: up iff b * 2^-8 < (|t| - lo) / (hi - lo) (both sides   */
/*    exact fp32 values; the difference is exact by Sterbenz, the division    */
/*    by a power of two).  |t| >= 6 gives 6, values on the grid are kept,     */
/*    the sign is kept (as in section 5).                                     */
/*    Random bits: one 32-bit word per group of 4 consecutive elements, as    */
/*    [P2] passes one `rbits` word to each 4-value conversion                 */
/*    (scale_cvt_Tx4_to_fp4x4<T, USE_SR>); element i takes byte i % 4 of word */
/*    i / 4, and word w is output w % 4 of Philox4x32-10 (Salmon, Moraes,     */
/*    Dror, Shaw, "Parallel random numbers: as easy as 1, 2, 3", SC 2011) at  */
/*    counter (w / 4 low, w / 4 high, 0, 0), key (seed low, seed high).       */
/* ------------------------------------------------------------------------ */
static void philox_round(uint32_t c[4], const uint32_t k[2]) {
  const uint64_t p0 = (uint64_t)0xD2511F53u * c[0];
  const uint64_t p1 = (uint64_t)0xCD9E8D57u * c[2];
  const uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
  const uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
  const uint32_t n0 = hi1 ^ c[1] ^ k[0], n1 = lo1, n2 = hi0 ^ c[3] ^ k[1], n3 = lo0;
  c[0] = n0; c[1] = n1; c[2] = n2; c[3] = n3;
}

void orc_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
  uint32_t c[4] = {ctr[0], ctr[1], ctr[2], ctr[3]};
  uint32_t k[2] = {key[0], key[1]};
  for (int r = 0; r < 10; ++r) {
    if (r > 0) { k[0] += 0x9E3779B9u; k[1] += 0xBB67AE85u; }
    philox_round(c, k);
  }
  for (int i = 0; i < 4; ++i) out[i] = c[i];
}

uint32_t orc_sr_bits(uint64_t seed, uint64_t i) {
  const uint64_t w = i >> 2, q = w >> 2;
  const uint32_t ctr[4] = {(uint32_t)q, (uint32_t)(q >> 32), 0u, 0u};
  const uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
  uint32_t out[4];
  orc_philox4x32_10(ctr, key, out);
  return (out[w & 3u] >> (8u * (uint32_t)(i & 3u))) & 0xFFu;
}

int orc_e2m1_sr_satfinite(float t, uint32_t r) {
  static const float mag[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
  const int neg = signbit(t) ? 8 : 0;
  const float a = fabsf(t);
  int m;
  if (a >= 6.0f) {
    m = 7;
  } else {
    int lo = 0;
    while (lo < 7 && mag[lo + 1] <= a) ++lo;  /* mag[lo] <= a < mag[lo + 1] */
    if (a == mag[lo]) {
      m = lo;
    } else {
      const float frac = (a - mag[lo]) / (mag[lo + 1] - mag[lo]);
      const float u = (float)r * 0x1p-8f;  /* r: 8 random bits */
      m = u < frac ? lo + 1 : lo;
    }
  }
  return neg | m;
}

void orc_nvfp4_quantize_sr(const void* x, int dt, int64_t rows, int64_t K, const float* g, uint64_t seed,
                           uint32_t* codes, uint8_t* scales) {
  const float E = encode_factor(g);
  const int64_t nb = K / 16;
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t b = 0; b < nb; ++b) {
      float xv[16];
      float a = 0.0f;
      for (int i = 0; i < 16; ++i) {
        xv[i] = (float)orc_load(x, dt, r * K + b * 16 + i);
        if (fabsf(xv[i]) > a) a = fabsf(xv[i]);
      }
      int s = nvfp4_scale_byte(a, E);
      scales[r * nb + b] = (uint8_t)s;
      float fs = (float)orc_e4m3_value(s);
      uint32_t w[2] = {0, 0};
      if (fs != 0.0f) {
        for (int i = 0; i < 16; ++i) {
          const uint64_t idx = (uint64_t)(r * K + b * 16 + i);
          uint32_t q = (uint32_t)orc_e2m1_sr_satfinite(nvfp4_scaled_value(xv[i], E, fs), orc_sr_bits(seed, idx));
          w[i / 8] |= q << (4 * (i % 8));
        }
      }
      codes[(r * K + b * 16) / 8] = w[0];
      codes[(r * K + b * 16) / 8 + 1] = w[1];
    }
  }
}

/* ------------------------------------------------------------------------ */
/* 9. Scale layout for the block-scaled MMA ([P5] qqmm_utils.cu comment:     */
/*    tmp = s.reshape(rb, 4, 32, cb, 4); tmp.transpose(0, 3, 2, 1, 4), and   */
/*    its worked index table; [P1] pad_and_swizzle_scales: pad to 128-row x  */
/*    4-column tiles, zero fill).                                            */
/*    Linear scale (r, c) of a [rows, cols] matrix goes to byte              */
/*      ((r/128) * (Cp/4) + c/4) * 512 + (r%32) * 16 + ((r%128)/32) * 4 + c%4 */
/*    of a [Rp, Cp] buffer, Rp = ceil128(rows), Cp = ceil4(cols); every      */
/*    byte not written is 0.                                                 */
/* ------------------------------------------------------------------------ */
void orc_swizzle_scales(const uint8_t* lin, int64_t rows, int64_t cols,
                        uint8_t* swz) {
  int64_t Rp = (rows + 127) / 128 * 128, Cp = (cols + 3) / 4 * 4;
  memset(swz, 0, (size_t)(Rp * Cp));
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t c = 0; c < cols; ++c) {
      int64_t off = ((r / 128) * (Cp / 4) + c / 4) * 512 + (r % 32) * 16 +
                    ((r % 128) / 32) * 4 + c % 4;
      swz[off] = lin[r * cols + c];
    }
  }
}

/* ------------------------------------------------------------------------ */
/* 10. Array helpers for the Python side                                     */
/* ------------------------------------------------------------------------ */
void orc_load_array(const void* x, int dt, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_load(x, dt, i);
}

void orc_store_array(const double* v, int64_t n, int dt, void* out) {
  for (int64_t i = 0; i < n; ++i) orc_store(out, dt, i, v[i]);
}
