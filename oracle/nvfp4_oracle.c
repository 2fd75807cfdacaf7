/*
 * NVFP4 reference oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, scalar C that defines what the NVFP4 hot path computes.  Only the
 * test suite, the package smoke check and the CPU-baseline leg of the benchmark
 * may load this library; the product path (the CUDA library behind
 * include/nvfp4.h) never calls it, and the two share no code.
 *
 * Sources (page title, section):
 *  - "Replay the Curvature: Accurate and Scalable NVFP4 Quantization ..." abstract:
 *    NVFP4 lets every 16 E2M1 values share one E4M3 block scale.
 *  - ARCQuant blog post (zizhi168.cn) section 1: E2M1 = 2-bit exponent, 1-bit
 *    mantissa; 16-element blocks each with an E4M3 scale; RTN as the baseline
 *    rounding.  Section 3.1: two-stage (main + residue) quantization, X_aug with
 *    K+S columns.  Section 4.2: E4M3 scale step 2^-3.
 *  - "ResServe: Accurate and Efficient FP4 LLM Inference with Residue
 *    Compensation" abstract: FP4 activation base plus an FP4-quantized residue.
 *
 * Readings where the pages are silent:
 *  - one FP32 per-tensor scale s = fl32(amax / (6*448));
 *  - block scale d = E4M3_RNE(fl32(amax_block / fl32(6*s))), saturating at 448;
 *  - element code c = E2M1_RNE(fl32(x * fl32(1 / fl32(d*s)))), ties to the even
 *    code, saturating at 6, sign bit kept (also for values that round to zero);
 *  - d == 0 (or s below 2^-110) gives inv = 0, i.e. all magnitudes 0;
 *  - residue r = fl32(x - fl32(fl32(v(c)*d) * s));
 *  - packed codes: element 2j in the low nibble of byte j.
 *
 * Rounding here is IEEE binary32/binary64 round-to-nearest-even; build with
 * -ffp-contract=off so no multiply-add is fused.
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#include <string.h>

#define ORC_API __attribute__((visibility("default")))

/* ------------------------------------------------------------------ E2M1 */

/* Magnitudes of the eight E2M1 codes 0..7 (sign is bit 3). */
static const double E2M1_MAG[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

ORC_API double orc_e2m1_decode(uint8_t c) {
  double v = E2M1_MAG[c & 7];
  return (c & 8) ? -v : v;
}

/* Nearest E2M1 magnitude by exhaustive search; ties go to the even code;
 * |q| >= 6 saturates to code 7; the sign bit of q is copied to bit 3. */
ORC_API uint8_t orc_e2m1_encode(float q) {
  uint8_t sign = signbit(q) ? 8 : 0;
  double a = fabs((double)q);
  if (a >= 6.0) return (uint8_t)(sign | 7);
  int best = 0;
  double best_dist = a;
  for (int c = 1; c < 8; ++c) {
    double dist = fabs(a - E2M1_MAG[c]);
    if (dist < best_dist || (dist == best_dist && (c & 1) == 0)) {
      best = c;
      best_dist = dist;
    }
  }
  return (uint8_t)(sign | best);
}

/* ------------------------------------------------------------------ E4M3 */

/* E4M3 (bias 7, no infinities, 0x7F/0xFF = NaN, max 448). */
ORC_API double orc_e4m3_decode(uint8_t b) {
  int e = (b >> 3) & 15, m = b & 7;
  if (e == 15 && m == 7) return NAN;
  double v = (e == 0) ? ldexp((double)m, -9) : ldexp((double)(8 + m), e - 10);
  return (b & 0x80) ? -v : v;
}

/* Nearest finite E4M3 value by exhaustive search over the 127 non-negative
 * finite encodings; ties go to the even encoding; |x| >= 448 saturates. */
ORC_API uint8_t orc_e4m3_encode(float x) {
  uint8_t sign = signbit(x) ? 0x80 : 0;
  double a = fabs((double)x);
  if (a >= 448.0) return (uint8_t)(sign | 0x7E);
  int best = 0;
  double best_dist = a;
  for (int b = 1; b < 0x7F; ++b) {
    double dist = fabs(a - orc_e4m3_decode((uint8_t)b));
    if (dist < best_dist || (dist == best_dist && (b & 1) == 0)) {
      best = b;
      best_dist = dist;
    }
  }
  return (uint8_t)(sign | best);
}

ORC_API void orc_e2m1_encode_array(const float* q, int64_t n, uint8_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e2m1_encode(q[i]);
}

ORC_API void orc_e4m3_encode_array(const float* x, int64_t n, uint8_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_encode(x[i]);
}

/* ------------------------------------------------------- per-tensor scale */

ORC_API float orc_amax(const float* x, int64_t rows, int64_t cols, int64_t ldx) {
  float m = 0.0f;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t k = 0; k < cols; ++k) {
      float a = fabsf(x[r * ldx + k]);
      if (a > m) m = a;
    }
  return m;
}

/* s = fl32(amax / 2688), 2688 = 6 (largest E2M1) * 448 (largest E4M3). */
ORC_API float orc_tensor_scale(float amax) {
  volatile float a = amax;
  return a / 2688.0f;
}

/* ---------------------------------------------------------- block quantizer */

/* Below this tensor scale every block is treated as all-zero (d = 0). */
#define ORC_MIN_TENSOR_SCALE 0x1p-110f

/* Quantize one 16-element block under tensor scale s.
 * codes_out: 16 unpacked codes; returns the E4M3 scale byte. */
static uint8_t quantize_block(const float* x, float s, uint8_t* codes_out) {
  float amax = 0.0f;
  for (int k = 0; k < 16; ++k) {
    float a = fabsf(x[k]);
    if (a > amax) amax = a;
  }
  uint8_t d_byte = 0;
  if (s >= ORC_MIN_TENSOR_SCALE) {
    volatile float t = 6.0f * s;
    volatile float ratio = amax / t;
    d_byte = orc_e4m3_encode(ratio);
  }
  float d = (float)orc_e4m3_decode(d_byte);
  float inv = 0.0f;
  if (d != 0.0f) {
    volatile float ds = d * s;
    inv = 1.0f / ds;
  }
  for (int k = 0; k < 16; ++k) {
    volatile float q = x[k] * inv;
    codes_out[k] = orc_e2m1_encode(q);
  }
  return d_byte;
}

/* Quantize rows x cols (cols % 16 == 0) with row stride ldx into packed codes
 * (rows x cols/2) and row-major block scales (rows x cols/16). */
ORC_API void orc_quantize(const float* x, int64_t rows, int64_t cols, int64_t ldx, float s,
                          uint8_t* codes, uint8_t* scales) {
  const int64_t nb = cols / 16;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    uint8_t c[16];
    for (int64_t b = 0; b < nb; ++b) {
      scales[r * nb + b] = quantize_block(x + r * ldx + b * 16, s, c);
      for (int j = 0; j < 8; ++j)
        codes[r * (cols / 2) + b * 8 + j] = (uint8_t)(c[2 * j] | (c[2 * j + 1] << 4));
    }
  }
}

/* fp32 dequantization as the residue stage uses it: fl32(fl32(v*d) * s). */
ORC_API void orc_dequant_f32(const uint8_t* codes, const uint8_t* scales, float s, int64_t rows,
                             int64_t cols, float* out) {
  const int64_t nb = cols / 16;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t k = 0; k < cols; ++k) {
      uint8_t byte = codes[r * (cols / 2) + k / 2];
      uint8_t c = (k & 1) ? (byte >> 4) : (byte & 15);
      float v = (float)orc_e2m1_decode(c);
      float d = (float)orc_e4m3_decode(scales[r * nb + k / 16]);
      volatile float vd = v * d;
      volatile float deq = vd * s;
      out[r * cols + k] = deq;
    }
}

/* Residue r = fl32(x - deq), deq as in orc_dequant_f32. */
ORC_API void orc_residue(const float* x, int64_t rows, int64_t cols, int64_t ldx,
                         const uint8_t* codes, const uint8_t* scales, float s, float* r_out) {
  const int64_t nb = cols / 16;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t k = 0; k < cols; ++k) {
      uint8_t byte = codes[r * (cols / 2) + k / 2];
      uint8_t c = (k & 1) ? (byte >> 4) : (byte & 15);
      float v = (float)orc_e2m1_decode(c);
      float d = (float)orc_e4m3_decode(scales[r * nb + k / 16]);
      volatile float vd = v * d;
      volatile float deq = vd * s;
      volatile float diff = x[r * ldx + k] - deq;
      r_out[r * cols + k] = diff;
    }
}

/* ---------------------------------------------------------------- RMSNorm */

/* Per-row RMS normalisation y = fl32(fl32(x * rinv) * gamma).
 *
 * The mean square is formed exactly, so its value does not depend on any
 * summation order: with e = floor(log2(max|x|)) of the row, each square is
 * truncated to an integer multiple of 2^(2e-34) (z = x * 2^(17-e),
 * q = floor(z*z) < 2^36) and the integers are summed exactly (the total stays
 * below 2^53 for rows of up to 2^16 elements).  Then, in binary64:
 *   mean = (Q * 2^(2e-34)) / K,   rinv = fl32(1 / sqrt(mean + eps)).
 * gamma == NULL means no gain.  rinv_out (may be NULL) receives rinv per row. */
ORC_API void orc_rmsnorm(const float* x, int64_t rows, int64_t cols, int64_t ldx,
                         const float* gamma, float eps, float* y, float* rinv_out) {
  for (int64_t r = 0; r < rows; ++r) {
    const float* xr = x + r * ldx;
    float amax = 0.0f;
    for (int64_t k = 0; k < cols; ++k) {
      float a = fabsf(xr[k]);
      if (a > amax) amax = a;
    }
    double q_sum = 0.0;
    int e = 0;
    if (amax > 0.0f) {
      e = ilogb(amax);
      for (int64_t k = 0; k < cols; ++k) {
        double z = ldexp((double)xr[k], 17 - e);
        q_sum += floor(z * z);
      }
    }
    double mean = ldexp(q_sum, 2 * e - 34) / (double)cols;
    double rinv_d = 1.0 / sqrt(mean + (double)eps);
    float rinv = (float)rinv_d;
    if (rinv_out) rinv_out[r] = rinv;
    for (int64_t k = 0; k < cols; ++k) {
      volatile float t = xr[k] * rinv;
      volatile float v = gamma ? t * gamma[k] : t;
      y[r * cols + k] = v;
    }
  }
}

/* ------------------------------------------------------------ fp64 dequant */

/* Exact binary64 dequantization deq = v(c) * d * s (row-major scales). */
ORC_API void orc_dequant_f64(const uint8_t* codes, const uint8_t* scales, float s, int64_t rows,
                             int64_t cols, double* out) {
  const int64_t nb = cols / 16;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t k = 0; k < cols; ++k) {
      uint8_t byte = codes[r * (cols / 2) + k / 2];
      uint8_t c = (k & 1) ? (byte >> 4) : (byte & 15);
      out[r * cols + k] =
          orc_e2m1_decode(c) * orc_e4m3_decode(scales[r * nb + k / 16]) * (double)s;
    }
}

/* ------------------------------------------------------------------ MXFP4
 * MX format (a NEXT row): 32-element blocks of E2M1 values sharing one E8M0
 * scale, a power of two 2^(b-127) for bytes 0..254 (255 is NaN); no tensor
 * scale (pages: ARCQuant blog sections 2.2 and 4.2 -- MX formats use E8M0
 * scales with step 2^1 and 32-element blocks).  The pages do not give the
 * scale rule; the reading taken is the shared-exponent rule of the MX format:
 * the block scale is 2^(floor(log2 amax_b) - 2), 2 being the exponent of the
 * largest E2M1 value, clamped to 2^-127..2^127, and 2^-127 for an all-zero
 * block.  Elements are E2M1_RNE(x / scale), saturating at +-6 (an element in
 * (6, 8) x scale clips to 6 x scale). */

ORC_API double orc_e8m0_decode(uint8_t b) {
  if (b == 255) return NAN;
  return ldexp(1.0, (int)b - 127);
}

/* E8M0 byte of one 32-element block (maximum magnitude amax). */
ORC_API uint8_t orc_mx_scale_byte(float amax) {
  if (!(amax > 0.0f)) return 0;                       /* all-zero block: 2^-127 */
  int e;
  (void)frexp((double)amax, &e);                      /* amax = f 2^e, f in [0.5, 1) */
  int x = (e - 1) - 2;                                /* floor(log2 amax) - 2 */
  if (x < -127) x = -127;
  if (x > 127) x = 127;
  return (uint8_t)(x + 127);
}

/* Quantize rows x cols (cols a multiple of 32) to unpacked E2M1 codes and
 * one E8M0 byte per 32-element block (row-major). */
ORC_API void orc_mx_quantize(const float* x, int64_t rows, int64_t cols, int64_t ldx, uint8_t* codes,
                             uint8_t* scales) {
  const int64_t nb = cols / 32;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t b = 0; b < nb; ++b) {
      const float* xb = x + r * ldx + b * 32;
      float amax = 0.0f;
      for (int i = 0; i < 32; ++i) {
        float a = fabsf(xb[i]);
        if (a > amax) amax = a;
      }
      const uint8_t sb = orc_mx_scale_byte(amax);
      scales[r * nb + b] = sb;
      const int e = (int)sb - 127;
      for (int i = 0; i < 32; ++i) {
        /* x / 2^e is exact in binary64; the E2M1 rounding sees the exact quotient */
        const double q = ldexp((double)xb[i], -e);
        codes[r * cols + b * 32 + i] = orc_e2m1_encode((float)q);
      }
    }
}

/* deq[r][k] = v(code) * 2^(b-127), in binary64 (exact). */
ORC_API void orc_mx_dequant_f64(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t cols,
                                double* out) {
  const int64_t nb = cols / 32;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t k = 0; k < cols; ++k)
      out[r * cols + k] = orc_e2m1_decode(codes[r * cols + k]) * orc_e8m0_decode(scales[r * nb + k / 32]);
}
