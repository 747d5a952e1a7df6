/*
 * qlinear_oracle.c -- plain, slow CPU oracle for the dynamically quantized
 * linear layer (FP8-E4M3 per-token / NVFP4 two-level block scaling, GEMM over
 * the decoded codes, fused epilogue).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library calls, links or
 * includes this file; only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark load it.  It shares no code, header, table or constant with
 * the CUDA path.
 *
 * What the method computes (sources):
 *  - "Cuantizacion Dinamica FP8" (wavespeed.ai, "Solucion de WaveSpeed para
 *    Acelerar la Generacion de Imagenes FLUX.1-dev"): weights and activations
 *    of the model are lowered to FP8 with scales found at run time, so that the
 *    8-bit tensor cores do the matmul.
 *  - algoritmulzilei.ro, "Accelerarea generarii de imagini cu FLUX 3 Image
 *    Klein", and bytechap.com, "Como funciona": NVFP4 lowers the precision of
 *    both weights and activations; the GEMMs carry fused epilogues (SwiGLU).
 *  - The bit formats (E4M3: S.EEEE.MMM bias 7, max 448, no Inf, only
 *    S.1111.111 is NaN; E2M1: S.EE.M bias 1, magnitudes 0..6) and the scale
 *    recipes (per-token scale = amax/448; NVFP4 global scale = amax/(448*6),
 *    16-element block scales in E4M3) are not on the pages; they follow the
 *    OCP 8-bit floating point and OCP MX format definitions.  Where a step is
 *    left open (division vs. reciprocal, all-zero rows, sign of zero), the
 *    plainest reading is taken and stated at the function.
 *
 * Arithmetic conventions: every float32 step is one IEEE binary32 operation
 * with round-to-nearest-even (build with -ffp-contract=off, no fast-math, so
 * no FMA contraction); the matmul and the epilogue run in binary64.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------- bf16 -- */

static float bf16_to_f32(uint16_t h) {
  uint32_t u = ((uint32_t)h) << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* ---------------------------------------------------------- decoding ---- */

/* E4M3 (OCP "E4M3FN"): sign, 4 exponent bits (bias 7), 3 mantissa bits.
 * exponent field 0 -> subnormal  m/8 * 2^-6 ; otherwise (1+m/8) * 2^(e-7);
 * S.1111.111 is NaN, there is no infinity. */
double or_e4m3_decode(uint8_t c) {
  int s = (c >> 7) & 1, e = (c >> 3) & 15, m = c & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0)
    v = ldexp((double)m / 8.0, -6);
  else
    v = ldexp(1.0 + (double)m / 8.0, e - 7);
  return s ? -v : v;
}

/* E2M1 (OCP MX FP4): sign, 2 exponent bits (bias 1), 1 mantissa bit.
 * exponent 0 -> subnormal m/2 ; otherwise (1+m/2) * 2^(e-1). */
double or_e2m1_decode(uint8_t c) {
  int s = (c >> 3) & 1, e = (c >> 1) & 3, m = c & 1;
  double v;
  if (e == 0)
    v = (double)m * 0.5;
  else
    v = ldexp(1.0 + (double)m / 2.0, e - 1);
  return s ? -v : v;
}

/* ---------------------------------------------------------- encoding ---- */

/* Round a non-negative double to the nearest integer, ties to even.  It is
 * only applied to exact power-of-two scalings of a float, so no rounding
 * happens before this step. */
static double rne_int(double q) {
  double f = floor(q);
  double r = q - f;
  if (r > 0.5) return f + 1.0;
  if (r < 0.5) return f;
  return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

/* float -> E4M3, round to nearest even, saturating to +-448 (satfinite).
 * NaN -> 0x7F with the sign; the sign of zero is kept. */
uint8_t or_e4m3_encode(float v) {
  uint32_t bits;
  memcpy(&bits, &v, 4);
  uint8_t sign = (bits >> 31) ? 0x80 : 0x00;
  if (isnan(v)) return (uint8_t)(sign | 0x7F);
  double a = fabs((double)v);
  if (a > 448.0) return (uint8_t)(sign | 0x7E);
  if (a < ldexp(1.0, -6)) {
    /* subnormal range: spacing 2^-9, code = round(a / 2^-9), 8 -> min normal */
    double q = rne_int(ldexp(a, 9));
    return (uint8_t)(sign | (uint8_t)q); /* q in 0..8, 8 == 0x08 == 2^-6 */
  }
  int e;
  (void)frexp(a, &e); /* a = f * 2^e, f in [0.5,1) -> unbiased exponent e-1 */
  int E = e - 1;      /* a in [2^E, 2^(E+1)) */
  double q = rne_int(ldexp(a, 3 - E)); /* in [8, 16] */
  if (q == 16.0) {
    q = 8.0;
    E += 1;
  }
  if (E > 8) return (uint8_t)(sign | 0x7E); /* cannot happen for a <= 448 */
  int efield = E + 7;
  int mfield = (int)q - 8;
  if (efield == 15 && mfield == 7) return (uint8_t)(sign | 0x7E);
  return (uint8_t)(sign | (efield << 3) | mfield);
}

/* float -> E2M1, round to nearest even, saturating to +-6.  NaN is outside
 * the format; it maps to +-6 here and is excluded from every test. */
uint8_t or_e2m1_encode(float v) {
  uint32_t bits;
  memcpy(&bits, &v, 4);
  uint8_t sign = (bits >> 31) ? 0x8 : 0x0;
  if (isnan(v)) return (uint8_t)(sign | 0x7);
  double a = fabs((double)v);
  if (a > 6.0) return (uint8_t)(sign | 0x7);
  if (a < 1.0) {
    /* subnormal range: spacing 0.5 */
    double q = rne_int(a * 2.0); /* 0, 1 or 2 (2 == 1.0 == code 2) */
    return (uint8_t)(sign | (uint8_t)q);
  }
  int e;
  (void)frexp(a, &e);
  int E = e - 1; /* 0, 1 or 2 */
  double q = rne_int(ldexp(a, 1 - E)); /* in [2, 4] */
  if (q == 4.0) {
    q = 2.0;
    E += 1;
  }
  if (E > 2) return (uint8_t)(sign | 0x7);
  return (uint8_t)(sign | ((E + 1) << 1) | ((int)q - 2));
}

/* Element-wise array forms of the two encoders (used by the exhaustive tests). */
void or_e4m3_encode_n(const float* v, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = or_e4m3_encode(v[i]);
}
void or_e2m1_encode_n(const float* v, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = or_e2m1_encode(v[i]);
}

/* ------------------------------------------- FP8 per-token quantization -- */

/* Per row r of x [rows, K] (bf16, row stride K):
 *   amax  = max_k |x|              (exact)
 *   s     = fl(amax / 448)         (stored scale)
 *   inv   = fl(448 / amax)         (0 when amax == 0)
 *   q[k]  = E4M3(fl(x[k] * inv))
 */
void or_quant_fp8_rows(const uint16_t* x, int64_t rows, int64_t K, uint8_t* codes,
                       float* scales) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    const uint16_t* xr = x + r * K;
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
      float a = fabsf(bf16_to_f32(xr[k]));
      if (a > amax) amax = a;
    }
    volatile float s = amax / 448.0f;
    volatile float inv = (amax > 0.0f) ? 448.0f / amax : 0.0f;
    scales[r] = s;
    for (int64_t k = 0; k < K; ++k) {
      volatile float y = bf16_to_f32(xr[k]) * inv;
      codes[r * K + k] = or_e4m3_encode(y);
    }
  }
}

/* ------------------------------------------------ NVFP4 quantization ----- */

/* Largest |x| over the whole tensor (exact). */
float or_tensor_amax(const uint16_t* x, int64_t n) {
  float amax = 0.0f;
  for (int64_t i = 0; i < n; ++i) {
    float a = fabsf(bf16_to_f32(x[i]));
    if (a > amax) amax = a;
  }
  return amax;
}

/* Two-level NVFP4 quantization of x [rows, K] (K % 16 == 0):
 *   A     = max |x| over the tensor (given)
 *   G     = fl(A / 2688)          fp32 global (decode) scale, 2688 = 448 * 6
 *   enc   = fl(448 / A)           (0 when A == 0)
 * per 16-element block b of a row:
 *   sb    = E4M3(fl(amax_b * enc))                 block scale code
 *   inv_b = fl(1 / fl(dec(sb) * G))                (0 when the product is 0)
 *   q[k]  = E2M1(fl(x[k] * inv_b))
 * codes: packed two per byte, element 2j in the low nibble, 2j+1 in the high
 * nibble, row stride K/2.  sf: one byte per block, logical order [rows, K/16].
 */
void or_quant_nvfp4(const uint16_t* x, int64_t rows, int64_t K, float A, uint8_t* codes,
                    uint8_t* sf, float* G_out) {
  volatile float G = A / 2688.0f;
  volatile float enc = (A > 0.0f) ? 448.0f / A : 0.0f;
  *G_out = G;
  int64_t nb = K / 16;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t b = 0; b < nb; ++b) {
      const uint16_t* xb = x + r * K + b * 16;
      float amax_b = 0.0f;
      for (int j = 0; j < 16; ++j) {
        float a = fabsf(bf16_to_f32(xb[j]));
        if (a > amax_b) amax_b = a;
      }
      volatile float t = amax_b * enc;
      uint8_t sb = or_e4m3_encode(t);
      sf[r * nb + b] = sb;
      volatile float dsb = (float)or_e4m3_decode(sb);
      volatile float den = dsb * G;
      volatile float inv = (den > 0.0f) ? 1.0f / den : 0.0f;
      for (int j = 0; j < 16; j += 2) {
        volatile float y0 = bf16_to_f32(xb[j]) * inv;
        volatile float y1 = bf16_to_f32(xb[j + 1]) * inv;
        uint8_t lo = or_e2m1_encode(y0), hi = or_e2m1_encode(y1);
        codes[r * (K / 2) + (b * 16 + j) / 2] = (uint8_t)(lo | (hi << 4));
      }
    }
  }
}

/* --------------------------------------------------------------- GEMMs --- */

/* FP8 GEMM over the decoded codes, for the listed activation rows:
 *   y[i, n] = ( sum_k dec(qa[row_i, k]) * dec(qw[n, k]) ) * sa[row_i] * sw[n]
 * qa [*, K] row-major, qw [N, K] row-major (both K-contiguous).  Products of
 * two E4M3 values are multiples of 2^-18 bounded by 448^2, so for K up to
 * about 2^32 the binary64 sum is exact and order independent. */
void or_gemm_fp8(const uint8_t* qa, const float* sa, const uint8_t* qw, const float* sw,
                 int64_t K, int64_t N, const int64_t* rows, int64_t nrows, double* y) {
  double lut[256];
  for (int c = 0; c < 256; ++c) lut[c] = or_e4m3_decode((uint8_t)c);
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < nrows; ++i) {
    const uint8_t* a = qa + rows[i] * K;
    for (int64_t n = 0; n < N; ++n) {
      const uint8_t* w = qw + n * K;
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k) acc += lut[a[k]] * lut[w[k]];
      y[i * N + n] = acc * (double)sa[rows[i]] * (double)sw[n];
    }
  }
}

/* Weight-only GEMM: bf16 activations (not quantized) against decoded FP8
 * weights, for the listed activation rows:
 *   y[i, n] = ( sum_k x[row_i, k] * dec(qw[n, k]) ) * sw[n]
 * x bf16 [*, K] row-major, qw [N, K].  A bf16 value times an E4M3 value has
 * at most 12 significant bits, so each product is exact in binary64; the sum
 * is rounded to binary64 (ordered by k). */
void or_gemm_w8a16(const uint16_t* x, const uint8_t* qw, const float* sw, int64_t K, int64_t N,
                   const int64_t* rows, int64_t nrows, double* y) {
  double lut[256];
  for (int c = 0; c < 256; ++c) lut[c] = or_e4m3_decode((uint8_t)c);
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < nrows; ++i) {
    const uint16_t* a = x + rows[i] * K;
    for (int64_t n = 0; n < N; ++n) {
      const uint8_t* w = qw + n * K;
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k) acc += (double)bf16_to_f32(a[k]) * lut[w[k]];
      y[i * N + n] = acc * (double)sw[n];
    }
  }
}

/* NVFP4 GEMM over the decoded codes, for the listed activation rows:
 *   y[i, n] = G_a * G_w * sum_b dec(sfa[row,b]) * dec(sfw[n,b])
 *                           * sum_{k in block b} dec(qa[row,k]) * dec(qw[n,k])
 * qa/qw packed as produced by or_quant_nvfp4, sfa/sfw logical [*, K/16]. */
void or_gemm_nvfp4(const uint8_t* qa, const uint8_t* sfa, float Ga, const uint8_t* qw,
                   const uint8_t* sfw, float Gw, int64_t K, int64_t N, const int64_t* rows,
                   int64_t nrows, double* y) {
  double lut4[16], lut8[256];
  for (int c = 0; c < 16; ++c) lut4[c] = or_e2m1_decode((uint8_t)c);
  for (int c = 0; c < 256; ++c) lut8[c] = or_e4m3_decode((uint8_t)c);
  int64_t nb = K / 16, kh = K / 2;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < nrows; ++i) {
    int64_t r = rows[i];
    for (int64_t n = 0; n < N; ++n) {
      double acc = 0.0;
      for (int64_t b = 0; b < nb; ++b) {
        double blk = 0.0;
        for (int j = 0; j < 8; ++j) {
          uint8_t pa = qa[r * kh + b * 8 + j], pw = qw[n * kh + b * 8 + j];
          blk += lut4[pa & 15] * lut4[pw & 15];
          blk += lut4[pa >> 4] * lut4[pw >> 4];
        }
        acc += lut8[sfa[r * nb + b]] * lut8[sfw[n * nb + b]] * blk;
      }
      y[i * N + n] = acc * (double)Ga * (double)Gw;
    }
  }
}

/* ----------------------------------------------------------- epilogues -- */

enum { OR_EPI_BIAS = 0, OR_EPI_BIAS_GELU = 1, OR_EPI_SWIGLU = 2,
       OR_EPI_BIAS_GATED_RESIDUAL = 3, OR_EPI_SPLIT_BIAS_GELU = 4 };

/* GELU, tanh form (Hendrycks & Gimpel, "Gaussian Error Linear Units"):
 *   0.5 v (1 + tanh( sqrt(2/pi) (v + 0.044715 v^3) )) */
double or_gelu_tanh(double v) {
  const double c = sqrt(2.0 / M_PI);
  return 0.5 * v * (1.0 + tanh(c * (v + 0.044715 * v * v * v)));
}

/* SiLU (swish): v / (1 + e^-v) */
double or_silu(double v) { return v / (1.0 + exp(-v)); }

/* Fused epilogue on y [nrows, N] (binary64) -> out [nrows, Nout] (binary64,
 * before any bf16 rounding).  bias bf16 [N] (NULL = 0); gate bf16 [Nout];
 * residual bf16 [*, Nout] indexed by rows[i].
 *   BIAS                : out = y + b
 *   BIAS_GELU           : out = gelu_tanh(y + b)
 *   SWIGLU              : Nout = N/2, out[:, j] = silu(y_g) * y_u with
 *                         y_g = y[:, j] + b[j], y_u = y[:, Nout+j] + b[Nout+j]
 *   BIAS_GATED_RESIDUAL : out = residual + gate * (y + b)
 *   SPLIT_BIAS_GELU     : n < split_col ? y + b : gelu_tanh(y + b)
 */
void or_epilogue(int kind, const double* y, int64_t nrows, int64_t N, const uint16_t* bias,
                 const uint16_t* residual, const int64_t* rows, const uint16_t* gate,
                 int64_t split_col, double* out) {
  int64_t Nout = (kind == OR_EPI_SWIGLU) ? N / 2 : N;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < nrows; ++i) {
    for (int64_t n = 0; n < Nout; ++n) {
      double v = y[i * N + n] + (bias ? (double)bf16_to_f32(bias[n]) : 0.0);
      double o;
      switch (kind) {
        case OR_EPI_BIAS:
          o = v;
          break;
        case OR_EPI_BIAS_GELU:
          o = or_gelu_tanh(v);
          break;
        case OR_EPI_SWIGLU: {
          double u = y[i * N + Nout + n] + (bias ? (double)bf16_to_f32(bias[Nout + n]) : 0.0);
          o = or_silu(v) * u;
          break;
        }
        case OR_EPI_BIAS_GATED_RESIDUAL:
          o = (double)bf16_to_f32(residual[rows[i] * Nout + n]) +
              (double)bf16_to_f32(gate[n]) * v;
          break;
        case OR_EPI_SPLIT_BIAS_GELU:
          o = (n < split_col) ? v : or_gelu_tanh(v);
          break;
        default:
          o = NAN;
      }
      out[i * Nout + n] = o;
    }
  }
}

/* QKV projection epilogue with query/key normalization and rotary position
 * embedding.  The fused QKV GEMM of algoritmulzilei.ro's "Accelerarea
 * generarii de imagini cu FLUX 3 Image Klein pe GPU-urile Blackwell" applies
 * "query/key normalization and rotary position embeddings"; the page gives no
 * formula, so the plain readings are taken:
 *   y [nrows, N], N = 3 * H * D: columns [0, N/3) are q, [N/3, 2N/3) are k,
 *   [2N/3, N) are v, each H heads of D consecutive columns.
 *   Every column: v = y + b (bias bf16 [N], NULL = 0).
 *   q and k heads: RMS normalization over the head's D values,
 *     u_d = v_d / sqrt(mean_d(v_d^2) + eps) * w_d   (w = qw or kw, bf16 [D]),
 *   then rotary embedding of the pairs (u_{2i}, u_{2i+1}), i < D/2:
 *     (a, b) -> (a cos - b sin, a sin + b cos),
 *   cos = rc[rows[r] * D/2 + i], sin = rs[rows[r] * D/2 + i] (fp32 tables,
 *   one angle per token and pair; the positions are the caller's).
 * out [nrows, N] binary64, before bf16 rounding. */
void or_qkv_norm_rope(const double* y, int64_t nrows, int64_t N, int64_t D,
                      const uint16_t* bias, const uint16_t* qw, const uint16_t* kw,
                      const float* rc, const float* rs, const int64_t* rows, double eps,
                      double* out) {
  const int64_t qk = 2 * (N / 3);
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < nrows; ++r) {
    for (int64_t n = 0; n < N; ++n)
      out[r * N + n] = y[r * N + n] + (bias ? (double)bf16_to_f32(bias[n]) : 0.0);
    for (int64_t h0 = 0; h0 < qk; h0 += D) {
      double* u = out + r * N + h0;
      const uint16_t* w = (h0 < N / 3) ? qw : kw;
      double ss = 0.0;
      for (int64_t d = 0; d < D; ++d) ss += u[d] * u[d];
      const double scale = 1.0 / sqrt(ss / (double)D + eps);
      for (int64_t d = 0; d < D; ++d) u[d] = u[d] * scale * (double)bf16_to_f32(w[d]);
      for (int64_t i = 0; i < D / 2; ++i) {
        const double c = rc[rows[r] * (D / 2) + i], sn = rs[rows[r] * (D / 2) + i];
        const double a = u[2 * i], b = u[2 * i + 1];
        u[2 * i] = a * c - b * sn;
        u[2 * i + 1] = a * sn + b * c;
      }
    }
  }
}

/* Number of OpenMP threads the oracle runs with (1 without OpenMP). */
int or_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
